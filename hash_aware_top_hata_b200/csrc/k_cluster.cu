// k_cluster.cu -- the whole decode step in ONE kernel for heads whose cache
// fits a thread-block cluster: one cluster of C <= 8 CTAs per (batch row,
// KV head), CTA r owning an equal range of up to 16384 tokens of the slab.
//
// HATA review page (arXiv 2506.02572): "What carries the argument" (hash
// q, XOR + popcount against every cached key code, attention over the
// top-k keys only), Figure 2 caption (Algorithm 1: the key code cache,
// extended by one token per decode step), referee report, major comment 1
// (Algorithm 3: a threshold top-k over the r + 1 Hamming values; boundary
// ties here go to the lower token index).
//
// Small problems (a few heads, tens of thousands of keys) are bound by the
// latency of kernel boundaries, not by bytes: the multi-kernel step runs
// four or five dependent kernels, each paying its launch, its first memory
// round trip and its grid-completion flush.  Here each CTA runs every step
// on its own tokens and the CTAs of a cluster meet twice, through
// distributed shared memory instead of global memory:
//
//   1. every CTA hashes the G query heads of its KV head (the same fp32
//      chain as the prep kernel, so codes are bit-exact) and, if its range
//      holds the new token, appends its code and K/V rows;
//   2. it scores its tokens against all G heads: distances stay in shared
//      memory (copied to the caller's rows only when asked for), counts go
//      to a shared histogram per head;
//   3. cluster barrier; every CTA reads the C histograms of its head group
//      from the other CTAs' shared memory: the sum gives T and #(< T), the
//      CTAs before it the keys below T and at T it must skip -- the same
//      placement arithmetic as the tile CTAs of the selection kernel;
//   4. it selects its share (byte-wise masks, one block scan per head) into
//      the head's index list, ascending;
//   5. its first 8 warps gather and attend its selected rows (G heads side
//      by side, 8 / G warps each, the tensor-core stage of attend_common.cuh) and
//      merge them into one partial (m, l, acc) per head, written into the
//      shared memory of the cluster's first CTA;
//   6. cluster barrier; the first CTA merges the C partials per head into
//      out.
//
// Every CTA of a cluster is resident at once (the hardware schedules a
// cluster as a unit), so the two barriers cannot wait on a CTA that never
// runs.  bf16 or fp32 K/V, r = 128, G in {1, 2, 4}.  512 threads: all 16 warps scan
// and select (the scan is latency-bound, so warps matter), the first 8
// attend (their rings take the 128 KB that held W_H and the code chunks);
// 126 registers, no spills.
#include <cooperative_groups.h>
#include <cuda_bf16.h>

#include <map>
#include <mutex>
#include <utility>

#include "hata_internal.cuh"
#include "async_copy.cuh"
#include "attend_common.cuh"
#include "score_common.cuh"
#include "select_common.cuh"

namespace hata {
namespace {

namespace cg = cooperative_groups;

constexpr int kCThreads = 512;
constexpr int kCWarps = kCThreads / 32;      // 16 warps scan and select
constexpr int kAWarps = 8;                   // the first 8 of them attend
constexpr int kCRing = 2;                    // attention stages per warp ring
constexpr size_t kCRingBytes = size_t(kAWarps) * kCRing * tc::kStageBytes;

// kM: a CTA holds up to 8192 kM tokens, 16 kM per thread in the selection
// (the plan uses kM = 2: 32 tokens, one mask word, per thread)
template <int kM>
struct ClusterSmem {
    static constexpr int kTok = 8192 * kM;
    static constexpr int kDistBytes = kClusterMaxG * kTok > kD * kRbit * 4 ? kClusterMaxG * kTok
                                                                          : kD * kRbit * 4;
    uint8_t ring[kCRingBytes];                        // code chunks (phase 2), attention rings
                                                      // (phase 5)
    union {
        uint8_t dist[kClusterMaxG][kTok];             // this CTA's distances (phase 2 on)
        uint8_t w[kDistBytes];                        // W_H of the KV head (phase 1)
    };
    uint32_t hist[kClusterMaxG][kHistStride];         // and their histograms
    float q[kClusterMaxG][kD];                        // the query rows
    float part[kAWarps][kPartStride];                 // attention warp partials
    float merged[kClusterMaxC][kClusterMaxG][kPartStride];  // CTA partials (first CTA)
    uint32_t qcode[kClusterMaxG][4];
    uint32_t kcode[4];                                // the appended key's code
    int2 scan[kCWarps + 1];
    int sel[kClusterMaxG][4];                         // T, n_less, start, count per head
};

// The fp32 chain acc = fmaf(x_i, W[i][j], acc), i = 0..127, of bit j of the
// code of row x with one head's W ([128][128]); both in shared memory.
__device__ __forceinline__ bool hash_bit(const float *x, const float *Ws, int j)
{
    float acc = 0.0f;
#pragma unroll 16
    for (int i = 0; i < kD; ++i) acc = __fmaf_rn(x[i], Ws[i * kRbit + j], acc);
    return acc > 0.0f;
}

constexpr int kChunk = 4096;  // tokens per code chunk (64 KB) of the scan

// Copy chunk c of this CTA's key codes (thread t: tokens t + 256 j of the
// chunk, 16 bytes each) into `dst` (64 KB of shared memory), zero-filling
// tokens that hold no key; always commits one group.
__device__ __forceinline__ void copy_chunk(const uint4 *codes, int c, int nloc, uint32_t dst, int tid)
{
    asm volatile("" ::: "memory");  // earlier reads of the slot stay before the copies
#pragma unroll
    for (int j = 0; j < kChunk / kCThreads; ++j) {
        const int t = kChunk * c + tid + kCThreads * j;
        const bool in = t < nloc;
        cp_async16_zfill(dst + 16u * uint32_t(tid + kCThreads * j), in ? codes + t : codes,
                         in ? 16u : 0u);
    }
    cp_async_commit();
}

template <int kM, bool kBF16>
__global__ void __launch_bounds__(kCThreads, 1) cluster_step_kernel(ClusterArgs a)
{
    constexpr int kCTok = ClusterSmem<kM>::kTok;  // token capacity of a CTA
    constexpr int kCPer = kCTok / kCThreads;      // tokens per thread in the selection
    constexpr int kGroups = kCPer / 32;
    extern __shared__ __align__(128) uint8_t smem_raw[];
    ClusterSmem<kM> &S = *reinterpret_cast<ClusterSmem<kM> *>(smem_raw);
    cg::cluster_group cl = cg::this_cluster();
    const int C = int(cl.num_blocks());
    const int rank = int(cl.block_rank());
    const int slab_id = int(blockIdx.x) / C;  // b * H_kv + h
    const int b = slab_id / a.H_kv, h = slab_id - b * a.H_kv;
    const int G = a.G;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t bh0 = int64_t(b) * a.H_q + int64_t(h) * G;  // first query head
    const int64_t slab = (int64_t(b) * a.H_kv + h) * a.n_cap;  // first K/V row and code
    const int32_t sl = a.seq_len[b];
    const int len = int(clamp_len(sl, a.max_seq_len, a.n_cap));
    const int t_beg = rank * a.tok_per_cta;                    // this CTA's range of the slab
    const int nloc = min(max(len - t_beg, 0), a.tok_per_cta);  // the tokens of it that hold keys
    const float *Wh = a.W + size_t(h) * kD * kRbit;

    // ---- 1. query rows, their codes, the append, the flags ----
    // W_H of the KV head (64 KB) goes to the distance area (written from
    // phase 2 on), the first two code chunks (2 x 64 KB) to the attention
    // rings (unused until phase 5): all three copies start now and overlap
    // the query loads and the hashing
    const uint32_t ring0 = smem_addr(S.ring);              // even chunks
    const uint32_t ring1 = ring0 + uint32_t(kChunk * 16);  // odd chunks
    const uint4 *codes = reinterpret_cast<const uint4 *>(a.codes) + slab + t_beg;
    for (int i = tid; i < kD * kRbit / 4; i += kCThreads)
        cp_async16(S.w + 16 * i, Wh + 4 * i);
    cp_async_commit();
    constexpr int kChunks = kCTok / kChunk;
    copy_chunk(codes, 0, nloc, ring0, tid);
    if (kChunks > 1)
        copy_chunk(codes, 1, nloc, ring1, tid);
    else
        cp_async_commit();
    const float *Ws = reinterpret_cast<const float *>(S.w);
    for (int i = tid; i < G * kD; i += kCThreads)
        S.q[i / kD][i % kD] = a.q[(bh0 + i / kD) * kD + i % kD];
    for (int i = tid; i < G * kHistStride; i += kCThreads) (&S.hist[0][0])[i] = 0u;
    if (a.ws_header && blockIdx.x == 0 && tid == 0) {
        a.ws_header[0] = kWsMagic;
        a.ws_header[1] = uint32_t(a.B);
    }
    if (rank == 0 && h == 0 && tid == 0) {
        uint32_t f = 0;
        if (sl < 0 || sl > a.max_seq_len || sl > a.n_cap) f |= HATA_FLAG_SEQ_LEN_RANGE;
        if (a.k_new && (int64_t(sl) - 1 < 0 || int64_t(sl) - 1 >= a.n_cap)) f |= HATA_FLAG_POS_RANGE;
        a.flags[b] = f;
    }
    // the new token (at seq_len - 1) belongs to the CTA whose range holds it;
    // a position past every range (a length beyond max_seq_len) to the last
    const int64_t pos = int64_t(sl) - 1;
    const bool append = a.k_new && pos >= 0 && pos < a.n_cap &&
                        min(int(pos / a.tok_per_cta), C - 1) == rank;
    cp_async_wait<2>();  // this thread's copies of W
    __syncthreads();
    // G chains of 128 steps per bit over the 512 threads (G <= 4: one each),
    // plus the appended key's 128 in the CTA that owns it
    {
        const int j = tid & (kRbit - 1);
        for (int g = tid >> 7; g < G; g += kCThreads / kRbit) {
            const bool bit = hash_bit(S.q[g], Ws, j);
            const uint32_t word = __ballot_sync(0xffffffffu, bit);
            if (lane == 0) S.qcode[g][j >> 5] = word;
        }
    }
    if (append) {
        // stage k_new (bf16 widened exactly, or fp32) in the merge buffer,
        // then hash
        float *xk = S.merged[0][0];
        const int64_t e0 = (int64_t(b) * a.H_kv + h) * kD;
        for (int i = tid; i < kD; i += kCThreads)
            xk[i] = kBF16 ? __uint_as_float(uint32_t(static_cast<const uint16_t *>(a.k_new)[e0 + i]) << 16)
                          : static_cast<const float *>(a.k_new)[e0 + i];
        __syncthreads();
        if (tid < kRbit) {
            const bool bit = hash_bit(xk, Ws, tid);
            const uint32_t word = __ballot_sync(0xffffffffu, bit);
            if (lane == 0) {
                S.kcode[tid >> 5] = word;  // the scan takes it from here: the copy of
                                           // its slot may predate this write
                a.codes[(slab + pos) * 4 + (tid >> 5)] = word;
            }
        }
        if (a.v_new && tid >= kRbit && tid < 2 * kRbit) {  // K and V rows of the new token
            const int e = tid - kRbit;  // 0..127
            if (kBF16) {
                static_cast<uint16_t *>(a.K)[(slab + pos) * kD + e] =
                    static_cast<const uint16_t *>(a.k_new)[e0 + e];
                static_cast<uint16_t *>(a.V)[(slab + pos) * kD + e] =
                    static_cast<const uint16_t *>(a.v_new)[e0 + e];
            } else {
                static_cast<float *>(a.K)[(slab + pos) * kD + e] = xk[e];
                static_cast<float *>(a.V)[(slab + pos) * kD + e] =
                    static_cast<const float *>(a.v_new)[e0 + e];
            }
        }
    }
    __syncthreads();
    if (a.q_out && rank == 0)
        for (int i = tid; i < G * 4; i += kCThreads) a.q_out[(bh0 + i / 4) * 4 + i % 4] = S.qcode[i / 4][i % 4];

    // ---- 2. scores of this CTA's tokens: chunks of 4096 through the rings,
    // two chunks in flight (thread t reads back only the tokens it copied) ----
    {
        uint4 qv[kClusterMaxG];
        uint2 qp[kClusterMaxG];
#pragma unroll
        for (int g = 0; g < kClusterMaxG; ++g) {
            const uint32_t *c = S.qcode[g < G ? g : 0];
            qv[g] = make_uint4(c[0], c[1], c[2], c[3]);
            qp[g] = make_uint2(c[0] ^ c[1], c[2] ^ c[3]);
        }
        // the appended token's position in this CTA's range, if it holds it
        const int lp = append ? int(pos) - t_beg : -1;
        const uint4 kap = append ? make_uint4(S.kcode[0], S.kcode[1], S.kcode[2], S.kcode[3])
                                 : make_uint4(0u, 0u, 0u, 0u);
        for (int c = 0; c < kChunks; ++c) {
            cp_async_wait<1>();  // this thread's copies of chunk c (chunk c + 1 may fly)
            const uint4 *mine = reinterpret_cast<const uint4 *>(S.ring + (c & 1) * kChunk * 16);
#pragma unroll 4
            for (int j = 0; j < kChunk / kCThreads; ++j) {
                const int tl = tid + kCThreads * j;     // in the chunk
                const int t = kChunk * c + tl;          // in the CTA's range
                uint4 kv = mine[tl];
                if (t == lp) kv = kap;
                const uint32_t k01 = kv.x ^ kv.y, k23 = kv.z ^ kv.w;
#pragma unroll
                for (int g = 0; g < kClusterMaxG; ++g) {
                    if (g < G) {
                        uint8_t byte = kDistPad;
                        if (t < nloc) {
                            const int d = hamming128(kv, k01, k23, qv[g], qp[g]);
                            atomicAdd(&S.hist[g][d], 1u);
                            byte = uint8_t(d);
                        }
                        S.dist[g][t] = byte;
                    }
                }
            }
            // chunk c + 2 into the slot chunk c leaves (this thread read only
            // the tokens it copied itself)
            if (c + 2 < kChunks)
                copy_chunk(codes, c + 2, nloc, (c & 1) ? ring1 : ring0, tid);
            else
                cp_async_commit();
        }
        cp_async_wait<0>();
    }
    __syncthreads();
    if (a.dist) {  // the caller's distance rows: this CTA's part of them (the last
                   // CTA's up to the row's end)
        const int64_t row_len = a.dist_row;
        const int64_t n_out =
            rank == C - 1 ? row_len - t_beg : min(int64_t(a.tok_per_cta), row_len - t_beg);
        for (int g = 0; g < G; ++g) {
            uint8_t *dst = a.dist + (bh0 + g) * row_len + t_beg;
            // past the CTA's capacity (the last CTA, rows longer than the
            // context): pad bytes
            for (int64_t i = int64_t(tid) * 16; i < n_out; i += int64_t(kCThreads) * 16)
                *reinterpret_cast<uint4 *>(dst + i) =
                    i < kCTok ? *reinterpret_cast<const uint4 *>(&S.dist[g][i])
                              : make_uint4(~0u, ~0u, ~0u, ~0u);
        }
    }

    // ---- 3. the cluster's histograms: T, #(< T), this CTA's placement ----
    cl.sync();
    const int k_eff = min(a.topk, len);
    if (warp < G) {
        const int g = warp;
        // lane l: bins 5l .. 5l+4, summed over the C CTAs; before: the CTAs
        // ranked below this one
        uint32_t tot[5] = {0u, 0u, 0u, 0u, 0u}, pre[5] = {0u, 0u, 0u, 0u, 0u};
        for (int r = 0; r < C; ++r) {
            const uint32_t *hr = cl.map_shared_rank(&S.hist[g][0], r);
#pragma unroll
            for (int e = 0; e < 5; ++e) {
                const uint32_t v = lane * 5 + e < kBins ? hr[lane * 5 + e] : 0u;
                tot[e] += v;
                pre[e] += r < rank ? v : 0u;
            }
        }
        const uint32_t run = tot[0] + tot[1] + tot[2] + tot[3] + tot[4];
        uint32_t acc = uint32_t(warp_inclusive_scan(int(run))) - run;
        int Tl = -1;
        uint32_t less_l = 0;
#pragma unroll
        for (int e = 0; e < 5; ++e) {
            if (Tl < 0 && lane * 5 + e < kBins && acc + tot[e] >= uint32_t(k_eff)) {
                Tl = lane * 5 + e;
                less_l = acc;
            }
            acc += tot[e];
        }
        const unsigned found = __ballot_sync(0xffffffffu, Tl >= 0);
        const int src = found ? __ffs(int(found)) - 1 : 0;
        const int T = found ? __shfl_sync(0xffffffffu, Tl, src) : kBins - 1;
        const int n_less = found ? __shfl_sync(0xffffffffu, int(less_l), src) : 0;
        int l = 0, q = 0;
#pragma unroll
        for (int e = 0; e < 5; ++e) {
            const int bin = lane * 5 + e;
            l += bin < T ? int(pre[e]) : 0;
            q += bin == T ? int(pre[e]) : 0;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            l += __shfl_xor_sync(0xffffffffu, l, o);
            q += __shfl_xor_sync(0xffffffffu, q, o);
        }
        if (lane == 0) {
            S.sel[g][0] = T;
            S.sel[g][1] = n_less;
            S.sel[g][2] = l;  // keys below T in the CTAs before this one
            S.sel[g][3] = q;  // keys at T in the CTAs before this one
        }
    }
    __syncthreads();

    // ---- 4. this CTA's share of every head's list (tokens 32 tid ...) ----
    for (int g = 0; g < G; ++g) {
        const int T = S.sel[g][0], n_less = S.sel[g][1];
        const int less_before = S.sel[g][2], ties_before = S.sel[g][3];
        const int r_ties = k_eff - n_less;  // boundary keys over the whole head
        const int ties_done = ties_before < r_ties ? ties_before : r_ties;
        int32_t *idx = a.idx + (bh0 + g) * a.topk;
        if (rank == 0)
            for (int i = k_eff + tid; i < a.topk; i += kCThreads) idx[i] = -1;
        uint32_t lt[kGroups], eq[kGroups];
        int n_lt = 0, n_eq = 0;
#pragma unroll
        for (int m = 0; m < kGroups; ++m) {
            lt[m] = eq[m] = 0u;
            if (k_eff > 0) {
                const uint8_t *dm = &S.dist[g][kCPer * tid + 32 * m];
                const uint4 v0 = *reinterpret_cast<const uint4 *>(dm);
                const uint4 v1 = *reinterpret_cast<const uint4 *>(dm + 16);
                const uint32_t dw[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
                const uint32_t T4 = uint32_t(T) * 0x01010101u, T4p = T4 + 0x01010101u;
                if (T < kRbit)
                    group_masks<false>(dw, T4, T4p, lt[m], eq[m]);
                else
                    group_masks<true>(dw, T4, T4p, lt[m], eq[m]);
            }
            n_lt += __popc(lt[m]);
            n_eq += __popc(eq[m]);
        }
        int tile_lt, tile_eq;
        const int2 before =
            block_exclusive_scan2<kCThreads>(n_lt, n_eq, S.scan, &tile_lt, &tile_eq);
        const int room = r_ties - ties_before > 0 ? r_ties - ties_before : 0;  // ties left
        const int take_cta = room < tile_eq ? room : tile_eq;
        const int taken_before = before.y < take_cta ? before.y : take_cta;
        int my_take = take_cta - before.y;
        my_take = my_take < 0 ? 0 : (my_take > n_eq ? n_eq : my_take);
        const int start = less_before + ties_done;  // this CTA's first list position
        emit_selected(lt, eq, my_take, start + before.x + taken_before, t_beg + kCPer * tid,
                      [&](int p, int tok) {
                          if (p < a.topk) idx[p] = tok;
                      });
        if (tid == 0) {
            S.sel[g][2] = start;
            S.sel[g][3] = k_eff > 0 ? tile_lt + take_cta : 0;  // entries of this CTA
        }
    }
    __syncthreads();  // the CTA's list entries (global memory) and counts are visible

    // ---- 5. gather + attention over this CTA's entries, G heads side by side ----
    if (!kBF16 && warp < kAWarps) {
        // fp32 K/V: CUDA cores, 4 rows a batch (their loads first), lane l
        // holding dims 4l .. 4l+3, scores reduced across the warp; scores in
        // log2 units (q pre-scaled by scale_log2), as in the bf16 stage
        const int wpg = kAWarps / G;
        const int g = warp / wpg, sub = warp - g * wpg;
        const int start = S.sel[g][2], cnt = S.sel[g][3];
        const int r0 = start + int(int64_t(sub) * cnt / wpg);
        const int r1 = start + int(int64_t(sub + 1) * cnt / wpg);
        const int32_t *idx = a.idx + (bh0 + g) * a.topk;
        const float4 *Kf = reinterpret_cast<const float4 *>(static_cast<const float *>(a.K) + slab * kD);
        const float4 *Vf = reinterpret_cast<const float4 *>(static_cast<const float *>(a.V) + slab * kD);
        float4 q4 = reinterpret_cast<const float4 *>(S.q[g])[lane];
        q4.x *= a.scale_log2; q4.y *= a.scale_log2; q4.z *= a.scale_log2; q4.w *= a.scale_log2;
        float m = -INFINITY, l = 0.0f, acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        for (int x0 = r0; x0 < r1; x0 += 4) {
            int32_t row[4];
            float4 kr[4], vr[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                row[u] = x0 + u < r1 ? idx[x0 + u] : -1;
                // the selection never yields an index outside [0, len)
                if (row[u] >= len) row[u] = -1;
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const float4 z = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                kr[u] = row[u] >= 0 ? Kf[int64_t(row[u]) * (kD / 4) + lane] : z;
                vr[u] = row[u] >= 0 ? Vf[int64_t(row[u]) * (kD / 4) + lane] : z;
            }
            float sc[4], mx = m;
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                float d = q4.x * kr[u].x;
                d = fmaf(q4.y, kr[u].y, d);
                d = fmaf(q4.z, kr[u].z, d);
                d = fmaf(q4.w, kr[u].w, d);
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
                sc[u] = row[u] >= 0 ? d : -INFINITY;
                mx = fmaxf(mx, sc[u]);
            }
            if (mx == -INFINITY) continue;  // warp-uniform
            const float alpha = m == -INFINITY ? 0.0f : exp2f(m - mx);
            l *= alpha;
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[i] *= alpha;
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const float pu = sc[u] == -INFINITY ? 0.0f : exp2f(sc[u] - mx);
                l += pu;
                acc[0] = fmaf(pu, vr[u].x, acc[0]);
                acc[1] = fmaf(pu, vr[u].y, acc[1]);
                acc[2] = fmaf(pu, vr[u].z, acc[2]);
                acc[3] = fmaf(pu, vr[u].w, acc[3]);
            }
            m = mx;
        }
        if (lane == 0) {
            S.part[warp][0] = m;
            S.part[warp][1] = l;
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) S.part[warp][4 + 4 * lane + i] = acc[i];
    }
    if (kBF16 && warp < kAWarps) {
        using namespace tc;
        const int wpg = kAWarps / G;  // warps per head
        const int g = warp / wpg, sub = warp - g * wpg;
        const int start = S.sel[g][2], cnt = S.sel[g][3];
        const int r0 = start + int(int64_t(sub) * cnt / wpg);
        const int r1 = start + int(int64_t(sub + 1) * cnt / wpg);
        const int n_st = (r1 - r0 + kSub - 1) / kSub;
        const int32_t *idx = a.idx + (bh0 + g) * a.topk;
        const int p = lane & 15, rh = lane >> 4;
        const uint8_t *Kp = static_cast<const uint8_t *>(a.K) + slab * kRowB + p * 16;
        const uint8_t *Vp = static_cast<const uint8_t *>(a.V) + slab * kRowB + p * 16;
        const uint32_t wring = smem_addr(S.ring) + uint32_t(warp * kCRing * kStageBytes);
        uint32_t doff[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) doff[u] = swz(8 * rh + u, p);
        auto issue = [&](int s) {
            if (s < n_st) {
                const uint32_t Ks = wring + uint32_t((s % kCRing) * kStageBytes);
                const uint32_t Vs = Ks + kSub * kRowB;
                const int x0 = r0 + s * kSub + 8 * rh;
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int32_t row = x0 + u < r1 ? idx[x0 + u] : -1;
                    // the selection never yields an index outside [0, len); the
                    // check keeps a corrupted list from steering a copy outside
                    // the cache.  Rows without a key are zero-filled.
                    const bool ok = row >= 0 && row < len;
                    const int64_t off = ok ? int64_t(row) * kRowB : 0;
                    cp_async16_zfill(Ks + doff[u], Kp + off, ok ? 16u : 0u);
                    cp_async16_zfill(Vs + doff[u], Vp + off, ok ? 16u : 0u);
                }
            }
            cp_async_commit();
        };
        for (int i = 0; i < kCRing - 1; ++i) issue(i);
        const LaneOffsets lo(lane);
        uint32_t qb[8][2];
        load_query<false>(S.q[g], a.scale_log2, lane, qb);
        float O[8][4];
#pragma unroll
        for (int j = 0; j < 8; ++j) O[j][0] = O[j][1] = O[j][2] = O[j][3] = 0.0f;
        float m_ref = -INFINITY, l_part = 0.0f;
        for (int s = 0; s < n_st; ++s) {
            cp_async_wait<kCRing - 2>();
            __syncwarp();
            issue(s + kCRing - 1);
            const int x = r0 + s * kSub + lane;
            const int32_t row = lane < kSub && x < r1 ? idx[x] : -1;
            const uint32_t vmask = __ballot_sync(0xffffffffu, row >= 0 && row < len);
            attend_stage(vmask, wring + uint32_t((s % kCRing) * kStageBytes), qb, lo, O, m_ref,
                         l_part, lane);
        }
        cp_async_wait<0>();
        for (int i = lane; i < kPartStride; i += 32) S.part[warp][i] = i == 0 ? -INFINITY : 0.0f;
        __syncwarp();
        if (n_st > 0) store_partial(S.part[warp], O, m_ref, l_part, lane);
    }
    __syncthreads();
    // the warps of each head merged into the CTA's partial, written into the
    // first CTA's shared memory
    {
        float *dst0 = cl.map_shared_rank(&S.merged[0][0][0], 0);
        const int wpg = kAWarps / G;
        for (int i = tid; i < G * kD; i += kCThreads) {
            const int g = i / kD, d = i % kD;
            float M = -INFINITY;
            for (int w = g * wpg; w < (g + 1) * wpg; ++w) M = fmaxf(M, S.part[w][0]);
            float L = 0.0f, A = 0.0f;
            if (M != -INFINITY)
                for (int w = g * wpg; w < (g + 1) * wpg; ++w) {
                    const float wt = S.part[w][0] == -INFINITY ? 0.0f : exp2f(S.part[w][0] - M);
                    L = fmaf(S.part[w][1], wt, L);
                    A = fmaf(S.part[w][4 + d], wt, A);
                }
            float *pp = dst0 + (size_t(rank) * kClusterMaxG + g) * kPartStride;
            if (d == 0) {
                pp[0] = M;
                pp[1] = L;
            }
            pp[4 + d] = A;
        }
    }

    // ---- 6. the first CTA merges the C partials of each head ----
    cl.sync();
    if (rank != 0) return;
    for (int i = tid; i < G * kD; i += kCThreads) {
        const int g = i / kD, d = i % kD;
        float M = -INFINITY;
        for (int r = 0; r < C; ++r) M = fmaxf(M, S.merged[r][g][0]);
        float L = 0.0f, A = 0.0f;
        if (M != -INFINITY)
            for (int r = 0; r < C; ++r) {
                const float wt = S.merged[r][g][0] == -INFINITY ? 0.0f : exp2f(S.merged[r][g][0] - M);
                L = fmaf(S.merged[r][g][1], wt, L);
                A = fmaf(S.merged[r][g][4 + d], wt, A);
            }
        a.out[(bh0 + g) * kD + d] = L > 0.0f ? A / L : 0.0f;
    }
}

// The cluster launch of instantiation kM over `ctas` CTAs in clusters of C.
template <int kM>
cudaLaunchConfig_t cluster_cfg(int64_t ctas, int C, cudaStream_t s, cudaLaunchAttribute *attr)
{
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(unsigned(ctas));
    cfg.blockDim = dim3(kCThreads);
    cfg.dynamicSmemBytes = sizeof(ClusterSmem<kM>);
    cfg.stream = s;
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = unsigned(C);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cfg;
}

// Clusters of C CTAs (instantiation kM) the current device holds at once;
// queried once per (device, C) and kept.
template <int kM, bool kBF16>
cudaError_t resident_clusters(int C, int *clusters)
{
    int dev = 0;
    if (cudaError_t e = cudaGetDevice(&dev)) return e;
    static std::mutex mu;
    static std::map<std::pair<int, int>, int> known;  // (device, C) -> clusters (per kernel)
    {
        std::lock_guard<std::mutex> lock(mu);
        auto it = known.find({dev, C});
        if (it != known.end()) {
            *clusters = it->second;
            return cudaSuccess;
        }
    }
    const void *fn = reinterpret_cast<const void *>(cluster_step_kernel<kM, kBF16>);
    if (cudaError_t e = ensure_smem_attr(fn, sizeof(ClusterSmem<kM>))) return e;
    cudaLaunchAttribute attr[1];
    cudaLaunchConfig_t cfg = cluster_cfg<kM>(C, C, nullptr, attr);
    int n = 0;
    if (cudaError_t e = cudaOccupancyMaxActiveClusters(&n, cluster_step_kernel<kM, kBF16>, &cfg))
        return e;
    std::lock_guard<std::mutex> lock(mu);
    known[{dev, C}] = n;
    *clusters = n;
    return cudaSuccess;
}

}  // namespace

// The cluster step's shape for these sizes: C = the CTAs of up to 16384
// tokens a head needs (C <= 8), each taking an equal range (a multiple of
// 32 tokens), when every cluster fits the device at once.  plan->kM = 0:
// the step does not serve them.
cudaError_t cluster_step_plan(int B, int H_q, int H_kv, int64_t max_seq_len, int topk, bool bf16,
                              ClusterPlan *plan)
{
    *plan = ClusterPlan{};
    const int G = H_q / H_kv;
    if ((G != 1 && G != 2 && G != 4) || topk <= 0 || max_seq_len <= 0) return cudaSuccess;
    const int64_t slabs = int64_t(B) * H_kv;
    for (int kM = 2; kM <= 2; ++kM) {  // 16384-token CTAs: 32 tokens a thread
        const int64_t C = ceil_div(max_seq_len, int64_t(8192) * kM);
        if (C > kClusterMaxC) continue;
        int clusters = 0;
        cudaError_t e = bf16 ? resident_clusters<2, true>(int(C), &clusters)
                             : resident_clusters<2, false>(int(C), &clusters);
        if (e != cudaSuccess) return e;
        if (clusters > 0 && int64_t(clusters) >= slabs) {  // one wave
            plan->kM = kM;
            plan->C = int(C);
            plan->tok_per_cta = int(ceil_div(ceil_div(max_seq_len, C), 32) * 32);
            return cudaSuccess;
        }
    }
    return cudaSuccess;
}

cudaError_t launch_cluster_step(const ClusterArgs &a, const ClusterPlan &p, cudaStream_t s)
{
    const int64_t ctas = int64_t(p.C) * a.B * a.H_kv;
    cudaLaunchAttribute attr[1];
    if (p.kM == 2) {
        auto kernel = a.kv_bf16 ? cluster_step_kernel<2, true> : cluster_step_kernel<2, false>;
        const void *fn = reinterpret_cast<const void *>(kernel);
        if (cudaError_t e = ensure_smem_attr(fn, sizeof(ClusterSmem<2>))) return e;
        cudaLaunchConfig_t cfg = cluster_cfg<2>(ctas, p.C, s, attr);
        return cudaLaunchKernelEx(&cfg, kernel, a);
    }
    return cudaErrorInvalidValue;
}

}  // namespace hata
