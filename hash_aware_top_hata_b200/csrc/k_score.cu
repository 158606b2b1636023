// k_score.cu -- Hamming scoring of every cached key code.
//
// HATA review page (arXiv 2506.02572), "What carries the argument": the query
// code is XOR-ed with every cached key code and a popcount reduction gives
// the Hamming score; major comment 1 (Algorithm 3): the top-k runs over
// these 129 possible scores.
//
// Work items are (b, h_kv, group of <= 8 query heads, chunk of 4096 tokens);
// CTA k takes items k, k + gridDim.x, ...  Inside an item every warp streams
// its own 512 tokens as four 128-token units, with no block-wide barrier:
// lane l owns tokens l, l+32, l+64, l+96 of a unit (four coalesced 16-byte
// loads per warp instruction).  The loads are asynchronous copies
// (cp.async) into a per-warp ring of kRing units in shared memory, issued
// kRing-1 units ahead; every lane reads back only the bytes it copied, so a
// lane's own wait_group is the only synchronisation, and the codes in
// flight cost no registers.  The code stream is read from HBM exactly once
// per KV head.  Each code is scored against every query head of the group:
//
//   x_w = code_w XOR q_w (w = 0..3)
//   (s, c)    = full-add(x0, x1, x2)    -- bitwise carry-save adder
//   (ones, c2) = half-add(s, x3)
//   dist = popc(ones) + 2 popc(c XOR c2) + 4 popc(c AND c2)
//
// i.e. three population counts instead of four: POPC issues at an eighth of
// the integer-logic rate on sm_100a, and it is what bounds the arithmetic.
//
// Per query head the kernel stores the u8 distance row (32 lanes write 32
// consecutive bytes per store; the row stays L2-resident for the selection
// kernel) and counts a 129-bin histogram per chunk in shared memory.  The
// block's single barrier per item closes the chunk: warp g publishes head
// g's histogram as a cumulative histogram (for the selection's offsets) and
// adds its non-zero bins into the head's total histogram.
#include "block_scan.cuh"
#include "hata_internal.cuh"
#include "tma.cuh"

namespace hata {
namespace {

constexpr int kWarps = kScoreThreads / 32;              // 8
constexpr int kUnit = 128;                              // tokens per warp step
constexpr int kUnitsPerWarp = kChunk / (kWarps * kUnit);  // 4
constexpr int kRing = 4;                                // units per warp ring
static_assert(kUnitsPerWarp * kWarps * kUnit == kChunk, "warps tile a chunk");
static_assert(kScoreHeads <= kWarps, "one publishing warp per head");

__device__ __forceinline__ int64_t clamp_len(int32_t sl, int64_t max_len, int64_t n_cap)
{
    int64_t l = sl < 0 ? 0 : sl;
    l = l < max_len ? l : max_len;
    return l < n_cap ? l : n_cap;
}

__device__ __forceinline__ int hamming128(const uint4 &k, const uint4 &q)
{
    const uint32_t x0 = k.x ^ q.x, x1 = k.y ^ q.y, x2 = k.z ^ q.z, x3 = k.w ^ q.w;
    const uint32_t s = x0 ^ x1 ^ x2;
    const uint32_t c = (x0 & x1) | (x2 & (x0 ^ x1));
    const uint32_t ones = s ^ x3, c2 = s & x3;
    return __popc(ones) + 2 * __popc(c ^ c2) + 4 * __popc(c & c2);
}

struct Item {
    int b, h, c, ng;
    int64_t len;
    size_t bh0;  // b * H_q + first query head of the group
};

struct ScoreSmem {
    uint4 ring[kWarps][kRing][kUnit];            // 64 KB of staged codes
    uint4 qs[2][kScoreHeads];                    // query codes, by item parity
    uint32_t hist[2][kScoreHeads][kHistStride];  // chunk histograms, by item parity
};

// Histogram increment: one shared-memory reduction, no return value.
__device__ __forceinline__ void red_shared_add1(uint32_t addr)
{
    asm volatile("red.shared.add.u32 [%0], 1;" ::"r"(addr) : "memory");
}

template <int GB>
__global__ void __launch_bounds__(kScoreThreads, 3) score_kernel(ScoreArgs a)
{
    extern __shared__ __align__(128) uint8_t smem_raw[];
    ScoreSmem &S = *reinterpret_cast<ScoreSmem *>(smem_raw);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    pdl_trigger();
    pdl_wait();  // query codes, the appended key code and cleared counters

    // item -> (b, h_kv, head group, chunk): 32-bit arithmetic
    auto item_of = [&](int k) {
        const int it = int(blockIdx.x) + k * int(gridDim.x);
        Item r;
        r.c = it % int(a.n_chunks);
        int g = it / int(a.n_chunks);
        const int z = g % a.zgroups;
        g /= a.zgroups;
        r.h = g % a.H_kv;
        r.b = g / a.H_kv;
        r.len = clamp_len(__ldg(a.seq_len + r.b), a.max_seq_len, a.n_cap);
        const int g0 = z * kScoreHeads;
        r.ng = min(GB, a.G - g0);
        r.bh0 = size_t(r.b) * a.H_q + size_t(r.h) * a.G + g0;
        return r;
    };
    // the query codes of item k into qs[k & 1] (threads 0 .. 4*GB-1)
    auto stage_q = [&](int k) {
        if (tid < 4 * GB) {
            const Item r = item_of(k);
            const int g = tid >> 2, w = tid & 3;
            reinterpret_cast<uint32_t *>(&S.qs[k & 1][0])[tid] =
                g < r.ng ? __ldg(a.qcodes + (r.bh0 + g) * kWords + w) : 0u;
        }
    };

    const int n_items = int(int64_t(a.B) * a.H_kv * a.zgroups * a.n_chunks);
    const int my_items =
        int(blockIdx.x) < n_items ? (n_items - 1 - int(blockIdx.x)) / int(gridDim.x) + 1 : 0;
    if (my_items == 0) return;
    for (int i = tid; i < 2 * kScoreHeads * kHistStride; i += kScoreThreads)
        (&S.hist[0][0][0])[i] = 0u;
    stage_q(0);
    if (my_items > 1) stage_q(1);
    __syncthreads();

    const uint4 *codes = reinterpret_cast<const uint4 *>(a.codes);
    const int n_units = my_items * kUnitsPerWarp;
    // copy this warp's unit j (of its item sequence) into ring slot j % kRing;
    // tokens past len are zero-filled without reading memory.  Always
    // commits one group (empty past the end) so the group count stays exact.
    Item ld = item_of(0);
    auto issue = [&](int j) {
        asm volatile("" ::: "memory");  // earlier reads of the ring stay before the copies
        if (j < n_units) {
            const int u = j % kUnitsPerWarp;
            if (u == 0 && j > 0) ld = item_of(j / kUnitsPerWarp);
            const int64_t t0 = int64_t(ld.c) * kChunk + (warp * kUnitsPerWarp + u) * kUnit + lane;
            const uint4 *src = codes + (int64_t(ld.b) * a.H_kv + ld.h) * a.n_cap + t0;
            const uint32_t dst = smem_addr(&S.ring[warp][j % kRing][lane]);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const bool ok = t0 + 32 * i < ld.len;
                cp_async16_zfill(dst + 512u * i, ok ? src + 32 * i : codes, ok ? 16u : 0u);
            }
        }
        cp_async_commit();
    };
    for (int j = 0; j < kRing - 1; ++j) issue(j);

    Item cp = item_of(0);  // item of the unit being scored
    for (int j = 0; j < n_units; ++j) {
        const int k = j / kUnitsPerWarp, u = j % kUnitsPerWarp;
        issue(j + kRing - 1);
        cp_async_wait<kRing - 1>();  // this lane's copies of unit j have landed
        uint4 cur[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) cur[i] = S.ring[warp][j % kRing][lane + 32 * i];
        if (u == 0 && j > 0) cp = item_of(k);
        const int p = k & 1;
        const int64_t t0 = int64_t(cp.c) * kChunk + (warp * kUnitsPerWarp + u) * kUnit;
        const int64_t nv64 = cp.len - t0;
        const int nv = nv64 <= 0 ? 0 : (nv64 >= kUnit ? kUnit : int(nv64));
        uint8_t *row0 = a.dist + cp.bh0 * a.dist_row + t0;
        if (nv == 0) {
            // past seq_len: pad bytes only (4 per lane, 128 per head)
#pragma unroll
            for (int g = 0; g < GB; ++g)
                if (g < cp.ng)
                    reinterpret_cast<uint32_t *>(row0 + g * a.dist_row)[lane] = 0xffffffffu;
        } else {
#pragma unroll
            for (int g = 0; g < GB; ++g) {
                if (g < cp.ng) {
                    const uint4 q = S.qs[p][g];
                    uint8_t *row = row0 + g * a.dist_row + lane;
                    const uint32_t H = smem_addr(S.hist[p][g]);
                    if (nv == kUnit) {
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const int d = hamming128(cur[i], q);
                            __stcg(row + 32 * i, uint8_t(d));
                            red_shared_add1(H + 4u * uint32_t(d));
                        }
                    } else {
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const int d = hamming128(cur[i], q);
                            const bool valid = lane + 32 * i < nv;
                            __stcg(row + 32 * i, valid ? uint8_t(d) : kDistPad);
                            if (valid) red_shared_add1(H + 4u * uint32_t(d));
                        }
                    }
                }
            }
        }
        if (u == kUnitsPerWarp - 1) {
            // ---- chunk done (all warps): publish its histogram ----
            __syncthreads();
            const int64_t nch = cp.len > 0 ? ceil_div(cp.len, kChunk) : 1;
            if (warp < cp.ng) {
                const int g = warp;
                uint32_t *H = S.hist[p][g];
                uint32_t vv[5];
                uint32_t run = 0;
#pragma unroll
                for (int e = 0; e < 5; ++e) {
                    const int t = lane * 5 + e;
                    vv[e] = t < kBins ? H[t] : 0u;
                    run += vv[e];
                }
                if (cp.c < nch) {
                    const size_t bh = cp.bh0 + g;
                    uint32_t acc = uint32_t(warp_inclusive_scan(int(run))) - run;
                    uint32_t *cum = a.cum + (bh * a.n_chunks + cp.c) * kCumStride;
#pragma unroll
                    for (int e = 0; e < 5; ++e) {
                        const int t = lane * 5 + e;
                        acc += vv[e];
                        if (t < kBins) {
                            cum[t] = acc;
                            if (vv[e]) atomicAdd(a.hist_total + bh * kHistStride + t, vv[e]);
                        }
                    }
                }
#pragma unroll
                for (int e = 0; e < 5; ++e)
                    if (lane * 5 + e < kBins) H[lane * 5 + e] = 0u;
            }
            // qs[p] is free (item k is scored): stage item k + 2's query codes
            if (k + 2 < my_items) stage_q(k + 2);
        }
    }
    cp_async_wait<0>();
}

template <int GB>
cudaError_t launch_score_t(const ScoreArgs &a, cudaStream_t s)
{
    const void *fn = reinterpret_cast<const void *>(score_kernel<GB>);
    if (cudaError_t e = ensure_smem_attr(fn, sizeof(ScoreSmem))) return e;
    int dev = 0, sms = 0, per_sm = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess)
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, score_kernel<GB>,
                                                          kScoreThreads, sizeof(ScoreSmem));
    if (e != cudaSuccess) return e;
    const int64_t cap = int64_t(per_sm > 0 ? per_sm : 1) * sms;
    const int64_t items = int64_t(a.B) * a.H_kv * a.zgroups * a.n_chunks;
    return launch_pdl(score_kernel<GB>, dim3(unsigned(items < cap ? items : cap)),
                      dim3(kScoreThreads), sizeof(ScoreSmem), s, a);
}

}  // namespace

cudaError_t launch_score(const ScoreArgs &a, cudaStream_t s)
{
    const int gb = a.G < kScoreHeads ? a.G : kScoreHeads;
    switch (gb) {
    case 1: return launch_score_t<1>(a, s);
    case 2: return launch_score_t<2>(a, s);
    case 3: return launch_score_t<3>(a, s);
    case 4: return launch_score_t<4>(a, s);
    case 5: return launch_score_t<5>(a, s);
    case 6: return launch_score_t<6>(a, s);
    case 7: return launch_score_t<7>(a, s);
    default: return launch_score_t<8>(a, s);
    }
}

}  // namespace hata
