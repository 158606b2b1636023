// k_attend.cu -- gather of the selected K/V rows + exact softmax attention.
//
// HATA review page (arXiv 2506.02572), "What carries the argument": the
// top-k indices select K/V for attention, which the page runs as a fused
// gather + FlashAttention over the selected keys.
//
// The selected rows of all heads form one flat space of B*H_q*topk rows
// (head bh owns [bh*topk, bh*topk + k_eff)).  Three kernels walk it:
//   * attend_tc_kernel (bf16 K/V): every warp is a stream-K worker over an
//     equal, contiguous slice of the flat space, gathering 16 rows per stage
//     through a private 3-stage ring of 16-byte cp.async copies and running
//     each stage on the tensor cores (mma.sync, keys along M, q and the
//     softmax weights as hi/lo bf16 pairs); when a warp leaves a head it
//     writes one partial (m, l, acc[128]) into the head's slot for it;
//   * attend_head_kernel (bf16, heads filling about one wave of CTAs): one
//     CTA per head, warp w takes the w-th eighth of the head's list, and the
//     eight partials merge in shared memory (no combine launch);
//   * attend_simt_kernel (fp32 K/V): CTA-level stream-K on the CUDA cores,
//     16 lanes per row, a 4-deep ring of up to 32 rows.
// combine_kernel, chained behind the stream-K kernels by programmatic
// dependent launch, merges each head's partials into out = acc / l, so no
// worker waits for another.  The random 256-byte row gathers of K and V
// peak at ~5.0 TB/s on B200 (one bulk-copy request per row reaches about
// half of that), which bounds all three.
#include <cuda_bf16.h>

#include <algorithm>

#include "hata_internal.cuh"
#include "async_copy.cuh"
#include "attend_common.cuh"

namespace hata {
namespace {

constexpr int kWarps = kAttnThreads / 32;
constexpr int kHalves = kWarps * 2;
constexpr int kStageRows = 32;
constexpr int kRing = 4;
constexpr int kRowsPerHalf = kStageRows / kHalves;  // 4

template <bool BF16>
struct Rows {
    static constexpr int kRowBytes = kD * (BF16 ? 2 : 4);
    static constexpr int kPieces = kRowBytes / 16;                 // 16-byte pieces per row
    static constexpr int kSlotBytes = 2 * kStageRows * kRowBytes;  // K and V
};

// 8 consecutive row elements (from shared memory) as fp32.
template <bool BF16>
__device__ __forceinline__ void frag8(const uint8_t *row, int l16, float (&f)[8])
{
    if (BF16) {
        const uint4 v = reinterpret_cast<const uint4 *>(row)[l16];
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            f[2 * i] = __uint_as_float(w[i] << 16);
            f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    } else {
        const float4 x = reinterpret_cast<const float4 *>(row)[2 * l16];
        const float4 y = reinterpret_cast<const float4 *>(row)[2 * l16 + 1];
        f[0] = x.x; f[1] = x.y; f[2] = x.z; f[3] = x.w;
        f[4] = y.x; f[5] = y.y; f[6] = y.z; f[7] = y.w;
    }
}

// Flat row x -> index of the CTA whose range [k*T/P, (k+1)*T/P) holds it.
__device__ __forceinline__ int64_t owner(int64_t x, int64_t T, int64_t P)
{
    return ((x + 1) * P + T - 1) / T - 1;
}

struct Stage {
    int bh;        // head (b * H_q + h_q)
    int b, h;      // batch row and KV head of that head
    int p0;        // first position in the head's index list
    int n;         // rows of this stage (0: the placeholder row of an empty head)
    bool last;     // last stage of this CTA in this head
};

// Walks one CTA's range in stages with incremental 32-bit cursors (no
// division in the loop).  A head with k_eff == 0 still gets one placeholder
// stage (n = 0) from the CTA that owns its first row, so that someone
// writes its (zero) output.
template <int kRows>
struct Walker {
    const AttendArgs *a;
    int64_t remaining;   // rows of the CTA range not yet walked
    int bh, b, hq, pos;  // cursor: head, its batch row / query head, position
    int keff;            // min(topk, len(b))
    int64_t len;

    __device__ __forceinline__ void load_len()
    {
        len = clamp_len(__ldg(a->seq_len + b), a->max_seq_len, a->n_cap);
        keff = int(int64_t(a->topk) < len ? int64_t(a->topk) : len);
    }
    __device__ __forceinline__ void init(const AttendArgs *args, int64_t beg, int64_t end)
    {
        a = args;
        remaining = end - beg;
        const int64_t h = beg / a->topk;  // once per CTA
        bh = int(h);
        pos = int(beg - h * a->topk);
        b = bh / a->H_q;
        hq = bh - b * a->H_q;
        load_len();
    }
    __device__ __forceinline__ bool next(Stage &st)
    {
        while (remaining > 0) {
            const int e = keff > 0 ? keff : 1;
            if (pos >= e) {  // the rest of this head is empty: skip to the next head
                remaining -= a->topk - pos;
                pos = 0;
                ++bh;
                if (++hq == a->H_q) {
                    hq = 0;
                    ++b;
                    if (remaining > 0) load_len();
                }
                continue;
            }
            const int seg = int(int64_t(e - pos) < remaining ? int64_t(e - pos) : remaining);
            const int n = seg < kRows ? seg : kRows;
            st.bh = bh;
            st.b = b;
            st.h = hq / a->G;
            st.p0 = pos;
            st.n = keff > 0 ? n : 0;
            st.last = n == seg;
            pos += n;
            remaining -= n;
            return true;
        }
        return false;
    }
};

// fp32 K/V: CUDA-core path (16 lanes per row, shuffle-reduced dot products).
template <bool BF16>
__global__ void __launch_bounds__(kAttnThreads) attend_simt_kernel(AttendArgs a)
{
    using RW = Rows<BF16>;
    constexpr int RB = RW::kRowBytes;
    extern __shared__ __align__(128) uint8_t smem[];  // [kRing][K rows | V rows]
    __shared__ int32_t rows_s[kRing][kStageRows];
    pdl_trigger();
    pdl_wait();  // the selected index lists
    __shared__ float red_m[kHalves], red_l[kHalves];
    __shared__ __align__(16) float red_acc[kHalves][kD];

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int half = lane >> 4, l16 = lane & 15, hw = warp * 2 + half;
    const int64_t T = int64_t(a.B) * a.H_q * a.topk, P = gridDim.x;
    const int64_t beg = blockIdx.x * T / P, end = (blockIdx.x + 1) * T / P;
    const uint8_t *Kg = static_cast<const uint8_t *>(a.K);
    const uint8_t *Vg = static_cast<const uint8_t *>(a.V);

    Walker<kStageRows> prod, cons;
    prod.init(&a, beg, end);
    cons.init(&a, beg, end);

    // ---- producer: gather the rows of stage `st` into ring slot `slot` ----
    // Each thread copies the same piece column p of rows i0, i0 + kRowStep, ...
    constexpr int kRowStep = kAttnThreads / RW::kPieces;          // 8 (bf16) / 4 (fp32)
    constexpr int kRowsPerThread = kStageRows / kRowStep;          // 4 / 8
    auto issue = [&](const Stage &st, int slot) {
        uint8_t *Ks = smem + size_t(slot) * RW::kSlotBytes;
        uint8_t *Vs = Ks + kStageRows * RB;
        const int64_t len = prod.len;  // the producer's cursor sits in this stage's head
        const int64_t slab = (int64_t(st.b) * a.H_kv + st.h) * a.n_cap;
        const int32_t *idx = a.idx + int64_t(st.bh) * a.topk + st.p0;
        const int p = tid % RW::kPieces, i0 = tid / RW::kPieces;
        int32_t rows[kRowsPerThread];
#pragma unroll
        for (int u = 0; u < kRowsPerThread; ++u) {  // all index loads first
            const int i = i0 + u * kRowStep;
            rows[u] = i < st.n ? __ldg(idx + i) : -1;
        }
#pragma unroll
        for (int u = 0; u < kRowsPerThread; ++u) {
            const int i = i0 + u * kRowStep;
            // the selection never yields an index outside [0, len); the check
            // keeps a corrupted list from steering a copy outside the cache
            const bool ok = rows[u] >= 0 && rows[u] < len;
            if (ok) {
                const int64_t off = (slab + rows[u]) * RB + p * 16;
                cp_async16(Ks + i * RB + p * 16, Kg + off);
                cp_async16(Vs + i * RB + p * 16, Vg + off);
            }
            if (p == 0) rows_s[slot][i] = ok ? rows[u] : -1;
        }
    };

    Stage ps;
    int n_issued = 0;
    for (; n_issued < kRing - 1; ++n_issued) {
        if (prod.next(ps)) issue(ps, n_issued);
        cp_async_commit();
    }

    // q of the current head, scaled; online-softmax state
    float qv[8], m = -INFINITY, l = 0.0f, acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) qv[e] = acc[e] = 0.0f;
    int64_t cur_bh = -1;
    Stage cs;
    for (int s = 0; cons.next(cs); ++s) {
        // stage s has landed (the kRing-2 younger groups may still be in flight)
        cp_async_wait<kRing - 2>();
        __syncthreads();
        if (prod.next(ps)) issue(ps, n_issued % kRing);
        ++n_issued;
        cp_async_commit();  // (possibly empty) group, keeps the accounting uniform

        if (cs.bh != cur_bh) {
            cur_bh = cs.bh;
            const float4 *qp =
                reinterpret_cast<const float4 *>(a.q + int64_t(cs.bh) * kD + l16 * 8);
            const float4 x = __ldg(qp), y = __ldg(qp + 1);
            qv[0] = x.x; qv[1] = x.y; qv[2] = x.z; qv[3] = x.w;
            qv[4] = y.x; qv[5] = y.y; qv[6] = y.z; qv[7] = y.w;
#pragma unroll
            for (int e = 0; e < 8; ++e) qv[e] *= a.scale_log2;
            m = -INFINITY;
            l = 0.0f;
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[e] = 0.0f;
        }

        const int slot = s % kRing;
        const uint8_t *Ks = smem + size_t(slot) * RW::kSlotBytes;
        const uint8_t *Vs = Ks + kStageRows * RB;
        float sc[kRowsPerHalf];
        float mx = m;
#pragma unroll
        for (int u = 0; u < kRowsPerHalf; ++u) {
            const int i = hw + u * kHalves;  // warp-uniform trip count: shuffles see all lanes
            const bool valid = i < cs.n && rows_s[slot][i] >= 0;
            float p = 0.0f;
            if (valid) {
                float kx[8];
                frag8<BF16>(Ks + i * RB, l16, kx);
#pragma unroll
                for (int e = 0; e < 8; ++e) p = fmaf(qv[e], kx[e], p);
            }
#pragma unroll
            for (int o = 8; o > 0; o >>= 1) p += __shfl_xor_sync(0xffffffffu, p, o);
            sc[u] = valid ? p : -INFINITY;
            mx = fmaxf(mx, sc[u]);
        }
        const float mref = mx == -INFINITY ? 0.0f : mx;
        const float alpha = exp2f(m - mref);
        l *= alpha;
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] *= alpha;
#pragma unroll
        for (int u = 0; u < kRowsPerHalf; ++u) {
            if (sc[u] != -INFINITY) {
                const float p = exp2f(sc[u] - mref);
                l += p;
                float vx[8];
                frag8<BF16>(Vs + (hw + u * kHalves) * RB, l16, vx);
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[e] = fmaf(p, vx[e], acc[e]);
            }
        }
        m = mx;

        if (!cs.last) continue;
        // ---- this CTA is done with head cs.bh: publish a partial ----
        if (l16 == 0) {
            red_m[hw] = m;
            red_l[hw] = l;
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) red_acc[hw][l16 * 8 + e] = acc[e];
        __syncthreads();
        const int slot_out = int(blockIdx.x - owner(int64_t(cs.bh) * a.topk, T, P));
        {
            float M = -INFINITY;
#pragma unroll
            for (int i = 0; i < kHalves; ++i) M = fmaxf(M, red_m[i]);
            const float Mref = M == -INFINITY ? 0.0f : M;
            float L = 0.0f, A = 0.0f;
#pragma unroll
            for (int i = 0; i < kHalves; ++i) {
                const float w = exp2f(red_m[i] - Mref);
                L = fmaf(red_l[i], w, L);
                A = fmaf(red_acc[i][tid], w, A);
            }
            float *pp = a.part + (int64_t(cs.bh) * a.n_split + slot_out) * kPartStride;
            if (tid == 0) {
                pp[0] = M;
                pp[1] = L;
            }
            pp[4 + tid] = A;
        }
        __syncthreads();  // red_* are rewritten by the next head
    }
    cp_async_wait<0>();
}

// ------------------------------------------------------------------------
// bf16 K/V: tensor-core path.
//
// Every warp is an independent stream-K worker: the flat row space is cut
// into n_workers contiguous ranges (eight warps per CTA, one CTA per SM), so
// a warp walks only its own rows and needs no block barrier.  Random
// 256-byte row gathers on B200 see a loaded DRAM latency of several
// microseconds; the copies are issued by many warps (one warp alone cannot
// issue cp.async fast enough), each keeping a private ring of three 16-key
// stages (K and V, 8 KB a stage) in flight two stages ahead of its
// arithmetic, with 16-byte cp.async copies.  The CTA's slice of the flat
// index list is loaded into shared memory up front, so no copy waits on an
// index load.
//
// Each stage runs on the tensor cores (attend_common.cuh).  When a warp
// leaves a head it writes a partial (m, l, acc[128]) for the combine kernel.
//
// A warp is done with head cs.bh: write its partial into the head's slot
// for this worker; the combine kernel merges the slots.
__device__ __forceinline__ void publish(const AttendArgs &a, const Stage &cs, int64_t wid,
                                        int64_t NW, int64_t T, const float (&O)[8][4],
                                        float m_ref, float l_part, int lane)
{
    const int64_t k_first = owner(int64_t(cs.bh) * a.topk, T, NW);
    tc::store_partial(a.part + (int64_t(cs.bh) * a.n_split + (wid - k_first)) * kPartStride, O,
                  m_ref, l_part, lane);
}


__global__ void __launch_bounds__(tc::kThreads, 1) attend_tc_kernel(AttendArgs a)
{
    using namespace tc;
    extern __shared__ __align__(128) uint8_t smem[];  // [warp][kRingW][K | V], then indices
    __shared__ int32_t rows_s[kTcWarps][kRingW][kSub];
    pdl_trigger();

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t T = int64_t(a.B) * a.H_q * a.topk;
    const int64_t NW = a.n_workers;  // warps that own rows (<= T, so none is empty)
    const int64_t wid = int64_t(blockIdx.x) * kTcWarps + warp;
    const int64_t cta_beg = int64_t(blockIdx.x) * kTcWarps * T / NW;
    int64_t cta_end = (int64_t(blockIdx.x) + 1) * kTcWarps;
    cta_end = (cta_end < NW ? cta_end : NW) * T / NW;
    const uint8_t *Kg = static_cast<const uint8_t *>(a.K);
    const uint8_t *Vg = static_cast<const uint8_t *>(a.V);
    const uint32_t wring = smem_addr(smem) + uint32_t(warp * kRingW * kStageBytes);
    int32_t *idx_s = reinterpret_cast<int32_t *>(smem + kRingBytes);
    const int64_t beg = wid * T / NW, end = (wid + 1) * T / NW;

    // The walkers read only seq_len, a step input: set them up while the
    // selection kernel is still running.
    Walker<kSub> prod, cons;
    if (wid < NW) {
        prod.init(&a, beg, end);
        cons.init(&a, beg, end);
    }
    pdl_wait();  // the selected index lists

    // the CTA's slice of the index list (the first kIdxCap of it): all loads
    // of a thread first, then the shared-memory stores
    if (cta_beg < cta_end) {
        const int64_t n_s = cta_end - cta_beg < kIdxCap ? cta_end - cta_beg : kIdxCap;
        constexpr int kPer = kIdxCap / kThreads;
        static_assert(kIdxCap % kThreads == 0, "whole rounds of the slice load");
        int32_t v[kPer];
#pragma unroll
        for (int u = 0; u < kPer; ++u) {
            const int64_t i = tid + int64_t(u) * kThreads;
            v[u] = i < n_s ? __ldg(a.idx + cta_beg + i) : 0;
        }
#pragma unroll
        for (int u = 0; u < kPer; ++u) {
            const int64_t i = tid + int64_t(u) * kThreads;
            if (i < n_s) idx_s[i] = v[u];
        }
    }
    __syncthreads();
    if (wid >= NW) return;
    auto index_of = [&](int64_t x) {  // flat row -> key index
        return x - cta_beg < kIdxCap ? idx_s[x - cta_beg] : __ldg(a.idx + x);
    };

    int64_t prod_x = beg;  // flat row of the producer walker's position
    int n_issued = 0;
    const int p = lane & 15, rb = lane >> 4;  // lane = piece p of rows rb, rb+2, ...
    uint32_t doff[kSub / 2];                   // this lane's swizzled destinations
#pragma unroll
    for (int u = 0; u < kSub / 2; ++u) doff[u] = swz(rb + 2 * u, p);

    // gather this warp's next stage into its ring (always commits one group)
    auto issue_next = [&]() {
        Stage st;
        const int64_t before = prod.remaining;
        if (prod.next(st)) {
            const int64_t used = before - prod.remaining;  // skipped + this stage's rows
            const int64_t x0 = prod_x + used - st.n;
            prod_x += used;
            const int slot = n_issued++ % kRingW;
            const uint32_t Ks = wring + uint32_t(slot * kStageBytes), Vs = Ks + kSub * kRowB;
            const int64_t slab = (int64_t(st.b) * a.H_kv + st.h) * a.n_cap;
#pragma unroll
            for (int u = 0; u < kSub / 2; ++u) {
                const int r = rb + 2 * u;
                const int32_t row = r < st.n ? index_of(x0 + r) : -1;
                // the selection never yields an index outside [0, len); the
                // check keeps a corrupted list from steering a copy outside
                // the cache.  Rows without a key are zero-filled.
                const bool ok = row >= 0 && row < prod.len;
                const int64_t off = ok ? (slab + row) * kRowB + p * 16 : 0;
                cp_async16_zfill(Ks + doff[u], Kg + off, ok ? 16u : 0u);
                cp_async16_zfill(Vs + doff[u], Vg + off, ok ? 16u : 0u);
                if (p == 0) rows_s[warp][slot][r] = ok ? row : -1;
            }
        }
        cp_async_commit();
    };
    for (int i = 0; i < kRingW - 1; ++i) issue_next();

    const LaneOffsets lo(lane);
    uint32_t qb[8][2];  // B operand of S^T: columns q_hi (lanes 0-3), q_lo (lanes 4-7)
    float O[8][4];
    float m_ref = -INFINITY, l_part = 0.0f;
    int cur_bh = -1;
    Stage cs;
    for (int s = 0; cons.next(cs); ++s) {
        if (cs.bh != cur_bh) {  // a new head: its query as hi/lo bf16 rows, fresh state
            cur_bh = cs.bh;
            load_query(a.q + int64_t(cs.bh) * kD, a.scale_log2, lane, qb);
#pragma unroll
            for (int j = 0; j < 8; ++j) O[j][0] = O[j][1] = O[j][2] = O[j][3] = 0.0f;
            m_ref = -INFINITY;
            l_part = 0.0f;
        }

        cp_async_wait<kRingW - 2>();
        __syncwarp();
        const int slot = s % kRingW;
        issue_next();
        const int32_t *rows = rows_s[warp][slot];
        const uint32_t vmask = __ballot_sync(
            0xffffffffu, lane < kSub && lane < cs.n && rows[lane < kSub ? lane : 0] >= 0);
        attend_stage(vmask, wring + uint32_t(slot * kStageBytes), qb, lo, O, m_ref, l_part, lane);

        if (cs.last) publish(a, cs, wid, NW, T, O, m_ref, l_part, lane);
    }
    cp_async_wait<0>();
}

// Head-per-CTA form, for heads that fill about one wave of CTAs: CTA bh
// attends the whole selected list of head bh.  Warp w takes the w-th eighth
// of the list (plain index arithmetic, no walker), the gather addresses are
// one multiply-add from the slab's base, and the warps' partials are merged
// in shared memory, so no combine launch follows.  Needs topk <= kIdxCap.
//
// The sequence-parallel step runs the same kernel with head_split CTAs per
// head (CTA c takes the c-th of head_split equal parts of the head's list,
// whose length k_head the kernel before wrote) and unnormalised partials
// out: into part_out directly (head_split = 1), or one per CTA into the
// head's partial slots for combine_kernel.
__global__ void __launch_bounds__(tc::kThreads, 1) attend_head_kernel(AttendArgs a)
{
    using namespace tc;
    extern __shared__ __align__(128) uint8_t smem[];  // [warp][kRingW][K | V], then indices
    __shared__ __align__(16) float part_s[kTcWarps][kPartStride];
    pdl_trigger();

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int split = a.head_split > 0 ? a.head_split : 1;
    const int bh = int(blockIdx.x) / split, cs = int(blockIdx.x) - bh * split;
    const int b = bh / a.H_q, h = (bh - b * a.H_q) / a.G;
    // seq_len is a step input: everything up to the wait overlaps the selection
    const int64_t len = clamp_len(__ldg(a.seq_len + b), a.max_seq_len, a.n_cap);
    int keff = int(int64_t(a.topk) < len ? int64_t(a.topk) : len);

    const int p = lane & 15, rh = lane >> 4;  // 16-byte piece p of rows 8 rh .. 8 rh + 7
    const int64_t slab = (int64_t(b) * a.H_kv + h) * a.n_cap;
    const uint8_t *Kp = static_cast<const uint8_t *>(a.K) + slab * kRowB + p * 16;
    const uint8_t *Vp = static_cast<const uint8_t *>(a.V) + slab * kRowB + p * 16;
    const uint32_t wring = smem_addr(smem) + uint32_t(warp * kRingW * kStageBytes);
    int32_t *idx_s = reinterpret_cast<int32_t *>(smem + kRingBytes);
    uint32_t doff[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) doff[u] = swz(8 * rh + u, p);
    // a warp with no row of the head leaves an empty partial
    for (int i = lane; i < kPartStride; i += 32) part_s[warp][i] = i == 0 ? -INFINITY : 0.0f;
    __syncwarp();
    pdl_wait();  // the selected index lists (and k_head)
    if (a.k_head) {
        const int kh = __ldg(a.k_head + bh);
        keff = kh < keff ? (kh > 0 ? kh : 0) : keff;
    }
    // this CTA's entries [c0, c1) of the head's list; warp w its w-th eighth
    const int c0 = int(int64_t(cs) * keff / split), c1 = int(int64_t(cs + 1) * keff / split);
    const int r0 = c0 + int(int64_t(warp) * (c1 - c0) / kTcWarps);
    const int r1 = c0 + int(int64_t(warp + 1) * (c1 - c0) / kTcWarps);
    const int n_st = (r1 - r0 + kSub - 1) / kSub;

    {  // the CTA's part of the list: all loads first, then the stores
        const int32_t *src = a.idx + int64_t(bh) * a.topk + c0;
        constexpr int kPer = kIdxCap / kThreads;
        int32_t v[kPer];
#pragma unroll
        for (int u = 0; u < kPer; ++u) {
            const int i = tid + u * kThreads;
            v[u] = i < c1 - c0 ? __ldg(src + i) : -1;
        }
#pragma unroll
        for (int u = 0; u < kPer; ++u) {
            const int i = tid + u * kThreads;
            if (i < c1 - c0) idx_s[i] = v[u];
        }
    }
    __syncthreads();

    // stage s of this warp (entries r0 + 16 s ...) into ring slot s % kRingW;
    // always commits one group
    auto issue = [&](int s) {
        if (s < n_st) {
            const uint32_t Ks = wring + uint32_t((s % kRingW) * kStageBytes);
            const uint32_t Vs = Ks + kSub * kRowB;
            const int x0 = r0 + s * kSub + 8 * rh;
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int32_t row = x0 + u < r1 ? idx_s[x0 + u - c0] : -1;
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
    for (int i = 0; i < kRingW - 1; ++i) issue(i);

    const LaneOffsets lo(lane);
    uint32_t qb[8][2];
    load_query(a.q + int64_t(bh) * kD, a.scale_log2, lane, qb);
    float O[8][4];
#pragma unroll
    for (int j = 0; j < 8; ++j) O[j][0] = O[j][1] = O[j][2] = O[j][3] = 0.0f;
    float m_ref = -INFINITY, l_part = 0.0f;

    for (int s = 0; s < n_st; ++s) {
        cp_async_wait<kRingW - 2>();
        __syncwarp();
        issue(s + kRingW - 1);
        const int x = r0 + s * kSub + lane;
        const int32_t row = lane < kSub && x < r1 ? idx_s[x - c0] : -1;
        const uint32_t vmask = __ballot_sync(0xffffffffu, row >= 0 && row < len);
        attend_stage(vmask, wring + uint32_t((s % kRingW) * kStageBytes), qb, lo, O, m_ref,
                     l_part, lane);
    }
    cp_async_wait<0>();
    if (n_st > 0) store_partial(part_s[warp], O, m_ref, l_part, lane);

    // merge the warps' partials of the head
    __syncthreads();
    if (tid < kD) {
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kTcWarps; ++w) M = fmaxf(M, part_s[w][0]);
        float L = 0.0f, A = 0.0f;
        if (M != -INFINITY) {
#pragma unroll
            for (int w = 0; w < kTcWarps; ++w) {
                const float wt = part_s[w][0] == -INFINITY ? 0.0f : exp2f(part_s[w][0] - M);
                L = fmaf(part_s[w][1], wt, L);
                A = fmaf(part_s[w][4 + tid], wt, A);
            }
        }
        if (a.part_out || split > 1) {  // an unnormalised partial (m, l, acc)
            float *pp = split > 1 ? a.part + (int64_t(bh) * a.n_split + cs) * kPartStride
                                  : a.part_out + int64_t(bh) * kPartStride;
            if (tid == 0) {
                pp[0] = M;
                pp[1] = L;
            }
            pp[4 + tid] = A;
        } else {
            a.out[int64_t(bh) * kD + tid] = L > 0.0f ? A / L : 0.0f;
        }
    }
}

// ------------------------------------------------------------------------
// Combine: kWph warps per head merge the partials of the head's
// contributors (workers k_first..k_last of the stream-K split, or the CTAs
// of a split head) into out = acc / l.  It runs as its own launch behind the
// attention kernel (programmatic dependent launch: its CTAs are resident
// early and wait for the attention grid to finish), so no attention worker
// waits for another or merges at the end of its range.  The contributor
// count depends only on seq_len (a step input), so it is known before the
// wait; after it, all loads of a round of kCombineRound partials (lane c: m
// and l of contributor c; every lane: its 4 output dims of each partial)
// are issued together, one dependent memory round trip per round.  Warp w
// of a head takes rounds w, w + kWph, ...; with kWph = 4 the head's first 64
// partials cost one round trip, and the warps' merged partials are merged
// once more in shared memory.
constexpr int kCombineWarps = 4;
constexpr int kCombineRound = 16;

template <int kWph>
__global__ void __launch_bounds__(32 * kCombineWarps) combine_kernel(AttendArgs a)
{
    static_assert(kCombineWarps % kWph == 0, "whole heads per CTA");
    __shared__ float part_s[kWph > 1 ? kCombineWarps : 1][kPartStride];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, sub = warp % kWph;
    const int64_t bh = int64_t(blockIdx.x) * (kCombineWarps / kWph) + warp / kWph;
    const bool live = bh < int64_t(a.B) * a.H_q;  // uniform over the head's warps
    int n_contrib = 0;
    if (live && a.head_split > 0) {
        n_contrib = a.head_split;  // one partial per CTA of the head
    } else if (live) {
        const int64_t T = int64_t(a.B) * a.H_q * a.topk, NW = a.n_workers;
        const int b = int(bh / a.H_q);
        const int64_t len = clamp_len(__ldg(a.seq_len + b), a.max_seq_len, a.n_cap);
        const int64_t keff = int64_t(a.topk) < len ? int64_t(a.topk) : len;
        const int64_t h0 = bh * a.topk;
        n_contrib = int(owner(h0 + (keff > 0 ? keff : 1) - 1, T, NW) - owner(h0, T, NW) + 1);
    }
    pdl_wait();  // every partial is written
    const float *pc = a.part + (live ? bh : 0) * a.n_split * kPartStride;
    float M = -INFINITY, L = 0.0f, A[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    for (int c0 = kCombineRound * sub; c0 < n_contrib; c0 += kCombineRound * kWph) {
        const int c = c0 + lane;
        const bool mine = lane < kCombineRound && c < n_contrib;
        const float mc = mine ? __ldcg(pc + c * kPartStride) : -INFINITY;
        const float lc = mine ? __ldcg(pc + c * kPartStride + 1) : 0.0f;
        float acc[kCombineRound][4];
#pragma unroll
        for (int j = 0; j < kCombineRound; ++j) {
            const float *q = pc + (c0 + j) * kPartStride + 4 + lane;
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[j][i] = c0 + j < n_contrib ? __ldcg(q + 32 * i) : 0.0f;
        }
        float mr = mc;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mr = fmaxf(mr, __shfl_xor_sync(0xffffffffu, mr, o));
        const float Mn = fmaxf(M, mr);
        if (Mn == -INFINITY) continue;  // warp-uniform: no weight yet
        if (M != Mn) {
            const float r = M == -INFINITY ? 0.0f : exp2f(M - Mn);
            L *= r;
#pragma unroll
            for (int i = 0; i < 4; ++i) A[i] *= r;
            M = Mn;
        }
        const float wc = mc == -INFINITY ? 0.0f : exp2f(mc - M);
        float lw = lc * wc;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) lw += __shfl_xor_sync(0xffffffffu, lw, o);
        L += lw;
#pragma unroll
        for (int j = 0; j < kCombineRound; ++j) {
            const float w = __shfl_sync(0xffffffffu, wc, j);
#pragma unroll
            for (int i = 0; i < 4; ++i) A[i] = fmaf(acc[j][i], w, A[i]);
        }
    }
    if constexpr (kWph > 1) {  // the head's warps: one more merge, in shared memory
        const int wp = kWph > 1 ? warp : 0;
        if (lane == 0) {
            part_s[wp][0] = M;
            part_s[wp][1] = L;
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) part_s[wp][4 + lane + 32 * i] = A[i];
        __syncthreads();
        if (sub != 0) return;
        const int w0 = wp;  // the head's first warp
        float Mh = -INFINITY;
#pragma unroll
        for (int w = 0; w < kWph; ++w) Mh = fmaxf(Mh, part_s[w0 + w][0]);
        L = 0.0f;
#pragma unroll
        for (int i = 0; i < 4; ++i) A[i] = 0.0f;
        if (Mh != -INFINITY) {
#pragma unroll
            for (int w = 0; w < kWph; ++w) {
                const float mw = part_s[w0 + w][0];
                const float wt = mw == -INFINITY ? 0.0f : exp2f(mw - Mh);
                L = fmaf(part_s[w0 + w][1], wt, L);
#pragma unroll
                for (int i = 0; i < 4; ++i) A[i] = fmaf(part_s[w0 + w][4 + lane + 32 * i], wt, A[i]);
            }
        }
        M = Mh;
    }
    if (!live) return;
    if (a.part_out) {  // the sequence-parallel step: this shard's unnormalised partial
        float *pp = a.part_out + bh * kPartStride;
        if (lane == 0) {
            pp[0] = M;
            pp[1] = L;
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) pp[4 + lane + 32 * i] = A[i];
        return;
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) a.out[bh * kD + lane + 32 * i] = L > 0.0f ? A[i] / L : 0.0f;
}

template <typename Kernel>
cudaError_t occupancy_grid(Kernel kernel, int threads, size_t smem, int64_t *grid)
{
    if (cudaError_t e = ensure_smem_attr(reinterpret_cast<const void *>(kernel), smem)) return e;
    int dev = 0, sms = 0, per_sm = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess)
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, threads, smem);
    *grid = int64_t(per_sm > 0 ? per_sm : 1) * sms;
    return e;
}

// Heads that nearly fill one wave of P CTAs: a CTA per head, merged in
// shared memory, saves the combine launch and its completion gap.
bool head_per_cta(int B, int H_q, int topk, int64_t P)
{
    const int64_t heads = int64_t(B) * H_q;
    return heads * 5 >= P * 4 && heads <= P && topk >= 16 * tc::kTcWarps &&
           topk <= tc::kIdxCap;
}

}  // namespace

cudaError_t attend_launch_count(int B, int H_q, int topk, bool bf16, int *n)
{
    int64_t P = 0;
    *n = 2;
    if (!bf16) return cudaSuccess;
    if (cudaError_t e = occupancy_grid(attend_tc_kernel, tc::kThreads, tc::kSmem, &P)) return e;
    if (head_per_cta(B, H_q, topk, P)) *n = 1;
    return cudaSuccess;
}

cudaError_t launch_attend(AttendArgs &a, bool bf16, cudaStream_t s)
{
    const int64_t T = int64_t(a.B) * a.H_q * a.topk;
    int64_t P = 0;
    if (bf16) {
        if (cudaError_t e = occupancy_grid(attend_tc_kernel, tc::kThreads, tc::kSmem, &P)) return e;
        int64_t NW = P * tc::kTcWarps;
        if (NW > kAttnMaxWorkers) NW = kAttnMaxWorkers;
        if (NW > T) NW = T;
        a.head_per_cta = head_per_cta(a.B, a.H_q, a.topk, P);
        a.head_split = 0;
        if (a.head_per_cta) {
            a.n_workers = 0;
            if (cudaError_t e = ensure_smem_attr(reinterpret_cast<const void *>(attend_head_kernel),
                                                 tc::kSmem))
                return e;
            return launch_pdl(attend_head_kernel, dim3(unsigned(int64_t(a.B) * a.H_q)),
                              dim3(tc::kThreads), tc::kSmem, s, a);
        }
        a.n_workers = NW;
        return launch_pdl(attend_tc_kernel, dim3(unsigned(ceil_div(NW, tc::kTcWarps))),
                          dim3(tc::kThreads), tc::kSmem, s, a);
    }
    constexpr size_t kSmemF32 = size_t(kRing) * Rows<false>::kSlotBytes;
    if (cudaError_t e = occupancy_grid(attend_simt_kernel<false>, kAttnThreads, kSmemF32, &P))
        return e;
    if (P > kAttnMaxWorkers) P = kAttnMaxWorkers;
    if (P > T) P = T;
    a.n_workers = P;
    a.head_per_cta = 0;
    a.head_split = 0;
    return launch_pdl(attend_simt_kernel<false>, dim3(unsigned(P)), dim3(kAttnThreads), kSmemF32,
                      s, a);
}

// The sequence-parallel step's attention (bf16): head_split CTAs per head,
// as many as one wave of CTAs holds (at least one), and enough to keep each
// CTA's part of a list within kIdxCap; a.n_split (partial slots per head)
// bounds head_split.
cudaError_t launch_attend_split(AttendArgs &a, cudaStream_t s)
{
    int64_t P = 0;
    if (cudaError_t e = occupancy_grid(attend_head_kernel, tc::kThreads, tc::kSmem, &P)) return e;
    const int64_t heads = int64_t(a.B) * a.H_q;
    int64_t split = std::max(ceil_div(a.topk, tc::kIdxCap), std::max<int64_t>(P / heads, 1));
    if (split > a.n_split) split = a.n_split;
    if (split * heads >= (int64_t(1) << 31) || ceil_div(a.topk, split) > tc::kIdxCap)
        return cudaErrorInvalidValue;
    a.head_split = int(split);
    a.head_per_cta = split == 1;  // merged inside the CTA: no combine launch
    a.n_workers = 0;
    return launch_pdl(attend_head_kernel, dim3(unsigned(split * heads)), dim3(tc::kThreads),
                      tc::kSmem, s, a);
}

// The merge of the split heads: launched right behind launch_attend (whose
// call sets a.n_workers), with programmatic dependent launch.
cudaError_t launch_combine(const AttendArgs &a, cudaStream_t s)
{
    if (a.head_per_cta) return cudaSuccess;  // merged inside the attention CTAs
    const int64_t heads = int64_t(a.B) * a.H_q;
    // most partials one head can have: its CTAs when split, else the
    // stream-K workers that can touch one head's topk rows
    int64_t most = a.head_split;
    if (most <= 0) {
        const int64_t T = heads * a.topk, per = a.n_workers > 0 ? T / a.n_workers : T;
        most = (a.topk + (per > 0 ? per : 1) - 1) / (per > 0 ? per : 1) + 1;
    }
    // the same carveout as the attention kernel, so its CTAs can join the
    // SMs without a shared-memory reconfiguration
    if (most > kCombineRound) {  // four warps per head: up to 64 partials in one round trip
        if (cudaError_t e = ensure_smem_attr(reinterpret_cast<const void *>(combine_kernel<4>), 0))
            return e;
        return launch_pdl(combine_kernel<4>, dim3(unsigned(heads)), dim3(32 * kCombineWarps), 0, s,
                          a);
    }
    if (cudaError_t e = ensure_smem_attr(reinterpret_cast<const void *>(combine_kernel<1>), 0))
        return e;
    return launch_pdl(combine_kernel<1>, dim3(unsigned(ceil_div(heads, kCombineWarps))),
                      dim3(32 * kCombineWarps), 0, s, a);
}

}  // namespace hata
