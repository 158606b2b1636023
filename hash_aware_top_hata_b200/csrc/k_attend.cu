// k_attend.cu -- top-k selection fused with gather + exact softmax attention.
//
// HATA review page (arXiv 2506.02572): "What carries the argument" (the top-k
// indices select K/V for attention; the page's implementation fuses the
// gather into FlashAttention) and major comment 1 (Algorithm 3: the top-k
// over Hamming scores; boundary ties here go to the lower token index).
//
// Grid: (chunk of 4096 tokens, b * H_q + h_q).  Each CTA
//   1. reads its chunk's u8 distances (L2-resident from the scoring kernel)
//      and the plan (T, take_c, off_c), and compacts, in token order, the keys
//      with dist < T plus its share of dist == T keys into a shared-memory
//      index list (two block scans; no sort);
//   2. writes those indices to sel_idx (optional) at off_c -- so the global
//      list comes out in ascending token order;
//   3. gathers the selected K and V rows straight from the cache (each 16-lane
//      half-warp owns one 256-byte bf16 row: one 128-bit load per lane, eight
//      rows per half-warp in flight) and runs an online softmax in fp32,
//      base-2 exponent with the scale folded into q;
//   4. merges its eight half-warp states into one partial (m, l, acc[128]);
//      the last CTA of the head (fence + arrival counter, no waiting) merges
//      all chunk partials into out = acc / l.
#include "block_scan.cuh"
#include "hata_internal.cuh"

namespace hata {
namespace {

constexpr int kWarps = kAttnThreads / 32;
constexpr int kRowsPerHalf = 8;        // rows gathered per half-warp per round
constexpr int kHalves = kWarps * 2;
constexpr int kBytesPerThread = kChunk / kAttnThreads;  // 32 distances

__device__ __forceinline__ int64_t clamp_len(int32_t sl, int64_t max_len, int64_t n_cap)
{
    int64_t l = sl < 0 ? 0 : sl;
    l = l < max_len ? l : max_len;
    return l < n_cap ? l : n_cap;
}

// 8 consecutive elements of a row (starting at element e0) as fp32.
template <bool BF16>
struct RowFrag;

template <>
struct RowFrag<true> {
    uint4 v;
    __device__ __forceinline__ void zero() { v = make_uint4(0, 0, 0, 0); }
    __device__ __forceinline__ void load(const void *base, int64_t elem)
    {
        v = __ldg(reinterpret_cast<const uint4 *>(reinterpret_cast<const uint16_t *>(base) + elem));
    }
    __device__ __forceinline__ void to_f32(float (&f)[8]) const
    {
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            f[2 * i] = __uint_as_float(w[i] << 16);
            f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    }
};

template <>
struct RowFrag<false> {
    float4 a, b;
    __device__ __forceinline__ void zero() { a = b = make_float4(0.f, 0.f, 0.f, 0.f); }
    __device__ __forceinline__ void load(const void *base, int64_t elem)
    {
        const float4 *p = reinterpret_cast<const float4 *>(reinterpret_cast<const float *>(base) + elem);
        a = __ldg(p);
        b = __ldg(p + 1);
    }
    __device__ __forceinline__ void to_f32(float (&f)[8]) const
    {
        f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
        f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
    }
};

template <bool BF16>
__global__ void __launch_bounds__(kAttnThreads) attend_kernel(AttendArgs a)
{
    const int c = blockIdx.x;
    const size_t bh = blockIdx.y;
    const int b = int(bh / a.H_q), hq = int(bh % a.H_q), h = hq / a.G;
    const int64_t len = clamp_len(a.seq_len[b], a.max_seq_len, a.n_cap);
    const int64_t nch = len > 0 ? ceil_div(len, kChunk) : 1;
    if (c >= nch) return;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    __shared__ int32_t idx_s[kChunk];
    __shared__ int scan_s[kWarps + 1];
    __shared__ float red_m[kHalves], red_l[kHalves];
    __shared__ __align__(16) float red_acc[kHalves][kD];
    __shared__ int s_last;

    const PlanHead ph = a.plan_head[bh];
    const PlanChunk pc = a.plan_chunk[bh * a.n_chunks + c];

    // ---- 1. ordered compaction of this chunk's selected keys ----
    const uint4 *dp = reinterpret_cast<const uint4 *>(a.dist + bh * a.dist_row +
                                                      int64_t(c) * kChunk) + tid * 2;
    const uint4 d0 = __ldg(dp), d1 = __ldg(dp + 1);
    const uint32_t dw[8] = {d0.x, d0.y, d0.z, d0.w, d1.x, d1.y, d1.z, d1.w};
    const uint32_t T4 = ph.T >= 0 ? uint32_t(ph.T) * 0x01010101u : 0u;
    uint32_t lt[8], eq[8];
    int n_lt = 0, n_eq = 0;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        lt[k] = ph.T >= 0 ? __vcmpltu4(dw[k], T4) : 0u;
        eq[k] = ph.T >= 0 ? __vcmpeq4(dw[k], T4) : 0u;
        n_lt += __popc(lt[k]) >> 3;
        n_eq += __popc(eq[k]) >> 3;
    }
    int tot;
    const int eq_before = block_exclusive_scan<kAttnThreads>(n_eq, scan_s, &tot);
    const int my_take = max(0, min(pc.take - eq_before, n_eq));
    int total;
    int wpos = block_exclusive_scan<kAttnThreads>(n_lt + my_take, scan_s, &total);
    {
        int eq_seen = 0;
        const int32_t tok0 = int32_t(int64_t(c) * kChunk) + tid * kBytesPerThread;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const bool is_lt = (lt[k] >> (8 * e)) & 1u;
                const bool is_eq = (eq[k] >> (8 * e)) & 1u;
                const bool take = is_lt || (is_eq && eq_seen < my_take);
                eq_seen += is_eq;
                if (take) idx_s[wpos++] = tok0 + k * 4 + e;
            }
        }
    }
    __syncthreads();
    if (a.sel_idx) {
        int32_t *dst = a.sel_idx + bh * a.topk + pc.off;
        const int lim = min(total, a.topk - pc.off);
        for (int i = tid; i < lim; i += kAttnThreads) dst[i] = idx_s[i];
    }

    // ---- 3. gather + online softmax ----
    const int half = lane >> 4, l16 = lane & 15, hw = warp * 2 + half;
    float qv[8];
    {
        const float4 *qp = reinterpret_cast<const float4 *>(a.q + bh * kD + l16 * 8);
        const float4 x = __ldg(qp), y = __ldg(qp + 1);
        qv[0] = x.x; qv[1] = x.y; qv[2] = x.z; qv[3] = x.w;
        qv[4] = y.x; qv[5] = y.y; qv[6] = y.z; qv[7] = y.w;
#pragma unroll
        for (int e = 0; e < 8; ++e) qv[e] *= a.scale_log2;
    }
    const int64_t slab = (int64_t(b) * a.H_kv + h) * a.n_cap;  // row of token 0
    float m = -INFINITY, l = 0.0f, acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.0f;

    for (int base = 0; base < total; base += kHalves * kRowsPerHalf) {
        RowFrag<BF16> kf[kRowsPerHalf], vf[kRowsPerHalf];
        bool valid[kRowsPerHalf];
#pragma unroll
        for (int u = 0; u < kRowsPerHalf; ++u) {
            const int ri = base + hw * kRowsPerHalf + u;
            const int32_t row = ri < total ? idx_s[ri] : -1;
            // distances past seq_len are 255 and never selected; the range
            // check keeps even a corrupted distance row inside the cache
            valid[u] = row >= 0 && row < len;
            if (valid[u]) {
                const int64_t e0 = (slab + row) * kD + l16 * 8;
                kf[u].load(a.K, e0);
                vf[u].load(a.V, e0);
            } else {
                kf[u].zero();  // weight 0 must meet a finite value
                vf[u].zero();
            }
        }
        float s[kRowsPerHalf];
        float mx = m;
#pragma unroll
        for (int u = 0; u < kRowsPerHalf; ++u) {
            float kx[8];
            kf[u].to_f32(kx);
            float p = 0.0f;
#pragma unroll
            for (int e = 0; e < 8; ++e) p = fmaf(qv[e], kx[e], p);
#pragma unroll
            for (int o = 8; o > 0; o >>= 1) p += __shfl_xor_sync(0xffffffffu, p, o);
            s[u] = valid[u] ? p : -INFINITY;
            mx = fmaxf(mx, s[u]);
        }
        const float mref = mx == -INFINITY ? 0.0f : mx;
        const float alpha = exp2f(m - mref);
        l *= alpha;
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] *= alpha;
#pragma unroll
        for (int u = 0; u < kRowsPerHalf; ++u) {
            const float p = exp2f(s[u] - mref);
            l += p;
            float vx[8];
            vf[u].to_f32(vx);
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[e] = fmaf(p, vx[e], acc[e]);
        }
        m = mx;
    }

    // ---- 4. merge half-warps, then chunks ----
    if (l16 == 0) {
        red_m[hw] = m;
        red_l[hw] = l;
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) red_acc[hw][l16 * 8 + e] = acc[e];
    __syncthreads();
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
        float *pp = a.part + (bh * a.n_chunks + c) * kPartStride;
        if (tid == 0) {
            pp[0] = M;
            pp[1] = L;
        }
        pp[4 + tid] = A;
    }
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = atomicAdd(a.cnt_attn + bh, 1u) == uint32_t(nch - 1);
    __syncthreads();
    if (!s_last) return;
    __threadfence();

    float M = -INFINITY, L = 0.0f, A = 0.0f;
    const float *pp = a.part + bh * a.n_chunks * kPartStride;
    for (int64_t cc = 0; cc < nch; ++cc, pp += kPartStride) {
        const float mc = __ldcg(pp), lc = __ldcg(pp + 1), ac = __ldcg(pp + 4 + tid);
        if (mc == -INFINITY) continue;
        const float Mn = fmaxf(M, mc);
        const float so = exp2f(M - Mn), sn = exp2f(mc - Mn);
        L = L * so + lc * sn;
        A = A * so + ac * sn;
        M = Mn;
    }
    a.out[bh * kD + tid] = L > 0.0f ? A / L : 0.0f;
}

}  // namespace

cudaError_t launch_attend(const AttendArgs &a, bool bf16, cudaStream_t s)
{
    const dim3 grid(unsigned(a.n_chunks), unsigned(a.B * a.H_q));
    if (bf16)
        attend_kernel<true><<<grid, kAttnThreads, 0, s>>>(a);
    else
        attend_kernel<false><<<grid, kAttnThreads, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace hata
