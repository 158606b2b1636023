// k_dense.cu -- dense decode attention over every cached key: the full
// attention HATA's speedup is quoted against (HATA review page, abstract:
// "up to 7.2x speedup compared to vanilla full attention"), and the reference
// the sparse path must equal when k >= seq_len.
//
// Split-K flash-decode.  Grid: (chunk of 2048 tokens, b * H_kv + h_kv, group
// of <= 4 query heads).  Every K/V row is loaded once per CTA and used by all
// query heads of the group (grouped-query attention shares the KV head);
// rows are streamed with 128-bit loads, 16 lanes per 256-byte bf16 row.
// Online softmax in fp32 with base-2 exponents; the last CTA of a
// (b, h_kv, group) merges the chunk partials.
#include "hata_internal.cuh"

namespace hata {
namespace {

constexpr int kThreads = 128;
constexpr int kWarps = kThreads / 32;
constexpr int kHalves = kWarps * 2;
constexpr int kU = 4;  // rows per half-warp per round
constexpr int kHeads = kDenseHeads;

template <bool BF16>
__device__ __forceinline__ void load8(const void *base, int64_t elem, float (&f)[8])
{
    if (BF16) {
        const uint4 v = __ldcs(reinterpret_cast<const uint4 *>(
            reinterpret_cast<const uint16_t *>(base) + elem));
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            f[2 * i] = __uint_as_float(w[i] << 16);
            f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    } else {
        const float4 *p = reinterpret_cast<const float4 *>(reinterpret_cast<const float *>(base) + elem);
        const float4 x = __ldcs(p), y = __ldcs(p + 1);
        f[0] = x.x; f[1] = x.y; f[2] = x.z; f[3] = x.w;
        f[4] = y.x; f[5] = y.y; f[6] = y.z; f[7] = y.w;
    }
}

template <bool BF16, int GB>
__global__ void __launch_bounds__(kThreads) dense_kernel(DenseArgs a)
{
    const int c = blockIdx.x;
    const int b = blockIdx.y / a.H_kv, h = blockIdx.y % a.H_kv;
    const int z = blockIdx.z, g0 = z * kHeads;
    const int ng = min(GB, a.G - g0);
    const int64_t len = clamp_len(a.seq_len[b], a.max_seq_len, a.n_cap);
    const int64_t nch = len > 0 ? ceil_div(len, kDenseChunk) : 1;
    if (c >= nch) return;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int half = lane >> 4, l16 = lane & 15, hw = warp * 2 + half;
    __shared__ float red_m[GB][kHalves], red_l[GB][kHalves];
    __shared__ __align__(16) float red_acc[GB][kHalves][kD];
    __shared__ int s_last;

    const size_t bh0 = size_t(b) * a.H_q + size_t(h) * a.G + g0;
    float qv[GB][8];
#pragma unroll
    for (int g = 0; g < GB; ++g) {
#pragma unroll
        for (int e = 0; e < 8; ++e)
            qv[g][e] = g < ng ? a.q[(bh0 + g) * kD + l16 * 8 + e] * a.scale_log2 : 0.0f;
    }
    float m[GB], l[GB], acc[GB][8];
#pragma unroll
    for (int g = 0; g < GB; ++g) {
        m[g] = -INFINITY;
        l[g] = 0.0f;
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[g][e] = 0.0f;
    }

    const int64_t slab = (int64_t(b) * a.H_kv + h) * a.n_cap;
    const int64_t n0 = int64_t(c) * kDenseChunk;
    const int64_t n1 = (n0 + kDenseChunk < len) ? n0 + kDenseChunk : len;
    for (int64_t base = n0; base < n1; base += kHalves * kU) {
        float kx[kU][8], vx[kU][8];
        bool valid[kU];
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            const int64_t n = base + hw * kU + u;
            valid[u] = n < n1;
            const int64_t e0 = (slab + (valid[u] ? n : n0)) * kD + l16 * 8;
            load8<BF16>(a.K, e0, kx[u]);
            load8<BF16>(a.V, e0, vx[u]);
        }
#pragma unroll
        for (int g = 0; g < GB; ++g) {
            float s[kU];
            float mx = m[g];
#pragma unroll
            for (int u = 0; u < kU; ++u) {
                float p = 0.0f;
#pragma unroll
                for (int e = 0; e < 8; ++e) p = fmaf(qv[g][e], kx[u][e], p);
#pragma unroll
                for (int o = 8; o > 0; o >>= 1) p += __shfl_xor_sync(0xffffffffu, p, o);
                s[u] = valid[u] ? p : -INFINITY;
                mx = fmaxf(mx, s[u]);
            }
            const float mref = mx == -INFINITY ? 0.0f : mx;
            const float alpha = exp2f(m[g] - mref);
            l[g] *= alpha;
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[g][e] *= alpha;
#pragma unroll
            for (int u = 0; u < kU; ++u) {
                const float p = exp2f(s[u] - mref);
                l[g] += p;
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[g][e] = fmaf(p, vx[u][e], acc[g][e]);
            }
            m[g] = mx;
        }
    }

#pragma unroll
    for (int g = 0; g < GB; ++g) {
        if (l16 == 0) {
            red_m[g][hw] = m[g];
            red_l[g][hw] = l[g];
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) red_acc[g][hw][l16 * 8 + e] = acc[g][e];
    }
    __syncthreads();
    for (int g = 0; g < ng; ++g) {
        float M = -INFINITY;
#pragma unroll
        for (int i = 0; i < kHalves; ++i) M = fmaxf(M, red_m[g][i]);
        const float Mref = M == -INFINITY ? 0.0f : M;
        float L = 0.0f, A = 0.0f;
#pragma unroll
        for (int i = 0; i < kHalves; ++i) {
            const float w = exp2f(red_m[g][i] - Mref);
            L = fmaf(red_l[g][i], w, L);
            A = fmaf(red_acc[g][i][tid], w, A);
        }
        float *pp = a.part + ((bh0 + g) * a.n_chunks + c) * kPartStride;
        if (tid == 0) {
            pp[0] = M;
            pp[1] = L;
        }
        pp[4 + tid] = A;
    }
    __threadfence();
    __syncthreads();
    if (tid == 0)
        s_last = atomicAdd(a.cnt + size_t(blockIdx.y) * a.zgroups + z, 1u) == uint32_t(nch - 1);
    __syncthreads();
    if (!s_last) return;
    __threadfence();

    for (int g = 0; g < ng; ++g) {
        float M = -INFINITY, L = 0.0f, A = 0.0f;
        const float *pp = a.part + (bh0 + g) * a.n_chunks * kPartStride;
        for (int64_t cc = 0; cc < nch; ++cc, pp += kPartStride) {
            const float mc = __ldcg(pp), lc = __ldcg(pp + 1), ac = __ldcg(pp + 4 + tid);
            if (mc == -INFINITY) continue;
            const float Mn = fmaxf(M, mc);
            const float so = exp2f(M - Mn), sn = exp2f(mc - Mn);
            L = L * so + lc * sn;
            A = A * so + ac * sn;
            M = Mn;
        }
        a.out[(bh0 + g) * kD + tid] = L > 0.0f ? A / L : 0.0f;
    }
}

template <bool BF16>
cudaError_t launch_dense_t(const DenseArgs &a, cudaStream_t s)
{
    const dim3 grid(unsigned(a.n_chunks), unsigned(a.B * a.H_kv), unsigned(a.zgroups));
    const int gb = a.G < kHeads ? a.G : kHeads;
    switch (gb) {
    case 1: dense_kernel<BF16, 1><<<grid, kThreads, 0, s>>>(a); break;
    case 2: dense_kernel<BF16, 2><<<grid, kThreads, 0, s>>>(a); break;
    case 3: dense_kernel<BF16, 3><<<grid, kThreads, 0, s>>>(a); break;
    default: dense_kernel<BF16, 4><<<grid, kThreads, 0, s>>>(a); break;
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_dense(const DenseArgs &a, bool bf16, cudaStream_t s)
{
    return bf16 ? launch_dense_t<true>(a, s) : launch_dense_t<false>(a, s);
}

}  // namespace hata
