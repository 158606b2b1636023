// k_sp.cu -- the exchange-side kernels of the sequence-parallel decode step.
//
// HATA review page (arXiv 2506.02572), major comment 1 (Algorithm 3): the
// top-k is a threshold on a histogram of r + 1 Hamming values, with the
// boundary bucket going to the lower token indices.  When a head's keys are
// split into contiguous shards, one per rank (rank order = token order), that
// selection needs only each shard's histogram:
//   T, #(< T) and the ties to take come from the sum of all shards' histograms;
//   the ties at T go to the lowest ranks first (their tokens are lower);
//   shard s keeps  k_s = #_s(< T) + clamp(r_ties - ties_before_s, 0, #_s(== T))
// and its local top-k_s under the same tie rule is exactly its part of the
// global selection.  Attention over a shard's part gives an unnormalised
// partial (m, l, acc); the log-sum-exp merge of all shards' partials is the
// attention over the whole selection.
//
//   sp_hist_kernel   one shard's per-head histogram (sum of its tile rows)
//   sp_quota_kernel  k_s per head from every shard's histogram
//   sp_merge_kernel  out = merge of every shard's partial
#include "hata_internal.cuh"

namespace hata {
namespace {

constexpr int kSpWarps = 4;  // heads per CTA (one warp each)
constexpr int kSpBPL = 9;    // bins per lane: 32 * 9 = 288 >= kSpHistWords
static_assert(32 * kSpBPL >= kSpHistWords, "a warp covers a histogram row");

__global__ void __launch_bounds__(32 * kSpWarps) sp_hist_kernel(const uint32_t *hist,
                                                                int64_t n_tiles, int stride,
                                                                int64_t BH, uint32_t *out)
{
    pdl_trigger();
    const int lane = threadIdx.x & 31;
    const int64_t bh = int64_t(blockIdx.x) * kSpWarps + (threadIdx.x >> 5);
    pdl_wait();  // the scoring kernel's tile histograms
    if (bh >= BH) return;
    const uint32_t *row = hist + bh * n_tiles * stride;
    for (int e = 0; e < kSpBPL; ++e) {
        const int bin = lane + 32 * e;
        if (bin >= kSpHistWords) break;
        uint32_t v = 0;
        if (bin < stride) {
#pragma unroll 8
            for (int64_t t = 0; t < n_tiles; ++t) v += __ldg(row + t * stride + bin);  // 8 in flight
        }
        out[bh * kSpHistWords + bin] = v;
    }
}

// Inclusive warp scan of 64-bit counts.
__device__ __forceinline__ uint64_t warp_scan_u64(uint64_t v, int lane)
{
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint64_t n = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += n;
    }
    return v;
}

__global__ void __launch_bounds__(32 * kSpWarps) sp_quota_kernel(const uint32_t *hist_all,
                                                                 int world, int rank, int64_t BH,
                                                                 int topk, int bins,
                                                                 int32_t *k_head)
{
    const int lane = threadIdx.x & 31;
    const int64_t bh = int64_t(blockIdx.x) * kSpWarps + (threadIdx.x >> 5);
    if (bh >= BH) return;
    // lane l owns bins kSpBPL l .. kSpBPL l + kSpBPL - 1: all shards' counts,
    // this shard's, and those of the shards before it
    uint64_t tot[kSpBPL], before[kSpBPL];
    uint32_t mine[kSpBPL];
#pragma unroll
    for (int e = 0; e < kSpBPL; ++e) tot[e] = before[e] = mine[e] = 0;
#pragma unroll 4
    for (int w = 0; w < world; ++w) {  // the loads of 4 ranks in flight together
        const uint32_t *row = hist_all + (int64_t(w) * BH + bh) * kSpHistWords;
#pragma unroll
        for (int e = 0; e < kSpBPL; ++e) {
            const int bin = lane * kSpBPL + e;
            const uint32_t v = bin < bins ? __ldg(row + bin) : 0u;
            tot[e] += v;
            if (w < rank) before[e] += v;
            if (w == rank) mine[e] = v;
        }
    }
    uint64_t run = 0;
#pragma unroll
    for (int e = 0; e < kSpBPL; ++e) run += tot[e];
    const uint64_t all = __shfl_sync(0xffffffffu, warp_scan_u64(run, lane), 31);
    const uint64_t k_eff = uint64_t(topk) < all ? uint64_t(topk) : all;
    uint64_t acc = warp_scan_u64(run, lane) - run;
    int Tl = -1;
    uint64_t less_l = 0;
#pragma unroll
    for (int e = 0; e < kSpBPL; ++e) {
        if (Tl < 0 && lane * kSpBPL + e < bins && acc + tot[e] >= k_eff) {
            Tl = lane * kSpBPL + e;
            less_l = acc;
        }
        acc += tot[e];
    }
    const unsigned found = __ballot_sync(0xffffffffu, Tl >= 0);
    const int src = found ? __ffs(int(found)) - 1 : 0;
    const int T = __shfl_sync(0xffffffffu, Tl, src);
    const uint64_t n_less = __shfl_sync(0xffffffffu, less_l, src);
    // this shard's keys below T, and the ties at T of this shard and before it
    uint64_t l = 0, tb = 0, tm = 0;
#pragma unroll
    for (int e = 0; e < kSpBPL; ++e) {
        const int bin = lane * kSpBPL + e;
        l += bin < T ? mine[e] : 0u;
        tb += bin == T ? before[e] : 0u;
        tm += bin == T ? mine[e] : 0u;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        l += __shfl_xor_sync(0xffffffffu, l, o);
        tb += __shfl_xor_sync(0xffffffffu, tb, o);
        tm += __shfl_xor_sync(0xffffffffu, tm, o);
    }
    if (lane == 0) {
        int64_t k = 0;
        if (k_eff > 0 && found) {
            const int64_t r_ties = int64_t(k_eff - n_less);  // boundary keys over all shards
            int64_t take = r_ties - int64_t(tb);
            take = take < 0 ? 0 : (take > int64_t(tm) ? int64_t(tm) : take);
            k = int64_t(l) + take;
        }
        k_head[bh] = int32_t(k);
    }
}

// One warp per head, an online merge over rounds of kRound ranks: all loads
// of a round (lane j < kRound: rank j's m and l; every lane: its 4 output
// dims of each rank's acc) are issued before any is used, so a step of up to
// kRound ranks costs one memory round trip.
__global__ void __launch_bounds__(32 * kSpWarps) sp_merge_kernel(const float *part_all, int world,
                                                                 int64_t BH, float *out)
{
    constexpr int kRound = 8;
    const int lane = threadIdx.x & 31;
    const int64_t bh = int64_t(blockIdx.x) * kSpWarps + (threadIdx.x >> 5);
    if (bh >= BH) return;
    auto rec = [&](int w) { return part_all + (int64_t(w) * BH + bh) * kPartStride; };
    float M = -INFINITY, L = 0.0f, A[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    for (int w0 = 0; w0 < world; w0 += kRound) {
        const bool mine = lane < kRound && w0 + lane < world;
        const float mc = mine ? __ldg(rec(w0 + lane)) : -INFINITY;
        const float lc = mine ? __ldg(rec(w0 + lane) + 1) : 0.0f;
        float acc[kRound][4];
#pragma unroll
        for (int j = 0; j < kRound; ++j)
#pragma unroll
            for (int i = 0; i < 4; ++i)
                acc[j][i] = w0 + j < world ? __ldg(rec(w0 + j) + 4 + lane + 32 * i) : 0.0f;
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
        for (int j = 0; j < kRound; ++j) {
            const float wj = __shfl_sync(0xffffffffu, wc, j);
#pragma unroll
            for (int i = 0; i < 4; ++i) A[i] = fmaf(acc[j][i], wj, A[i]);
        }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) out[bh * kD + lane + 32 * i] = L > 0.0f ? A[i] / L : 0.0f;
}

}  // namespace

cudaError_t launch_sp_hist(const uint32_t *hist, int64_t n_tiles, int stride, int64_t BH,
                           uint32_t *out, cudaStream_t s)
{
    return launch_pdl(sp_hist_kernel, dim3(unsigned(ceil_div(BH, kSpWarps))), dim3(32 * kSpWarps),
                      0, s, hist, n_tiles, stride, BH, out);
}

cudaError_t launch_sp_quota(const uint32_t *hist_all, int world, int rank, int64_t BH, int topk,
                            int bins, int32_t *k_head, cudaStream_t s)
{
    // a plain launch: its input comes from the exchange, not from a kernel
    // of this library
    sp_quota_kernel<<<unsigned(ceil_div(BH, kSpWarps)), 32 * kSpWarps, 0, s>>>(
        hist_all, world, rank, BH, topk, bins, k_head);
    return cudaGetLastError();
}

cudaError_t launch_sp_merge(const float *part_all, int world, int64_t BH, float *out,
                            cudaStream_t s)
{
    sp_merge_kernel<<<unsigned(ceil_div(BH, kSpWarps)), 32 * kSpWarps, 0, s>>>(part_all, world,
                                                                             BH, out);
    return cudaGetLastError();
}

}  // namespace hata
