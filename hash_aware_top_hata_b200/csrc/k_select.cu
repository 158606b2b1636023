// k_select.cu -- top-k selection over the Hamming distances, no sort.
//
// HATA review page (arXiv 2506.02572), major comment 1 (Algorithm 3): the
// top-k runs over Hamming scores that take only 129 values, so the boundary
// usually falls inside a large bucket of equal scores; the page leaves the
// choice inside that bucket open.  Here it goes to the lower token index, so
// the selected set is unique:
//   k_eff = min(topk, len)
//   T     = the smallest distance t with #(dist <= t) >= k_eff
//   S     = {n : dist[n] < T}  +  the r = k_eff - #(dist < T) lowest-index
//           keys with dist[n] == T.
//
// Grid: (segment of kSegChunks scoring chunks, b * H_q + h_q), 256 threads.
// A CTA finds T from the head's total histogram and, from the cumulative
// histograms of the chunks before its segment, the output offset of its
// first key and how many boundary keys precede it (ties are taken greedily
// in token order).  Then it walks its chunks in order: each thread owns 16
// consecutive distances (one 16-byte load), counts "< T" and "== T" with
// SIMD byte compares, and ONE block scan of the packed pair gives every
// thread its output position -- the ties a thread may take follow from the
// ties before it: taken_before = min(ties_before, r - ties_before_chunk).
// Indices are written straight to the head's list, ascending.
#include "block_scan.cuh"
#include "hata_internal.cuh"

namespace hata {
namespace {

constexpr int kThreads = 128;
constexpr int kWarps = kThreads / 32;
constexpr int kPerThread = kChunk / kThreads;  // 32 distances: two 16-byte loads
static_assert(kPerThread == 32, "two 16-byte loads per thread per chunk");
static_assert(kSelSegChunks == 2, "the distances of a segment are loaded up front");

__device__ __forceinline__ int64_t clamp_len(int32_t sl, int64_t max_len, int64_t n_cap)
{
    int64_t l = sl < 0 ? 0 : sl;
    l = l < max_len ? l : max_len;
    return l < n_cap ? l : n_cap;
}

// Block-wide sum of a 64-bit value (all threads get the total).
__device__ __forceinline__ int64_t block_sum64(int64_t v, int64_t *scratch)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) scratch[warp] = v;
    __syncthreads();
    int64_t t = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) t += scratch[w];
    __syncthreads();
    return t;
}

__global__ void __launch_bounds__(kThreads) select_kernel(SelectArgs a)
{
    const int seg = blockIdx.x;
    const size_t bh = blockIdx.y;
    const int b = int(bh / a.H_q);
    const int64_t len = clamp_len(a.seq_len[b], a.max_seq_len, a.n_cap);
    const int64_t nch = len > 0 ? ceil_div(len, kChunk) : 1;
    const int64_t c0 = int64_t(seg) * kSelSegChunks;
    if (c0 >= nch) return;
    const int64_t c1 = c0 + kSelSegChunks < nch ? c0 + kSelSegChunks : nch;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int k_eff = int(int64_t(a.topk) < len ? int64_t(a.topk) : len);
    int32_t *idx = a.idx + bh * a.topk;

    __shared__ int scan_s[kWarps + 1];
    __shared__ int64_t red_s[kWarps];
    __shared__ int s_T, s_nless;

    if (seg == 0)
        for (int i = k_eff + tid; i < a.topk; i += kThreads) idx[i] = -1;
    if (k_eff <= 0) return;

    // the segment's distances: in flight while T and the offsets are found
    const uint8_t *drow = a.dist + bh * a.dist_row;
    uint4 dv[kSelSegChunks][2];
#pragma unroll
    for (int k = 0; k < kSelSegChunks; ++k) {
        const uint4 *dp = reinterpret_cast<const uint4 *>(drow + (c0 + k) * kChunk) + 2 * tid;
        const bool in = c0 + k < c1;
        dv[k][0] = in ? __ldg(dp) : make_uint4(0, 0, 0, 0);
        dv[k][1] = in ? __ldg(dp + 1) : make_uint4(0, 0, 0, 0);
    }

    // ---- T from the head's total histogram ----
    if (warp == 0) {
        const uint32_t *ht = a.hist_total + bh * kHistStride;
        uint32_t v[5];
        uint32_t run = 0;
#pragma unroll
        for (int e = 0; e < 5; ++e) {
            const int t = lane * 5 + e;
            v[e] = t < kBins ? __ldg(ht + t) : 0u;
            run += v[e];
        }
        uint32_t acc = uint32_t(warp_inclusive_scan(int(run))) - run;
        int T = -1;
        uint32_t less = 0;
#pragma unroll
        for (int e = 0; e < 5; ++e) {
            if (T < 0 && lane * 5 + e < kBins && acc + v[e] >= uint32_t(k_eff)) {
                T = lane * 5 + e;
                less = acc;
            }
            acc += v[e];
        }
        // cumulative counts are monotone: the lowest lane that found a bin holds T
        const unsigned found = __ballot_sync(0xffffffffu, T >= 0);
        const int src = found ? __ffs(int(found)) - 1 : 0;
        const int Tf = __shfl_sync(0xffffffffu, T, src);
        const int nl = __shfl_sync(0xffffffffu, int(less), src);
        if (lane == 0) {
            s_T = found ? Tf : 128;  // unreachable fallback: every key qualifies
            s_nless = found ? nl : 0;
        }
    }
    __syncthreads();
    const int T = s_T;
    const int r_ties = k_eff - s_nless;  // boundary keys taken over the whole head

    // ---- keys (< T) and boundary keys (== T) in the chunks before c0 ----
    int64_t less_before = 0, ties_before = 0;
    {
        int64_t lsum = 0, tsum = 0;
        for (int64_t cc = tid; cc < c0; cc += kThreads) {
            const uint32_t *cp = a.cum + (bh * a.n_chunks + cc) * kCumStride;
            const uint32_t le = T > 0 ? __ldg(cp + T - 1) : 0u;
            lsum += le;
            tsum += __ldg(cp + T) - le;
        }
        if (c0 > 0) {
            less_before = block_sum64(lsum, red_s);
            ties_before = block_sum64(tsum, red_s);
        }
    }
    int64_t off = less_before + (ties_before < r_ties ? ties_before : r_ties);

    // ---- ordered compaction, chunk by chunk ----
    const uint32_t T4 = uint32_t(T) * 0x01010101u;
#pragma unroll
    for (int k = 0; k < kSelSegChunks; ++k) {
        const int64_t c = c0 + k;
        if (c >= c1) break;
        const uint32_t dw[8] = {dv[k][0].x, dv[k][0].y, dv[k][0].z, dv[k][0].w,
                                dv[k][1].x, dv[k][1].y, dv[k][1].z, dv[k][1].w};
        // byte masks (0xff / 0x00) -> one bit per distance: byte e of word w
        // becomes bit 4w + e (the multiply gathers bits 7, 15, 23, 31 into 28..31)
        uint32_t lt_bits = 0, eq_bits = 0;
#pragma unroll
        for (int w = 0; w < 8; ++w) {
            const uint32_t lt = __vcmpltu4(dw[w], T4) & 0x80808080u;
            const uint32_t eq = __vcmpeq4(dw[w], T4) & 0x80808080u;
            lt_bits |= ((lt * 0x00204081u) >> 28) << (4 * w);
            eq_bits |= ((eq * 0x00204081u) >> 28) << (4 * w);
        }
        const int n_lt = __popc(lt_bits), n_eq = __popc(eq_bits);
        // one scan of the packed pair (each count <= 4096 per chunk)
        int tot;
        const int before = block_exclusive_scan<kThreads>((n_lt << 16) | n_eq, scan_s, &tot);
        const int lt_before = before >> 16, eq_before = before & 0xffff;
        const int chunk_eq = tot & 0xffff, chunk_lt = tot >> 16;
        const int64_t room = r_ties - ties_before > 0 ? r_ties - ties_before : 0;  // ties left
        const int take_chunk = int(room < chunk_eq ? room : chunk_eq);
        const int taken_before = eq_before < take_chunk ? eq_before : take_chunk;
        int my_take = take_chunk - eq_before;
        my_take = my_take < 0 ? 0 : (my_take > n_eq ? n_eq : my_take);
        uint32_t sel = lt_bits;
        for (int t = 0; t < my_take; ++t) {  // the lowest-index my_take ties
            sel |= eq_bits & (0u - eq_bits);
            eq_bits &= eq_bits - 1u;
        }
        int64_t pos = off + lt_before + taken_before;
        const int32_t tok0 = int32_t(c * kChunk) + tid * kPerThread;
        while (sel) {
            const int e = __ffs(int(sel)) - 1;
            sel &= sel - 1u;
            if (pos < a.topk) idx[pos] = tok0 + e;
            ++pos;
        }
        off += chunk_lt + take_chunk;
        ties_before += chunk_eq;
    }
}

}  // namespace

cudaError_t launch_select(const SelectArgs &a, cudaStream_t s)
{
    const dim3 grid(unsigned(ceil_div(a.n_chunks, kSelSegChunks)), unsigned(a.B * a.H_q));
    select_kernel<<<grid, kThreads, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace hata
