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
// Grid: (part, b * H_q + h_q), 256 threads.  A tile is 256 x 128 = 32K
// tokens, each thread owning 128 consecutive distances (eight 16-byte
// loads); the launcher splits each head's tiles into as many parts as fill
// one wave of CTAs, and a CTA walks its part's tiles in order, carrying the
// counts.  The CTA issues its first tile's loads, finds T from the head's
// total histogram and -- for parts after the first -- the keys below T and
// the boundary keys before the part from the scoring kernel's cumulative
// chunk histograms.  Each thread turns its 128 distances into "< T" and
// "== T" bit masks with byte-wise integer compares, ONE block scan of the
// two counts gives every thread its output position, and the ties a thread
// may take follow from the ties before it: taken_before = min(ties_before,
// room).  Indices are written straight to the head's list, ascending.
#include "block_scan.cuh"
#include "hata_internal.cuh"

namespace hata {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kPer = 128;                               // distances per thread
constexpr int kPieces = kPer / 16;                      // 16-byte loads per thread
constexpr int kGroups = kPer / 32;                      // 32-distance mask words
constexpr int64_t kTile = int64_t(kThreads) * kPer;     // 32K tokens
static_assert(kTile % kChunk == 0, "a tile is whole scoring chunks");
constexpr int kTileChunks = int(kTile / kChunk);

__device__ __forceinline__ int64_t clamp_len(int32_t sl, int64_t max_len, int64_t n_cap)
{
    int64_t l = sl < 0 ? 0 : sl;
    l = l < max_len ? l : max_len;
    return l < n_cap ? l : n_cap;
}

// Byte-wise compares of four distances (bytes of w: 0..128 or the pad 255)
// against T (0..128, in every byte of T4), plain integer logic: bit 7 of
// each byte of the result is the answer, the other bits are zero.
//   d < T:  (d | 0x80) - T never borrows across bytes (T <= 128); its bit 7
//           is set iff d >= T when d < 128, and d >= 128 is never below T.
//   d == T: x = d ^ T is zero iff equal; (x & 0x7f) + 0x7f sets bit 7 iff
//           the low seven bits of x are not all zero (no carry out).
__device__ __forceinline__ uint32_t byte_lt_mask(uint32_t w, uint32_t T4)
{
    const uint32_t y = (w | 0x80808080u) - T4;
    return ~(w | y) & 0x80808080u;
}
__device__ __forceinline__ uint32_t byte_eq_mask(uint32_t w, uint32_t T4)
{
    const uint32_t x = w ^ T4;
    const uint32_t t = (x & 0x7f7f7f7fu) + 0x7f7f7f7fu;
    return ~(t | x) & 0x80808080u;
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

// Mask word of 32 distances, bit 8e + w <-> distance 4w + e; the same bits
// in token order (bit 4w + e).  Only words that select something need it.
__device__ __forceinline__ uint32_t to_token_order(uint32_t m)
{
    uint32_t t = 0;
#pragma unroll
    for (int w = 0; w < 8; ++w) {
        // bits w, w+8, w+16, w+24 -> bits 21..24 (the products do not overlap)
        const uint32_t x = (m >> w) & 0x01010101u;
        t |= ((x * 0x00204081u) >> 21 & 0xfu) << (4 * w);
    }
    return t;
}

__global__ void __launch_bounds__(kThreads, 4) select_kernel(SelectArgs a, int parts)
{
    pdl_trigger();
    pdl_wait();  // distances and histograms of the scoring kernel
    const int part = blockIdx.x;
    const size_t bh = blockIdx.y;
    const int b = int(bh / a.H_q);
    const int64_t len = clamp_len(a.seq_len[b], a.max_seq_len, a.n_cap);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int k_eff = int(int64_t(a.topk) < len ? int64_t(a.topk) : len);
    int32_t *idx = a.idx + bh * a.topk;
    const int64_t n_tiles = ceil_div(len, kTile);
    const int64_t t_beg = int64_t(part) * n_tiles / parts;
    const int64_t t_end = int64_t(part + 1) * n_tiles / parts;

    __shared__ int2 scan_s[kWarps + 1];
    __shared__ int64_t red_s[kWarps];
    __shared__ int s_T, s_nless;

    if (part == 0)
        for (int i = k_eff + tid; i < a.topk; i += kThreads) idx[i] = -1;
    if (k_eff <= 0 || t_beg >= t_end) return;

    const uint8_t *drow = a.dist + bh * a.dist_row;
    // this thread's 128 distances of tile t (bytes past the row read as padding)
    uint4 dv[kPieces];
    auto load_tile = [&](int64_t t) {
        const int64_t my0 = t * kTile + int64_t(tid) * kPer;
#pragma unroll
        for (int v = 0; v < kPieces; ++v) {
            const int64_t o = my0 + 16 * v;
            dv[v] = o < a.dist_row ? __ldg(reinterpret_cast<const uint4 *>(drow + o))
                                   : make_uint4(~0u, ~0u, ~0u, ~0u);
        }
    };
    load_tile(t_beg);  // in flight while T and the offsets are found

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

    // ---- keys (< T) and boundary keys (== T) before this part ----
    int64_t less_before = 0, ties_before = 0;
    if (t_beg > 0) {
        const int64_t c0 = t_beg * kTileChunks;
        int64_t lsum = 0, tsum = 0;
        for (int64_t cc = tid; cc < c0; cc += kThreads) {
            const uint32_t *cp = a.cum + (bh * a.n_chunks + cc) * kCumStride;
            const uint32_t le = T > 0 ? __ldg(cp + T - 1) : 0u;
            lsum += le;
            tsum += __ldg(cp + T) - le;
        }
        less_before = block_sum64(lsum, red_s);
        ties_before = block_sum64(tsum, red_s);
    }

    const uint32_t T4 = uint32_t(T) * 0x01010101u;
    for (int64_t t = t_beg; t < t_end; ++t) {
        if (less_before + (ties_before < r_ties ? ties_before : r_ties) >= k_eff) break;
        if (t > t_beg) load_tile(t);
        // ---- masks: group m = pieces 2m, 2m+1 = distances 32m .. 32m+31 ----
        uint32_t lt_bits[kGroups], eq_bits[kGroups];
        int n_lt = 0, n_eq = 0;
#pragma unroll
        for (int m = 0; m < kGroups; ++m) {
            const uint32_t dw[8] = {dv[2 * m].x,     dv[2 * m].y,     dv[2 * m].z,
                                    dv[2 * m].w,     dv[2 * m + 1].x, dv[2 * m + 1].y,
                                    dv[2 * m + 1].z, dv[2 * m + 1].w};
            uint32_t lb = 0, eb = 0;
#pragma unroll
            for (int w = 0; w < 8; ++w) {
                // flag of byte e at bit 8e + 7 -> bit 8e + w
                lb |= byte_lt_mask(dw[w], T4) >> (7 - w);
                eb |= byte_eq_mask(dw[w], T4) >> (7 - w);
            }
            lt_bits[m] = lb;
            eq_bits[m] = eb;
            n_lt += __popc(lb);
            n_eq += __popc(eb);
        }

        int tile_lt, tile_eq;
        const int2 before =
            block_exclusive_scan2<kThreads>(n_lt, n_eq, scan_s, &tile_lt, &tile_eq);
        const int64_t room = r_ties - ties_before > 0 ? r_ties - ties_before : 0;  // ties left
        const int take_tile = int(room < tile_eq ? room : tile_eq);
        const int taken_before = before.y < take_tile ? before.y : take_tile;
        int my_take = take_tile - before.y;
        my_take = my_take < 0 ? 0 : (my_take > n_eq ? n_eq : my_take);

        int64_t pos = less_before + (ties_before < r_ties ? ties_before : r_ties) + before.x +
                      taken_before;
        const int32_t tok0 = int32_t(t * kTile + int64_t(tid) * kPer);
#pragma unroll
        for (int m = 0; m < kGroups; ++m) {
            uint32_t sel = lt_bits[m];
            if (my_take > 0 && eq_bits[m]) {
                const int ne = __popc(eq_bits[m]);
                if (my_take >= ne) {  // every tie of this word
                    sel |= eq_bits[m];
                    my_take -= ne;
                } else {              // the lowest-index my_take ties
                    uint32_t eqt = to_token_order(eq_bits[m]);
                    uint32_t selt = to_token_order(sel);
                    for (; my_take > 0; --my_take) {
                        selt |= eqt & (0u - eqt);
                        eqt &= eqt - 1u;
                    }
                    while (selt) {
                        const int e = __ffs(int(selt)) - 1;
                        selt &= selt - 1u;
                        if (pos < a.topk) idx[pos] = tok0 + 32 * m + e;
                        ++pos;
                    }
                    continue;
                }
            }
            if (sel) {
                uint32_t selt = to_token_order(sel);
                while (selt) {
                    const int e = __ffs(int(selt)) - 1;
                    selt &= selt - 1u;
                    if (pos < a.topk) idx[pos] = tok0 + 32 * m + e;
                    ++pos;
                }
            }
        }
        less_before += tile_lt;
        ties_before += tile_eq;
    }
}

}  // namespace

cudaError_t launch_select(const SelectArgs &a, cudaStream_t s)
{
    int dev = 0, sms = 0, per_sm = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess)
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, select_kernel, kThreads, 0);
    if (e != cudaSuccess) return e;
    // as many parts per head as fill one wave (at least one, at most a tile each)
    const int64_t heads = int64_t(a.B) * a.H_q;
    const int64_t slots = int64_t(per_sm > 0 ? per_sm : 1) * sms;
    const int64_t tiles = ceil_div(a.max_seq_len, kTile);
    int64_t parts = slots / heads;
    parts = parts < 1 ? 1 : (parts > tiles ? tiles : parts);
    const dim3 grid(static_cast<unsigned>(parts), static_cast<unsigned>(heads));
    return launch_pdl(select_kernel, grid, dim3(kThreads), 0, s, a, int(parts));
}

}  // namespace hata
