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
// Grid: (36K-token tile, b * H_q + h_q), 288 threads, each thread owning 128
// consecutive distances (eight 16-byte loads, issued first).  Warp 0 sums
// the head's tile histograms (written by the scoring kernel) while they are
// in flight: the total gives T and r, the tiles before this one the keys
// below T and at T already placed.
// Each thread turns its 128 distances into "< T" and "== T" bit masks with
// byte-wise integer compares, ONE block scan of the two counts gives every
// thread its output position, and the ties a thread may take follow from
// the ties before it: taken_before = min(ties_before, room).  Indices are
// written straight to the head's list, ascending.
#include "block_scan.cuh"
#include "hata_internal.cuh"
#include "tma.cuh"

namespace hata {
namespace {

constexpr int kThreads = 288;  // 9 warps x 128 distances = one tile
constexpr int kWarps = kThreads / 32;
constexpr int kPer = 128;                               // distances per thread
constexpr int kPieces = kPer / 16;                      // 16-byte loads per thread
constexpr int kGroups = kPer / 32;                      // 32-distance mask words
static_assert(kThreads * kPer == kTile, "a CTA covers one histogram tile per pass");

__device__ __forceinline__ int64_t clamp_len(int32_t sl, int64_t max_len, int64_t n_cap)
{
    int64_t l = sl < 0 ? 0 : sl;
    l = l < max_len ? l : max_len;
    return l < n_cap ? l : n_cap;
}

// Byte-wise zero test of four distances (bytes of w: 0..128 or the pad
// 255) against T4 (one value in every byte), plain integer logic: bit 7 of
// each byte of the result is set iff the byte equals T; the other bits are
// zero.  x = d ^ T is zero iff equal; (x & 0x7f) + 0x7f sets bit 7 iff the
// low seven bits of x are not all zero (no carry out).
__device__ __forceinline__ uint32_t byte_eq_mask(uint32_t w, uint32_t T4)
{
    const uint32_t x = w ^ T4;
    const uint32_t t = (x & 0x7f7f7f7fu) + 0x7f7f7f7fu;
    return ~(t | x) & 0x80808080u;
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

// T = the smallest distance t with #(dist <= t) >= k_eff, #(dist < T), and
// the keys below T and at T in the tiles before `tile`, from head bh's tile
// histograms.  One warp; lane l owns bins 5l .. 5l+4; out: {T, #(< T),
// below-T before the tile, at-T before the tile}.
__device__ __forceinline__ void head_threshold(const SelectArgs &a, size_t bh, int k_eff, int tile,
                                               int lane, int *out)
{
    constexpr int kRegTiles = 4;  // rows held in registers per round
    const uint32_t *hrow = a.hist + bh * size_t(a.n_tiles) * kHistStride;
    const int n_tiles = int(a.n_tiles);
    auto row_bins = [&](int t, uint32_t (&v)[5]) {
#pragma unroll
        for (int e = 0; e < 5; ++e)
            v[e] = lane * 5 + e < kBins ? __ldg(hrow + t * kHistStride + lane * 5 + e) : 0u;
    };
    uint32_t tot[5] = {0u, 0u, 0u, 0u, 0u}, pre[5] = {0u, 0u, 0u, 0u, 0u};
    // rounds of kRegTiles rows: all loads of a round are issued before any
    // is summed, so a round costs one round trip to L2
    for (int t0 = 0; t0 < n_tiles; t0 += kRegTiles) {
        uint32_t rv[kRegTiles][5];
#pragma unroll
        for (int t = 0; t < kRegTiles; ++t) {
            if (t0 + t < n_tiles) {
                row_bins(t0 + t, rv[t]);
            } else {
#pragma unroll
                for (int e = 0; e < 5; ++e) rv[t][e] = 0u;
            }
        }
#pragma unroll
        for (int t = 0; t < kRegTiles; ++t)
#pragma unroll
            for (int e = 0; e < 5; ++e) {
                tot[e] += rv[t][e];
                pre[e] += t0 + t < tile ? rv[t][e] : 0u;
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
    // cumulative counts are monotone: the lowest lane that found a bin holds T
    const unsigned found = __ballot_sync(0xffffffffu, Tl >= 0);
    const int src = found ? __ffs(int(found)) - 1 : 0;
    const int T = found ? __shfl_sync(0xffffffffu, Tl, src) : 128;  // unreachable fallback
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
        out[0] = T;
        out[1] = n_less;
        out[2] = l;
        out[3] = q;
    }
}

__global__ void __launch_bounds__(kThreads, 4) select_kernel(SelectArgs a)
{
    pdl_trigger();
    const int tile = blockIdx.x;
    const size_t bh = blockIdx.y;
    const int b = int(bh) / a.H_q;
    const int len = int(clamp_len(__ldg(a.seq_len + b), a.max_seq_len, a.n_cap));  // step input
    const int tid = threadIdx.x;
    const int k_eff = a.topk < len ? a.topk : len;
    pdl_wait();  // distances and tile histograms of the scoring kernel
    int32_t *idx = a.idx + bh * a.topk;

    __shared__ int2 scan_s[kWarps + 1];
    __shared__ int s_thr[4];
    __shared__ __align__(16) uint8_t dist_s[kThreads * kPer];  // the tile's distances

    if (tile == 0)
        for (int i = k_eff + tid; i < a.topk; i += kThreads) idx[i] = -1;
    if (k_eff <= 0 || tile * kTile >= len) return;

    // this thread's 128 distances (bytes past the row read as padding)
    const uint8_t *drow = a.dist + bh * a.dist_row;
    const int my0 = tile * kTile + tid * kPer;
    // ---- warp 0 first finds T, #(dist < T) and the keys below T / at T in
    // the tiles before this one from the head's tile histograms (one round
    // trip to L2 per 4 tiles), ahead of its own distance loads;
    // the other warps' distance loads are in flight meanwhile ----
    if (tid < 32) head_threshold(a, bh, k_eff, tile, tid, s_thr);
    // the warp's 4 KB arrive by coalesced 16-byte copies (lane l: bytes
    // 16l .. 16l+15 of each 512-byte block) into a swizzled shared tile,
    // piece v of thread t at t*128 + 16*(v ^ (t & 7)), so that each thread
    // then reads its own 128 bytes without bank conflicts
    const uint32_t sbase = smem_addr(dist_s);
    const int wbase = (tid >> 5) * 32 * kPer;  // this warp's first byte in the tile
#pragma unroll
    for (int k = 0; k < kPieces; ++k) {
        const int byte = wbase + k * 512 + (tid & 31) * 16;
        const int t = byte >> 7, v = (byte >> 4) & 7;
        const int64_t g = int64_t(tile) * kTile + byte;
        const bool in = g < a.dist_row;  // past the row: no read (padding below)
        cp_async16_zfill(sbase + uint32_t(t * kPer + 16 * (v ^ (t & 7))), in ? drow + g : drow,
                         in ? 16u : 0u);
    }
    cp_async_commit();
    cp_async_wait<0>();
    __syncwarp();
    uint4 dv[kPieces];
#pragma unroll
    for (int v = 0; v < kPieces; ++v)
        dv[v] = my0 + 16 * v < a.dist_row
                    ? *reinterpret_cast<const uint4 *>(dist_s + tid * kPer + 16 * (v ^ (tid & 7)))
                    : make_uint4(~0u, ~0u, ~0u, ~0u);
    __syncthreads();
    const int T = s_thr[0], n_less = s_thr[1], lp = s_thr[2], tp = s_thr[3];
    const int r_ties = k_eff - n_less;  // boundary keys taken over the whole head
    const int less_before = lp, ties_before = tp;
    if (less_before + (ties_before < r_ties ? ties_before : r_ties) >= k_eff)
        return;  // every key of the head is placed before this tile (CTA-uniform)

    // ---- masks: group m = pieces 2m, 2m+1 = distances 32m .. 32m+31 ----
    // "< T" and "<= T" from one (d | 0x80) per byte: (d | 0x80) - t never
    // borrows for t <= 128, so only T = 128 (where "<= T" means "not the pad
    // 255") needs the zero-byte test.  Ties = "<= T" and not "< T".  Flags
    // move into the packed word with a multiply-high and an add (a right
    // shift of the word so far; the bits never overlap).
    const uint32_t T4 = uint32_t(T) * 0x01010101u, T4p = T4 + 0x01010101u;
    uint32_t lt_bits[kGroups], eq_bits[kGroups];
    int n_lt = 0, n_eq = 0;
#pragma unroll
    for (int m = 0; m < kGroups; ++m) {
        const uint32_t dw[8] = {dv[2 * m].x,     dv[2 * m].y,     dv[2 * m].z,     dv[2 * m].w,
                                dv[2 * m + 1].x, dv[2 * m + 1].y, dv[2 * m + 1].z, dv[2 * m + 1].w};
        uint32_t lb = 0, le = 0;
#pragma unroll
        for (int w = 0; w < 8; ++w) {
            const uint32_t wh = dw[w] | 0x80808080u;
            const uint32_t lt = ~(dw[w] | (wh - T4)) & 0x80808080u;
            const uint32_t lq = T < 128 ? ~(dw[w] | (wh - T4p)) & 0x80808080u
                                        : ~byte_eq_mask(dw[w], 0xffffffffu) & 0x80808080u;
            // flag of byte e: bit 8e + 7 of word w -> bit 8e + w of the group
            lb = __umulhi(lb, 0x80000000u) + lt;
            le = __umulhi(le, 0x80000000u) + lq;
        }
        lt_bits[m] = lb;
        eq_bits[m] = le & ~lb;
        n_lt += __popc(lb);
        n_eq += __popc(eq_bits[m]);
    }

    int tile_lt, tile_eq;
    const int2 before = block_exclusive_scan2<kThreads>(n_lt, n_eq, scan_s, &tile_lt, &tile_eq);
    const int room = r_ties - ties_before > 0 ? r_ties - ties_before : 0;  // ties left
    const int take_tile = room < tile_eq ? room : tile_eq;
    const int taken_before = before.y < take_tile ? before.y : take_tile;
    int my_take = take_tile - before.y;
    my_take = my_take < 0 ? 0 : (my_take > n_eq ? n_eq : my_take);

    int pos = less_before + (ties_before < r_ties ? ties_before : r_ties) + before.x + taken_before;
#pragma unroll
    for (int m = 0; m < kGroups; ++m) {
        uint32_t sel = lt_bits[m];
        if (my_take > 0 && eq_bits[m]) {
            const int ne = __popc(eq_bits[m]);
            if (my_take >= ne) {  // every tie of this word
                sel |= eq_bits[m];
                my_take -= ne;
            } else {              // the lowest-index my_take ties
                uint32_t eqt = to_token_order(eq_bits[m]), kept = 0u;
                for (; my_take > 0; --my_take) {
                    kept |= eqt & (0u - eqt);
                    eqt &= eqt - 1u;
                }
                uint32_t selt = to_token_order(sel) | kept;
                while (selt) {
                    const int e = __ffs(int(selt)) - 1;
                    selt &= selt - 1u;
                    if (pos < a.topk) idx[pos] = my0 + 32 * m + e;
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
                if (pos < a.topk) idx[pos] = my0 + 32 * m + e;
                ++pos;
            }
        }
    }
}

}  // namespace

cudaError_t launch_select(const SelectArgs &a, cudaStream_t s)
{
    if (cudaError_t e = ensure_smem_attr(reinterpret_cast<const void *>(select_kernel), 0))
        return e;
    // one CTA per (36K-token tile, head)
    const dim3 grid(static_cast<unsigned>(ceil_div(a.max_seq_len, kTile)),
                    static_cast<unsigned>(int64_t(a.B) * a.H_q));
    return launch_pdl(select_kernel, grid, dim3(kThreads), 0, s, a);
}

}  // namespace hata
