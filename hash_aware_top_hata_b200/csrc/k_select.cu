// k_select.cu -- top-k selection over the Hamming distances, no sort.
//
// HATA review page (arXiv 2506.02572), major comment 1 (Algorithm 3): the
// top-k runs over Hamming scores that take only r + 1 values, so the boundary
// usually falls inside a large bucket of equal scores; the page leaves the
// choice inside that bucket open.  Here it goes to the lower token index, so
// the selected set is unique:
//   k_eff = min(topk, len)
//   T     = the smallest distance t with #(dist <= t) >= k_eff
//   S     = {n : dist[n] < T}  +  the r = k_eff - #(dist < T) lowest-index
//           keys with dist[n] == T.
//
// Grid: (36K-token tile, b * H_q + h_q), 288 threads, each thread owning 128
// consecutive distances (eight 16-byte loads, issued first).  The head's
// tile histograms (written by the scoring kernel) are summed while those
// loads are in flight -- by warp 0 for up to 4 tiles, by every warp for a
// share of more (one round trip to L2 either way): the total gives T and
// r, the tiles before this one the keys below T and at T already placed.
// Each thread turns its 128 distances into "< T" and "== T" bit masks with
// byte-wise integer compares, ONE block scan of the two counts gives every
// thread its output position, and the ties a thread may take follow from
// the ties before it: taken_before = min(ties_before, room).  Indices are
// written straight to the head's list, ascending.
//
// 256-bit codes: the stored distance saturates at 255 (distances run to
// 256), the tile histograms hold all 257 bins.  With T <= 254 the byte
// compares stay exact (a stored 255 is above T); the rare T of 255 or 256
// takes the exact distance of every saturated key from the codes.
//
// The sequence-parallel step passes k_head: the keys each head takes from
// this shard, which makes the shard's selection its own top-k_head with the
// same tie rule.
#include "select_common.cuh"
#include "async_copy.cuh"

namespace hata {
namespace {

constexpr int kThreads = 288;  // 9 warps x 128 distances = one tile
constexpr int kWarps = kThreads / 32;
constexpr int kPer = 128;                               // distances per thread
constexpr int kPieces = kPer / 16;                      // 16-byte loads per thread
constexpr int kGroups = kPer / 32;                      // 32-distance mask words
static_assert(kThreads * kPer == kTile, "a CTA covers one histogram tile per pass");

// Exact distance of key `tok` of head bh's KV slab to the head's 256-bit
// query code (q: its two 16-byte halves).
__device__ __forceinline__ int exact_dist_wide(const SelectArgs &a, size_t bh, const uint4 (&q)[2],
                                               int tok)
{
    const int b = int(bh) / a.H_q, h = (int(bh) - b * a.H_q) / a.G;
    const uint4 *c = reinterpret_cast<const uint4 *>(a.codes) +
                     ((int64_t(b) * a.H_kv + h) * a.n_cap + tok) * 2;
    int d = 0;
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
        const uint4 k = __ldg(c + hf);
        d += __popc(k.x ^ q[hf].x) + __popc(k.y ^ q[hf].y) + __popc(k.z ^ q[hf].z) +
             __popc(k.w ^ q[hf].w);
    }
    return d;
}

template <bool kWide>
__global__ void __launch_bounds__(kThreads, kWide ? 2 : 4) select_kernel(SelectArgs a)
{
    pdl_trigger();
    const int tile = blockIdx.x;
    const size_t bh = blockIdx.y;
    const int b = int(bh) / a.H_q;
    const int len = int(clamp_len(__ldg(a.seq_len + b), a.max_seq_len, a.n_cap));  // step input
    const int tid = threadIdx.x;
    int k_eff = a.topk < len ? a.topk : len;
    pdl_wait();  // distances and tile histograms of the scoring kernel
    if (a.k_head) {  // written by the kernel before this one
        const int kh = __ldg(a.k_head + bh);
        k_eff = kh < k_eff ? (kh > 0 ? kh : 0) : k_eff;
    }
    constexpr int kStride = kWide ? kHistStrideWide : kHistStride;
    int32_t *idx = a.idx + bh * a.topk;

    __shared__ int2 scan_s[kWarps + 1];
    __shared__ int s_thr[4];
    __shared__ __align__(16) uint8_t dist_s[kThreads * kPer];  // the tile's distances
    __shared__ uint32_t hsum[kWarps][2][160];                   // per-warp bin sums (many tiles)

    if (tile == 0)
        for (int i = k_eff + tid; i < a.topk; i += kThreads) idx[i] = -1;
    if (k_eff <= 0 || tile * kTile >= len) return;

    // this thread's 128 distances (bytes past the row read as padding)
    const uint8_t *drow = a.dist + bh * a.dist_row;
    const int my0 = tile * kTile + tid * kPer;
    // ---- T, #(dist < T) and the keys below T / at T in the tiles before
    // this one, from the head's tile histograms.  Up to 4 tiles: warp 0, one
    // round trip to L2, ahead of its own distance loads; more tiles: every
    // warp sums its share of them (one round trip for up to 36 tiles) while
    // the distance copies are in flight, and warp 0 adds the shares ----
    const uint32_t *hrow = a.hist + bh * size_t(a.n_tiles) * kStride;
    const bool many = !kWide && a.n_tiles > 4;  // CTA-uniform
    if (!many && tid < 32)
        head_threshold<false, 4, kWide>(hrow, int(a.n_tiles), k_eff, tile, tid, s_thr);
    // the warp's 4 KB arrive by coalesced 16-byte copies (lane l: bytes
    // 16l .. 16l+15 of each 512-byte block) into a swizzled shared tile,
    // piece v of thread t at t*128 + 16*(v ^ (t & 7)), so that each thread
    // then reads its own 128 bytes without bank conflicts
    const uint32_t sbase = smem_addr(dist_s);
    const int lane = tid & 31, wbase = (tid >> 5) * 32 * kPer;  // the warp's first byte
    const bool full = int64_t(tile + 1) * kTile <= a.dist_row;    // CTA-uniform
    uint4 dv[kPieces];
    if (full) {
        // copy k: byte wbase + 512 k + 16 lane = thread t = wbase/128 + 4k + lane/8, piece
        // lane & 7; t & 7 = lane/8 + 4 (k & 1), so odd copies flip address bit 6
        const uint8_t *src = drow + int64_t(tile) * kTile + wbase + 16 * lane;
        const uint32_t o0 = uint32_t(wbase + 128 * (lane >> 3) + 16 * ((lane & 7) ^ (lane >> 3)));
        const uint32_t d0 = sbase + o0, d1 = sbase + (o0 ^ 64u);
#pragma unroll
        for (int k = 0; k < kPieces; ++k)
            cp_async16_zfill((k & 1 ? d1 : d0) + 512u * k, src + 512 * k, 16u);
    } else {  // the row's last tile: pieces past the row read as padding
#pragma unroll
        for (int k = 0; k < kPieces; ++k) {
            const int byte = wbase + k * 512 + lane * 16;
            const int t = byte >> 7, v = (byte >> 4) & 7;
            const int64_t g = int64_t(tile) * kTile + byte;
            const bool in = g < a.dist_row;
            cp_async16_zfill(sbase + uint32_t(t * kPer + 16 * (v ^ (t & 7))), in ? drow + g : drow,
                             in ? 16u : 0u);
        }
    }
    cp_async_commit();
    if (many) {
        const int warp = tid >> 5;
        uint32_t tot[5], pre[5];
        tile_sums(hrow, int(a.n_tiles), warp, kWarps, tile, lane, tot, pre);
#pragma unroll
        for (int e = 0; e < 5; ++e) {
            hsum[warp][0][lane * 5 + e] = tot[e];
            hsum[warp][1][lane * 5 + e] = pre[e];
        }
        __syncthreads();
        if (warp == 0) {
#pragma unroll
            for (int e = 0; e < 5; ++e) {
                uint32_t t = 0u, p = 0u;
#pragma unroll
                for (int w = 0; w < kWarps; ++w) {
                    t += hsum[w][0][lane * 5 + e];
                    p += hsum[w][1][lane * 5 + e];
                }
                tot[e] = t;
                pre[e] = p;
            }
            threshold_from_sums(tot, pre, k_eff, lane, s_thr);
        }
    }
    cp_async_wait<0>();
    __syncwarp();
    if (full) {
        const uint8_t *mine = dist_s + tid * kPer;
#pragma unroll
        for (int v = 0; v < kPieces; ++v)
            dv[v] = *reinterpret_cast<const uint4 *>(mine + 16 * (v ^ (tid & 7)));
    } else {
#pragma unroll
        for (int v = 0; v < kPieces; ++v)
            dv[v] = my0 + 16 * v < a.dist_row
                        ? *reinterpret_cast<const uint4 *>(dist_s + tid * kPer + 16 * (v ^ (tid & 7)))
                        : make_uint4(~0u, ~0u, ~0u, ~0u);
    }
    __syncthreads();
    const int T = s_thr[0], n_less = s_thr[1], lp = s_thr[2], tp = s_thr[3];
    const int r_ties = k_eff - n_less;  // boundary keys taken over the whole head
    const int less_before = lp, ties_before = tp;
    if (less_before + (ties_before < r_ties ? ties_before : r_ties) >= k_eff)
        return;  // every key of the head is placed before this tile (CTA-uniform)

    // ---- masks: group m = pieces 2m, 2m+1 = distances 32m .. 32m+31 ----
    const uint32_t T4 = uint32_t(T) * 0x01010101u, T4p = T4 + 0x01010101u;
    uint32_t lt_bits[kGroups], eq_bits[kGroups];
    int n_lt = 0, n_eq = 0;
    if (kWide && T >= 255) {
        // the boundary reached the saturated byte: exact distances of the
        // saturated keys (bit 8e + w of group m <-> distance 32 m + 4 w + e;
        // keys at or past len never count)
        uint4 q[2];
        q[0] = __ldg(reinterpret_cast<const uint4 *>(a.qcodes) + bh * 2);
        q[1] = __ldg(reinterpret_cast<const uint4 *>(a.qcodes) + bh * 2 + 1);
        const uint8_t *mine = dist_s + tid * kPer;
#pragma unroll
        for (int m = 0; m < kGroups; ++m) {
            uint32_t lt = 0u, eq = 0u;
            for (int j = 0; j < 32; ++j) {
                const int o = 32 * m + j, tok = my0 + o;
                int d = 1 << 20;  // past len: never selected
                if (tok < len) {
                    d = mine[16 * ((o >> 4) ^ (tid & 7)) + (o & 15)];
                    if (d == 255) d = exact_dist_wide(a, bh, q, tok);
                }
                const uint32_t bit = 1u << (8 * (j & 3) + (j >> 2));
                lt |= d < T ? bit : 0u;
                eq |= d == T ? bit : 0u;
            }
            lt_bits[m] = lt;
            eq_bits[m] = eq;
            n_lt += __popc(lt);
            n_eq += __popc(eq);
        }
    } else {
#pragma unroll
        for (int m = 0; m < kGroups; ++m) {
            const uint32_t dw[8] = {dv[2 * m].x,     dv[2 * m].y,     dv[2 * m].z,
                                    dv[2 * m].w,     dv[2 * m + 1].x, dv[2 * m + 1].y,
                                    dv[2 * m + 1].z, dv[2 * m + 1].w};
            if (kWide)
                group_masks_any(dw, T4, lt_bits[m], eq_bits[m]);
            else if (T < 128)
                group_masks<false>(dw, T4, T4p, lt_bits[m], eq_bits[m]);
            else
                group_masks<true>(dw, T4, T4p, lt_bits[m], eq_bits[m]);
            n_lt += __popc(lt_bits[m]);
            n_eq += __popc(eq_bits[m]);
        }
    }

    int tile_lt, tile_eq;
    const int2 before = block_exclusive_scan2<kThreads>(n_lt, n_eq, scan_s, &tile_lt, &tile_eq);
    const int room = r_ties - ties_before > 0 ? r_ties - ties_before : 0;  // ties left
    const int take_tile = room < tile_eq ? room : tile_eq;
    const int taken_before = before.y < take_tile ? before.y : take_tile;
    int my_take = take_tile - before.y;
    my_take = my_take < 0 ? 0 : (my_take > n_eq ? n_eq : my_take);

    const int pos =
        less_before + (ties_before < r_ties ? ties_before : r_ties) + before.x + taken_before;
    emit_selected(lt_bits, eq_bits, my_take, pos, my0, [&](int p, int tok) {
        if (p < a.topk) idx[p] = tok;
    });
}

}  // namespace

cudaError_t launch_select(const SelectArgs &a, cudaStream_t s)
{
    auto kernel = a.words == 8 ? select_kernel<true> : select_kernel<false>;
    if (cudaError_t e = ensure_smem_attr(reinterpret_cast<const void *>(kernel), 0)) return e;
    // one CTA per (36K-token tile, head)
    const dim3 grid(static_cast<unsigned>(ceil_div(a.max_seq_len, kTile)),
                    static_cast<unsigned>(int64_t(a.B) * a.H_q));
    return launch_pdl(kernel, grid, dim3(kThreads), 0, s, a);
}

}  // namespace hata
