// select_common.cuh -- the pieces of the histogram top-k of the selection
// kernel (one CTA per 36K-token tile of a head): the threshold from the tile
// histograms, the byte-wise masks and the ordered emission.
//
// HATA review page (arXiv 2506.02572), major comment 1 (Algorithm 3): the
// top-k runs over Hamming scores that take only r + 1 values (129 at the
// page's r = 128); the boundary bucket goes to the lower token indices:
//   k_eff = min(topk, len)
//   T     = the smallest distance t with #(dist <= t) >= k_eff
//   S     = {n : dist[n] < T}  +  the k_eff - #(dist < T) lowest-index keys
//           with dist[n] == T.
#pragma once

#include "block_scan.cuh"
#include "hata_internal.cuh"

namespace hata {

// Byte-wise equality test of four distances (any byte values) against T4
// (one value in every byte), plain integer logic: bit 7 of
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

// "< T" and "== T" masks of 32 consecutive distances (words dw[0..7], byte e
// of word w = distance 4w + e), bit 8e + w of each mask.  "< T" and "<= T"
// come from one (d | 0x80) per byte: (d | 0x80) - t never borrows for
// t <= 128, so only T = 128 (where "<= T" means "not the pad 255") needs the
// zero-byte test.  The flags move into the packed word with a multiply-high
// and an add (a right shift of the word so far; the bits never overlap).
template <bool kT128>
__device__ __forceinline__ void group_masks(const uint32_t (&dw)[8], uint32_t T4, uint32_t T4p,
                                            uint32_t &lt_out, uint32_t &eq_out)
{
    uint32_t lb = 0, le = 0;
#pragma unroll
    for (int w = 0; w < 8; ++w) {
        const uint32_t wh = dw[w] | 0x80808080u;
        const uint32_t lt = ~(dw[w] | (wh - T4)) & 0x80808080u;
        const uint32_t lq = kT128 ? ~byte_eq_mask(dw[w], 0xffffffffu) & 0x80808080u
                                  : ~(dw[w] | (wh - T4p)) & 0x80808080u;
        // flag of byte e: bit 8e + 7 of word w -> bit 8e + w of the group
        lb = __umulhi(lb, 0x80000000u) + lt;
        le = __umulhi(le, 0x80000000u) + lq;
    }
    lt_out = lb;
    eq_out = le & ~lb;
}

// "< T" and "== T" masks of 32 consecutive distances for any T in 0..255
// (the 256-bit codes, whose stored distances run 0..255), packed like
// group_masks.  Per byte, unsigned x < T: t = (x | 0x80) - (T & 0x7f) never
// borrows across bytes and its bit 7 says "low seven bits of x >= those of
// T", so x < T iff (x7 < T7) or (x7 == T7 and not that):
// ((~x & T) | (~(x ^ T) & ~t)) & 0x80 -- plain integer logic (the SIMD
// byte-compare intrinsics are emulated at many instructions each).
__device__ __forceinline__ void group_masks_any(const uint32_t (&dw)[8], uint32_t T4,
                                                uint32_t &lt_out, uint32_t &eq_out)
{
    const uint32_t tlow = T4 & 0x7f7f7f7fu;
    uint32_t lb = 0, lq = 0;
#pragma unroll
    for (int w = 0; w < 8; ++w) {
        const uint32_t x = dw[w];
        const uint32_t t = (x | 0x80808080u) - tlow;
        const uint32_t lt = ((~x & T4) | (~(x ^ T4) & ~t)) & 0x80808080u;
        lb = __umulhi(lb, 0x80000000u) + lt;
        lq = __umulhi(lq, 0x80000000u) + byte_eq_mask(x, T4);
    }
    lt_out = lb;
    eq_out = lq;
}

// T = the smallest distance t with #(dist <= t) >= k_eff, #(dist < T), and
// the keys below T and at T in the tiles before `tile`, from one head's
// tile histograms (hrow: n_tiles rows of kHistStride words, or of
// kHistStrideWide words for the 257 bins of 256-bit codes).  One warp; lane
// l owns bins kBPL l .. kBPL l + kBPL - 1; out: {T, #(< T), below-T before
// the tile, at-T before the tile}.  kCoherent: the rows were written by the
// running kernel itself (loads through L2 only); otherwise by an earlier
// kernel.
template <bool kCoherent = false, int kRegTiles = 4, bool kWide = false>
__device__ __forceinline__ void head_threshold(const uint32_t *hrow, int n_tiles, int k_eff,
                                               int tile, int lane, int *out)
{
    constexpr int kBPL = kWide ? 9 : 5;  // bins per lane: 32 lanes cover 257 / 129 bins
    constexpr int kNB = kWide ? kBinsWide : kBins;
    constexpr int kStride = kWide ? kHistStrideWide : kHistStride;
    auto row_bins = [&](int t, uint32_t (&v)[kBPL]) {
#pragma unroll
        for (int e = 0; e < kBPL; ++e)
            v[e] = lane * kBPL + e < kNB
                       ? (kCoherent ? __ldcg(hrow + t * kStride + lane * kBPL + e)
                                    : __ldg(hrow + t * kStride + lane * kBPL + e))
                       : 0u;
    };
    uint32_t tot[kBPL], pre[kBPL];
#pragma unroll
    for (int e = 0; e < kBPL; ++e) tot[e] = pre[e] = 0u;
    // rounds of kRegTiles rows: all loads of a round are issued before any
    // is summed, so a round costs one round trip to L2
    for (int t0 = 0; t0 < n_tiles; t0 += kRegTiles) {
        uint32_t rv[kRegTiles][kBPL];
#pragma unroll
        for (int t = 0; t < kRegTiles; ++t) {
            if (t0 + t < n_tiles) {
                row_bins(t0 + t, rv[t]);
            } else {
#pragma unroll
                for (int e = 0; e < kBPL; ++e) rv[t][e] = 0u;
            }
        }
#pragma unroll
        for (int t = 0; t < kRegTiles; ++t)
#pragma unroll
            for (int e = 0; e < kBPL; ++e) {
                tot[e] += rv[t][e];
                pre[e] += t0 + t < tile ? rv[t][e] : 0u;
            }
    }
    uint32_t run = 0;
#pragma unroll
    for (int e = 0; e < kBPL; ++e) run += tot[e];
    uint32_t acc = uint32_t(warp_inclusive_scan(int(run))) - run;
    int Tl = -1;
    uint32_t less_l = 0;
#pragma unroll
    for (int e = 0; e < kBPL; ++e) {
        if (Tl < 0 && lane * kBPL + e < kNB && acc + tot[e] >= uint32_t(k_eff)) {
            Tl = lane * kBPL + e;
            less_l = acc;
        }
        acc += tot[e];
    }
    // cumulative counts are monotone: the lowest lane that found a bin holds T
    const unsigned found = __ballot_sync(0xffffffffu, Tl >= 0);
    const int src = found ? __ffs(int(found)) - 1 : 0;
    const int T = found ? __shfl_sync(0xffffffffu, Tl, src) : kNB - 1;  // unreachable fallback
    const int n_less = found ? __shfl_sync(0xffffffffu, int(less_l), src) : 0;
    int l = 0, q = 0;
#pragma unroll
    for (int e = 0; e < kBPL; ++e) {
        const int bin = lane * kBPL + e;
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

// Partial sums of one head's tile histograms (hrow: n_tiles rows of
// kHistStride words) over the tiles first, first + step, ...: tot = all of
// them, pre = those before `tile`.  Lane l: bins 5l .. 5l+4.  The loads of
// up to 4 tiles are issued before any is summed.
__device__ __forceinline__ void tile_sums(const uint32_t *hrow, int n_tiles, int first, int step,
                                          int tile, int lane, uint32_t (&tot)[5],
                                          uint32_t (&pre)[5])
{
#pragma unroll
    for (int e = 0; e < 5; ++e) tot[e] = pre[e] = 0u;
    for (int t0 = first; t0 < n_tiles; t0 += 4 * step) {
        uint32_t rv[4][5];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const int t = t0 + r * step;
#pragma unroll
            for (int e = 0; e < 5; ++e)
                rv[r][e] = t < n_tiles && lane * 5 + e < kBins
                               ? __ldg(hrow + t * kHistStride + lane * 5 + e)
                               : 0u;
        }
#pragma unroll
        for (int r = 0; r < 4; ++r)
#pragma unroll
            for (int e = 0; e < 5; ++e) {
                tot[e] += rv[r][e];
                pre[e] += t0 + r * step < tile ? rv[r][e] : 0u;
            }
    }
}

// head_threshold's second half: T, #(< T), and the keys below / at T in
// the tiles before this one, from the summed bins (lane l: bins 5l ..
// 5l+4); one warp; out as head_threshold's.
__device__ __forceinline__ void threshold_from_sums(const uint32_t (&tot)[5],
                                                    const uint32_t (&pre)[5], int k_eff, int lane,
                                                    int *out)
{
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
    const int T = found ? __shfl_sync(0xffffffffu, Tl, src) : kBins - 1;  // unreachable fallback
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

// Store the tokens of the set bits of sel (bit 8e + w <-> token tok + 4w + e)
// at positions pos + (their rank in token order), without transposing the
// word: the rank of a bit is the number of set bits of lower tokens (lower w,
// or the same w and lower e).
template <class Put>
__device__ __forceinline__ void put_ranked(uint32_t sel, int pos, int tok, Put &put)
{
    uint32_t rest = sel;
    while (rest) {
        const int bit = __ffs(int(rest)) - 1;
        rest &= rest - 1u;
        const int w = bit & 7, e = bit >> 3;
        const uint32_t lower =
            ((1u << w) - 1u) * 0x01010101u | ((0x01010101u << w) & ((1u << (8 * e)) - 1u));
        put(pos + __popc(sel & lower), tok + 4 * w + e);
    }
}

// Emit a thread's selected tokens in ascending order: group m (tokens
// tok0 + 32 m ...) selects every "< T" key and, while my_take lasts, its
// ties at T from the lowest index up.  put(pos, token) stores one entry;
// positions run on from pos.
template <int kGroupsN, class Put>
__device__ __forceinline__ void emit_selected(const uint32_t (&lt_bits)[kGroupsN],
                                              const uint32_t (&eq_bits)[kGroupsN], int my_take,
                                              int pos, int tok0, Put &&put)
{
#pragma unroll
    for (int m = 0; m < kGroupsN; ++m) {
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
                    put(pos++, tok0 + 32 * m + e);
                }
                continue;
            }
        }
        if (sel) {
            put_ranked(sel, pos, tok0 + 32 * m, put);
            pos += __popc(sel);
        }
    }
}

}  // namespace hata
