// score_common.cuh -- the Hamming distance of a query code to a key code,
// shared by the scoring kernels.
//
// HATA review page (arXiv 2506.02572), "What carries the argument": the
// query code is XOR-ed with a cached key code and a population count gives
// the Hamming score.
#pragma once

#include <stdint.h>

namespace hata {

// dist(k, q) for 128-bit codes, summed bit position by bit position from
// the XOR-ed words x_w = k_w ^ q_w taken in pairs: x0 + x1 = u + 2a and
// x2 + x3 = v + 2b (u = x0 ^ x1, v = x2 ^ x3, a = x0 & x1, b = x2 & x3), so
//   x0 + x1 + x2 + x3 = (u ^ v) + 2 (a + b + (u & v))
// where a and u & v never both hold: c = a | (u & v) = (u ? v : x0), and
// b = x2 & ~v.  dist = popc(u ^ v) + 2 (popc(c) + popc(e = b)): three
// population counts instead of four, and six three-input logic operations,
// since u and v reach the key through k0 ^ k1 and k2 ^ k3 (k01, k23, shared
// by every query head scored against the key) and the query through
// q0 ^ q1 and q2 ^ q3 (qp).
__device__ __forceinline__ int hamming128(const uint4 &k, uint32_t k01, uint32_t k23,
                                          const uint4 &q, const uint2 &qp)
{
    const uint32_t u = k01 ^ qp.x, v = k23 ^ qp.y;
    const uint32_t c = (u & v) | (~u & (k.x ^ q.x));
    const uint32_t e = (k.z ^ q.z) & ~v;
    return __popc(u ^ v) + 2 * (__popc(c) + __popc(e));
}

// dist(k, q) for codes of W words (r = 32 W bits): the carry-save form
// above for W = 4 (kp = its k01, k23), plain population counts of the
// XOR-ed words otherwise.
template <int W>
__device__ __forceinline__ int hamming_w(const uint4 &k, const uint2 &kp, const uint4 &q,
                                         const uint2 &qp)
{
    if constexpr (W == 4) return hamming128(k, kp.x, kp.y, q, qp);
    if constexpr (W == 2) return __popc(k.x ^ q.x) + __popc(k.y ^ q.y);
    return __popc(k.x ^ q.x);
}

}  // namespace hata
