// score_common.cuh -- the Hamming distance of a query code to a key code,
// shared by the scoring kernels.
//
// HATA review page (arXiv 2506.02572), "What carries the argument": the
// query code is XOR-ed with a cached key code and a population count gives
// the Hamming score.
#pragma once

#include <stdint.h>

namespace hata {

// dist(k, q) with the XOR-ed words x_w = k_w ^ q_w, summed bit position by
// bit position with a full adder and a half adder:
//   x0 + x1 + x2 = s + 2c,  s = x0 ^ x1 ^ x2,  c = maj(x0, x1, x2)
//   s + x3       = o + 2e,  o = s ^ x3,        e = s & x3
// so dist = popc(o) + 2 (popc(c) + popc(e)).  s and o depend on the key only
// through k0 ^ k1 ^ k2 and k0 ^ k1 ^ k2 ^ k3 (k012, k0123, shared by every
// head of the group) and on the query through q012, q0123 (qd).
__device__ __forceinline__ int hamming128(const uint4 &k, uint32_t k012, uint32_t k0123,
                                          const uint4 &q, const uint2 &qd)
{
    const uint32_t x0 = k.x ^ q.x, x1 = k.y ^ q.y, x2 = k.z ^ q.z;
    const uint32_t c = (x0 & x1) | (x2 & (x0 ^ x1));
    const uint32_t o = k0123 ^ qd.y;
    const uint32_t e = (k012 ^ qd.x) & (k.w ^ q.w);
    return __popc(o) + 2 * (__popc(c) + __popc(e));
}

// The same distance from the pair sums x0 + x1 = u + 2a and x2 + x3 = v + 2b
// (u = x0 ^ x1, v = x2 ^ x3, a = x0 & x1, b = x2 & x3):
//   x0 + x1 + x2 + x3 = (u ^ v) + 2 (a + b + (u & v))
// where a and u & v never both hold, so c = a | (u & v) = (u ? v : x0), and
// b = x2 & ~v.  u and v reach the key through k0 ^ k1 and k2 ^ k3 (k01, k23,
// shared by every head of the group) and the query through q0 ^ q1, q2 ^ q3
// (qp): six three-input logic operations per (key, query) instead of seven.
__device__ __forceinline__ int hamming128_pairs(const uint4 &k, uint32_t k01, uint32_t k23,
                                                const uint4 &q, const uint2 &qp)
{
    const uint32_t u = k01 ^ qp.x, v = k23 ^ qp.y;
    const uint32_t c = (u & v) | (~u & (k.x ^ q.x));
    const uint32_t e = (k.z ^ q.z) & ~v;
    return __popc(u ^ v) + 2 * (__popc(c) + __popc(e));
}

// dist(k, q) for codes of W words (r = 32 W bits): the pair-sum carry-save
// form for W = 4 (kp = k01, k23 and qp = q01, q23 of it), plain population
// counts of the XOR-ed words otherwise.
template <int W>
__device__ __forceinline__ int hamming_w(const uint4 &k, const uint2 &kp, const uint4 &q,
                                         const uint2 &qp)
{
    if constexpr (W == 4) return hamming128_pairs(k, kp.x, kp.y, q, qp);
    if constexpr (W == 2) return __popc(k.x ^ q.x) + __popc(k.y ^ q.y);
    return __popc(k.x ^ q.x);
}

}  // namespace hata
