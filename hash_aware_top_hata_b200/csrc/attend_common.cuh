// attend_common.cuh -- the tensor-core attention stage over 16 gathered
// bf16 K/V rows, shared by the attention kernels.
//
// HATA review page (arXiv 2506.02572), "What carries the argument": the
// top-k indices select K/V rows and exact softmax attention runs over them.
//
// A warp computes a 16-key stage as mma.sync m16n8k16 bf16 tiles with fp32
// accumulation and the keys along M: S^T = K Q^T, then O^T += V^T P^T,
// 8 + 8 mma per stage, fed by ldmatrix (transposed for V) from an
// XOR-swizzled layout (16-byte piece p of key row r sits at piece p ^ (r & 7),
// so the eight rows one ldmatrix reads hit eight different bank groups).
// The B operands are the query (resp. the softmax weights) split into two
// bf16 columns, hi = bf16(x) and lo = bf16(x - hi), whose sum carries ~16
// mantissa bits, so the tensor cores reproduce the fp32 result; the two
// columns are summed inside a lane.  The softmax rescale is lazy: the
// reference maximum moves only when a score exceeds it by more than 2^8
// (exact: weights stay <= 2^8).
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "hata_internal.cuh"

namespace hata {
namespace tc {


constexpr int kSub = 16;                           // keys per stage
constexpr int kRingW = 3;                          // stages per warp ring
constexpr int kTcWarps = 8;
constexpr int kThreads = 32 * kTcWarps;
constexpr int kRowB = kD * 2;                      // bf16 row bytes
constexpr int kStageBytes = 2 * kSub * kRowB;      // K + V
constexpr int kIdxCap = 4096;                      // indices of the CTA slice kept in smem
constexpr float kLazy = 8.0f;                      // rescale threshold, log2 units
constexpr size_t kRingBytes = size_t(kTcWarps) * kRingW * kStageBytes;
constexpr size_t kSmem = kRingBytes + sizeof(int32_t) * kIdxCap;

__device__ __forceinline__ uint32_t swz(int row, int piece)
{
    return uint32_t(row * kRowB + ((piece ^ (row & 7)) << 4));
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2,
                                        uint32_t &r3)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2,
                                          uint32_t &r3)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

__device__ __forceinline__ uint32_t pack2(float lo, float hi)
{
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&v);
}

// x as the bf16 row `part` of a hi/lo pair: part 0 -> bf16(x), 1 -> bf16(x - bf16(x)).
__device__ __forceinline__ float split(float x, int part)
{
    const float hi = __bfloat162float(__float2bfloat16_rn(x));
    return part == 0 ? hi : x - hi;
}

// 2^x on the special-function unit (relative error ~2^-22; -inf -> +0).
__device__ __forceinline__ float fast_exp2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// d += A(16x16) * B(16x8), all four A registers live.
__device__ __forceinline__ void mma16816_full(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                              uint32_t a3, uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Per-lane ldmatrix offsets inside a stage (constant for a warp's life).
// Matrix mi = lane >> 3 of an x4 load, row lane & 7 of it:
//   K (A = 16 keys x 16 dims of k-tile kt): key (mi & 1)*8 + (lane & 7),
//     16-byte piece 2 kt + (mi >> 1);
//   V (A = 16 dims of m-tile mt x 16 keys, transposed load): key
//     (mi >> 1)*8 + (lane & 7), piece 2 mt + (mi & 1).
// Piece 2t + b swizzles to (2t + b) ^ (r & 7) = ((b ^ (r & 7)) ^ 2t), so tile
// t's offset is the tile-0 offset XOR (t << 5).
struct LaneOffsets {
    uint32_t k0, v0;
    __device__ __forceinline__ explicit LaneOffsets(int lane)
    {
        const int mi = lane >> 3, r7 = lane & 7;
        k0 = swz((mi & 1) * 8 + r7, mi >> 1);
        v0 = swz((mi >> 1) * 8 + r7, mi & 1);
    }
    __device__ __forceinline__ uint32_t k(int kt) const { return k0 ^ uint32_t(kt << 5); }
    __device__ __forceinline__ uint32_t v(int mt) const { return v0 ^ uint32_t(mt << 5); }
};

// One 16-key stage of one warp.  Keys run along the M dimension of the
// tiles: S^T = K Q^T with B = [q_hi q_lo 0 ...] (16 dims x 8 columns), then
// O^T += V^T P^T with B = [p_hi p_lo 0 ...] (16 keys x 8 columns), so each
// stage is 8 + 8 mma and the hi + lo columns are summed inside a lane.
// Lane (g = lane / 4, t = lane % 4) of an m16n8 accumulator holds rows g and
// g + 8, columns 2t and 2t + 1: only lanes with t == 0 see the two live
// columns.  O[mt] in those lanes: dims 16 mt + g (O[mt][0] + O[mt][1]) and
// 16 mt + g + 8 (O[mt][2] + O[mt][3]).
// The B operand of S^T = K Q^T for query row q (pre-scaled by scale_log2):
// column 0 (lanes 0-3) holds bf16(q), column 1 (lanes 4-7) the remainder
// q - bf16(q); the other columns are zero.
// kLdg: q was written by an earlier kernel (read-only path); otherwise plain
// loads (q staged in shared memory).
template <bool kLdg = true>
__device__ __forceinline__ void load_query(const float *q, float scale_log2, int lane,
                                           uint32_t (&qb)[8][2])
{
    auto ld2 = [](const float *p) {
        if constexpr (kLdg) return __ldg(reinterpret_cast<const float2 *>(p));
        else return *reinterpret_cast<const float2 *>(p);
    };
    const int part = (lane >> 2) & 1, q4 = lane & 3;
#pragma unroll
    for (int kt = 0; kt < 8; ++kt) {
        const int d0 = 16 * kt + 2 * q4;
        if (lane < 8) {
            const float2 x = ld2(q + d0);
            const float2 y = ld2(q + d0 + 8);
            qb[kt][0] = pack2(split(x.x * scale_log2, part), split(x.y * scale_log2, part));
            qb[kt][1] = pack2(split(y.x * scale_log2, part), split(y.y * scale_log2, part));
        } else {
            qb[kt][0] = qb[kt][1] = 0u;
        }
    }
}

// vmask: bit j set if key j of the stage holds a row.
__device__ __forceinline__ void attend_stage(uint32_t vmask, uint32_t Ks,
                                             const uint32_t (&qb)[8][2], const LaneOffsets &lo,
                                             float (&O)[8][4], float &m_ref, float &l_part,
                                             int lane)
{
    const uint32_t Vs = Ks + kSub * kRowB;
    const int g = lane >> 2, t = lane & 3;
    // ---- S^T = K Q^T: even / odd k-tiles in separate accumulators ----
    float S[2][4];
#pragma unroll
    for (int h = 0; h < 2; ++h) S[h][0] = S[h][1] = S[h][2] = S[h][3] = 0.0f;
#pragma unroll
    for (int kt = 0; kt < 8; ++kt) {
        uint32_t a0, a1, a2, a3;
        ldsm_x4(Ks + lo.k(kt), a0, a1, a2, a3);
        mma16816_full(S[kt & 1], a0, a1, a2, a3, qb[kt][0], qb[kt][1]);
    }
    // lanes t == 0: key g (columns hi + lo) and key g + 8
    const float s_g = (S[0][0] + S[1][0]) + (S[0][1] + S[1][1]);
    const float s_g8 = (S[0][2] + S[1][2]) + (S[0][3] + S[1][3]);
    // every lane takes keys 2t, 2t + 1, 2t + 8, 2t + 9 (the P^T fragment's rows)
    float sc[4];
    sc[0] = __shfl_sync(0xffffffffu, s_g, 8 * t);
    sc[2] = __shfl_sync(0xffffffffu, s_g8, 8 * t);
    sc[1] = __shfl_sync(0xffffffffu, s_g, 8 * t + 4);
    sc[3] = __shfl_sync(0xffffffffu, s_g8, 8 * t + 4);
    bool valid[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const int key = 2 * t + (e & 1) + 8 * (e >> 1);
        valid[e] = (vmask >> key) & 1u;
        if (!valid[e]) sc[e] = -INFINITY;
    }
    float mx = fmaxf(fmaxf(sc[0], sc[1]), fmaxf(sc[2], sc[3]));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));  // the same in every lane
    if (mx == -INFINITY) return;
    if (mx > m_ref + kLazy) {
        const float alpha = fast_exp2(m_ref - mx);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            O[j][0] *= alpha; O[j][1] *= alpha; O[j][2] *= alpha; O[j][3] *= alpha;
        }
        l_part *= alpha;
        m_ref = mx;
    }
    float pv[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const float pe = valid[e] ? fast_exp2(sc[e] - m_ref) : 0.0f;
        l_part += pe;
        pv[e] = split(pe, g & 1);
    }
    const uint32_t b0 = g < 2 ? pack2(pv[0], pv[1]) : 0u;
    const uint32_t b1 = g < 2 ? pack2(pv[2], pv[3]) : 0u;
    // ---- O^T += V^T P^T: 8 m-tiles of 16 dims, one k-tile of 16 keys ----
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
        uint32_t a0, a1, a2, a3;
        ldsm_x4_t(Vs + lo.v(mt), a0, a1, a2, a3);
        mma16816_full(O[mt], a0, a1, a2, a3, b0, b1);
    }
}

// Write a warp's partial (m, l, acc[128]) to pp (global or shared).
__device__ __forceinline__ void store_partial(float *pp, const float (&O)[8][4], float m_ref,
                                              float l_part, int lane)
{
    float lw = lane < 4 ? l_part : 0.0f;  // lanes 0-3 hold all 16 keys of every stage
    lw += __shfl_xor_sync(0xffffffffu, lw, 1);
    lw += __shfl_xor_sync(0xffffffffu, lw, 2);
    if ((lane & 3) == 0) {  // lane 4g: dims 16 mt + g and 16 mt + g + 8, hi + lo columns
        const int g = lane >> 2;
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
            pp[4 + 16 * mt + g] = O[mt][0] + O[mt][1];
            pp[4 + 16 * mt + g + 8] = O[mt][2] + O[mt][3];
        }
    }
    if (lane == 0) {
        pp[0] = m_ref;
        pp[1] = lw;
    }
}

}  // namespace tc
}  // namespace hata
