// k_score.cu -- Hamming scoring of every cached key code.
//
// HATA review page (arXiv 2506.02572), "What carries the argument": the query
// code is XOR-ed with every cached key code and a popcount reduction gives
// the Hamming score; major comment 1 (Algorithm 3): the top-k runs over
// these 129 possible scores.
//
// The work is the flat sequence of 128-token units over all (b, h_kv, group
// of <= 8 query heads) slabs; CTA c takes one contiguous range of about
// U / gridDim.x units, so every CTA gets the same amount of work whatever
// the shapes.  Within its range the CTA's 32 warps take units in the
// order they free up, with no block-wide barrier: lane l scores tokens
// 4l .. 4l+3 of a unit.  The codes arrive by asynchronous copies (cp.async)
// into a per-warp ring of kRing units in shared memory, issued kRing-1
// units ahead: lane l copies tokens l, l+32, l+64, l+96 (coalesced 16-byte
// pieces), each landing in the 64-byte row of the lane that scores it at a
// column XOR-ed with the row (so both the copies and the row reads are free
// of bank conflicts); a wait_group then a warp barrier make the unit
// visible, and the codes in flight cost no registers.  The code stream is
// read from HBM exactly once per KV head.  Each code is scored against every
// query head of the group with a bitwise carry-save sum of its four XOR-ed
// words (x_w = code_w XOR q_w):
//
//   u = x0 ^ x1, v = x2 ^ x3                     (pair sums, weight 1)
//   c = u ? v : x0,  e = x2 & ~v                 (their carries, weight 2)
//   dist = popc(u ^ v) + 2 (popc(c) + popc(e))
//
// i.e. three population counts instead of four (POPC issues at a quarter
// of the integer-logic rate on sm_100a, and it is what bounds the
// arithmetic), and six logic operations, since u and v take the key's
// words as k0 ^ k1 and k2 ^ k3, shared by the group's heads.  Codes of 32
// or 64 bits (the ablation widths) take 4- or 8-byte copies into the same
// 16-byte ring slots and one or two population counts.
//
// Per query head the kernel stores the u8 distance row (a lane's four
// distances as one 32-bit word: a warp writes the head's 128 bytes of the
// unit at once; the row stays L2-resident for the selection kernel) and
// counts a 129-bin histogram per (head, 36K-token tile) in shared memory;
// a range touches at most kMaxKeys (slab, tile) pairs.  At
// the end of its range the CTA adds the non-zero bins into the tile
// histograms in global memory (zeroed by the prep kernel), one reduction
// per bin, so the selection kernel finds both the boundary distance and the
// counts before any tile from them.
//
// 256-bit codes (the widest of the ablation) take their own, plainer kernel
// (score_wide_kernel below): distances 0..256 have 257 values, one more than
// a byte holds, so the stored row saturates at 255 while the histogram keeps
// all 257 bins exactly; the selection recomputes the exact distance of a
// saturated key from the codes when the boundary reaches 255.
#include <algorithm>

#include "hata_internal.cuh"
#include "async_copy.cuh"
#include "score_common.cuh"

namespace hata {
namespace {

constexpr int kWarps = kScoreThreads / 32;  // 32
constexpr int kUnit = 128;                  // tokens per warp step
constexpr int kRing = 2;                    // units per warp ring
constexpr int kTileUnits = kTile / kUnit;   // 288
constexpr int kMaxKeys = 8;                 // (slab, tile) histograms per CTA range
constexpr int kMaxRange = 2048;             // units per CTA range

// Histogram increment: one shared-memory reduction, no return value.
__device__ __forceinline__ void red_shared_add1(uint32_t addr)
{
    asm volatile("red.shared.add.u32 [%0], 1;" ::"r"(addr) : "memory");
}

// One unit's distances against the GB query heads of its group: lane l's
// tokens 4l .. 4l+3 (codes cur[i]) as one 32-bit word per head at word l of
// the head's row (row + g * dist_row), and one count in bin d of head g
// (histogram base hb).  kFull: all 128 tokens hold keys; otherwise the
// tokens from nv on get the pad byte and no count.
template <int GB, int W, bool kFull>
__device__ __forceinline__ void score_unit(const uint4 (&cur)[4], const uint4 *qs,
                                           const uint2 *qp, int ng, uint8_t *row,
                                           int64_t dist_row, uint32_t hb, int lane, int nv)
{
    uint2 kp[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
        kp[i] = W == 4 ? make_uint2(cur[i].x ^ cur[i].y, cur[i].z ^ cur[i].w) : make_uint2(0u, 0u);
#pragma unroll
    for (int g = 0; g < GB; ++g) {
        if (g < ng) {
            const uint4 q = qs[g];
            const uint2 qx = qp[g];
            uint32_t word = 0u;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const uint32_t d = uint32_t(hamming_w<W>(cur[i], kp[i], q, qx));
                if (kFull || 4 * lane + i < nv) {
                    red_shared_add1(hb + uint32_t(g * kHistStride * 4) + 4u * d);
                    word |= d << (8 * i);
                } else {
                    word |= uint32_t(kDistPad) << (8 * i);
                }
            }
            __stcg(reinterpret_cast<uint32_t *>(row + g * dist_row) + lane, word);
        }
    }
}

// A (slab, tile) histogram key of the CTA range: where its rows live.
struct KeyInfo {
    uint4 q[kScoreHeads];  // query codes of the slab's heads
    uint2 qp[kScoreHeads]; // their q0 ^ q1 and q2 ^ q3
    int64_t code0;         // first code (uint4 index) of the slab
    int64_t dist0;         // first distance byte of head 0 of the slab
    int len, ng, slab, pad;
};

template <int GB>
struct ScoreSmem {
    uint4 ring[kWarps][kRing][kUnit];           // 2 KB per unit
    KeyInfo key[kMaxKeys];
    uint32_t hist[kMaxKeys][GB][kHistStride];
    uint32_t unit[kMaxRange];                   // per unit of the range: key << 28 | unit in slab
    int next;                                   // units of the range handed out
};

template <int GB, int W>
__global__ void __launch_bounds__(kScoreThreads, 1) score_kernel(ScoreArgs a)
{
    extern __shared__ __align__(128) uint8_t smem_raw[];
    ScoreSmem<GB> &S = *reinterpret_cast<ScoreSmem<GB> *>(smem_raw);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    pdl_trigger();

    const int nu = int(a.dist_row / kUnit);  // units per slab (pads included)
    const int n_tiles = int(a.n_tiles);
    const int n_units = int(int64_t(a.B) * a.H_kv * a.zgroups * nu);
    const int f_beg = int(int64_t(blockIdx.x) * n_units / gridDim.x);
    const int f_end = int(int64_t(blockIdx.x + 1) * n_units / gridDim.x);
    auto key_of = [&](int f) {
        const int slab = f / nu;
        return slab * n_tiles + (f - slab * nu) / kTileUnits;
    };
    const int k_lo = key_of(f_beg), k_hi = key_of(f_end - 1);
    const int n_keys = k_hi - k_lo + 1;

    // ---- before the dependency wait: the range's keys (seq_len is a step
    // input), cleared histograms, the unit counter ----
    for (int i = tid; i < n_keys * GB * kHistStride; i += kScoreThreads)
        (&S.hist[0][0][0])[i] = 0u;
    if (tid < n_keys) {
        const int slab = (k_lo + tid) / n_tiles;
        const int z = slab % a.zgroups, bh = slab / a.zgroups;
        const int h = bh % a.H_kv, b = bh / a.H_kv;
        const int g0 = z * kScoreHeads;
        KeyInfo &K = S.key[tid];
        K.len = int(clamp_len(__ldg(a.seq_len + b), a.max_seq_len, a.n_cap));
        K.ng = min(GB, a.G - g0);
        K.slab = slab;
        K.code0 = (int64_t(b) * a.H_kv + h) * a.n_cap;
        K.dist0 = (int64_t(b) * a.H_q + int64_t(h) * a.G + g0) * a.dist_row;
    }
    for (int u = tid; u < f_end - f_beg; u += kScoreThreads) {
        const int f = f_beg + u, slab = f / nu;
        S.unit[u] = uint32_t(key_of(f) - k_lo) << 28 | uint32_t(f - slab * nu);
    }
    if (tid == 0) S.next = 0;
    pdl_wait();  // query codes, the appended key code and cleared tile histograms
    if (tid < n_keys * GB) {
        const int kk = tid / GB, g = tid % GB;
        const int slab = (k_lo + kk) / n_tiles;
        const int z = slab % a.zgroups, bh = slab / a.zgroups;
        const int h = bh % a.H_kv, b = bh / a.H_kv;
        const int g0 = z * kScoreHeads;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);  // words past W stay zero
        if (g < min(GB, a.G - g0)) {
            const uint32_t *qp = a.qcodes + (size_t(b) * a.H_q + size_t(h) * a.G + g0 + g) * W;
            if constexpr (W == 4) {
                v = __ldg(reinterpret_cast<const uint4 *>(qp));
            } else {
                v.x = __ldg(qp);
                if constexpr (W == 2) v.y = __ldg(qp + 1);
            }
        }
        S.key[kk].q[g] = v;
        S.key[kk].qp[g] = make_uint2(v.x ^ v.y, v.z ^ v.w);
    }
    __syncthreads();

    // ---- units of the range go to warps on demand (one shared counter):
    // the oldest warps of the SM, which the scheduler favours, take more,
    // and every warp finishes within about one unit of the others ----
    const uint32_t *codes = a.codes;  // W words per token
    const int n_range = f_end - f_beg;
    auto grab = [&]() {
        int u = 0;
        if (lane == 0) u = atomicAdd(&S.next, 1);
        return __shfl_sync(0xffffffffu, u, 0);
    };
    // Token p of a unit lands in row p / 4 (the lane that scores it), at
    // 16-byte column (p % 4) ^ (p / 8 % 4).  Lane l copies tokens l + 32 i,
    // at byte 64 (l / 4) + 16 ((l % 4) ^ (l / 8 % 4)) + 512 i of the slot;
    // it reads token 4 l + i back from column i ^ (l / 2 % 4) of row l.
    const uint32_t copy_off = 64u * uint32_t(lane >> 2) + 16u * uint32_t((lane & 3) ^ ((lane >> 3) & 3));
    // issue the copies of unit u (range-relative) into ring slot `slot`
    auto issue = [&](int u, int slot) {
        asm volatile("" ::: "memory");  // earlier reads of the ring stay before the copies
        if (u < n_range) {
            const uint32_t e = S.unit[u];
            const int uis = int(e & 0x0fffffffu);
            const KeyInfo &K = S.key[e >> 28];
            const int left = K.len - uis * kUnit;
            // 16 bytes per token in the ring, W words of them used
            const uint32_t *src = codes + (K.code0 + int64_t(uis) * kUnit + lane) * W;
            const uint32_t dst = smem_addr(&S.ring[warp][slot][0]) + copy_off;
            if (left >= kUnit) {
#pragma unroll
                for (int i = 0; i < 4; ++i) cp_async_n<4 * W>(dst + 512u * i, src + 32 * W * i);
            } else {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const bool ok = lane + 32 * i < left;  // zero fill past len, no read
                    cp_async_zfill<4 * W>(dst + 512u * i, ok ? src + 32 * W * i : codes,
                                          ok ? 4u * W : 0u);
                }
            }
        }
        cp_async_commit();
    };
    int u_cur = grab();
    issue(u_cur, 0);
    for (int j = 0; u_cur < n_range; ++j) {
        const int u_next = grab();
        __syncwarp();  // every lane is done reading the slot the next copies overwrite
        issue(u_next, (j + 1) % kRing);
        cp_async_wait<kRing - 1>();  // this lane's copies of the current unit have landed
        __syncwarp();                // and so have the other lanes'
        uint4 cur[4];
        const uint4 *mine = &S.ring[warp][j % kRing][4 * lane];
#pragma unroll
        for (int i = 0; i < 4; ++i) cur[i] = mine[(i ^ (lane >> 1)) & 3];
        const uint32_t e = S.unit[u_cur];
        const int uis = int(e & 0x0fffffffu), kk = int(e >> 28);
        const KeyInfo &K = S.key[kk];
        const int c_left = K.len - uis * kUnit;
        uint8_t *c_row = a.dist + K.dist0 + int64_t(uis) * kUnit;
        if (c_left <= 0) {
            // past seq_len: pad bytes only (4 per lane, 128 per head)
#pragma unroll
            for (int g = 0; g < GB; ++g)
                if (g < K.ng) reinterpret_cast<uint32_t *>(c_row + g * a.dist_row)[lane] = 0xffffffffu;
        } else {
            const uint32_t hb = smem_addr(&S.hist[kk][0][0]);
            if (c_left >= kUnit && K.ng == GB)
                score_unit<GB, W, true>(cur, K.q, K.qp, GB, c_row, a.dist_row, hb, lane, kUnit);
            else if (c_left >= kUnit)
                score_unit<GB, W, true>(cur, K.q, K.qp, K.ng, c_row, a.dist_row, hb, lane, kUnit);
            else
                score_unit<GB, W, false>(cur, K.q, K.qp, K.ng, c_row, a.dist_row, hb, lane, c_left);
        }
        u_cur = u_next;
    }
    cp_async_wait<0>();

    // ---- publish: add the non-zero bins of every touched (slab, tile) ----
    __syncthreads();
    for (int i = tid; i < n_keys * GB * kBins; i += kScoreThreads) {
        const int kk = i / (GB * kBins), g = (i / kBins) % GB, t = i % kBins;
        const uint32_t v = S.hist[kk][g][t];
        if (v == 0u || g >= S.key[kk].ng) continue;
        const int key = k_lo + kk;
        atomicAdd(a.hist + (size_t(S.key[kk].dist0 / a.dist_row + g) * size_t(n_tiles) +
                            key % n_tiles) * kHistStride + t,
                  v);
    }
}

// Most (slab, tile) keys any CTA range touches when the U units are cut into
// P ranges (keys are numbered in flat unit order, so a range [f0, f1) touches
// key_of(f1 - 1) - key_of(f0) + 1 of them).
inline int64_t max_keys_per_range(int64_t U, int64_t P, int64_t nu, int64_t n_tiles)
{
    auto key_of = [&](int64_t f) { return (f / nu) * n_tiles + (f % nu) / kTileUnits; };
    int64_t m = 0;
    for (int64_t c = 0; c < P; ++c) {
        const int64_t f0 = c * U / P, f1 = (c + 1) * U / P;
        if (f1 > f0) m = std::max(m, key_of(f1 - 1) - key_of(f0) + 1);
    }
    return m;
}

template <int GB, int W>
cudaError_t launch_score_t(const ScoreArgs &a, cudaStream_t s)
{
    const void *fn = reinterpret_cast<const void *>(score_kernel<GB, W>);
    if (cudaError_t e = ensure_smem_attr(fn, sizeof(ScoreSmem<GB>))) return e;
    int dev = 0, sms = 0, per_sm = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess)
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, score_kernel<GB, W>,
                                                          kScoreThreads, sizeof(ScoreSmem<GB>));
    if (e != cudaSuccess) return e;
    // One range per resident CTA (one per SM); more ranges only if a range
    // would touch more than kMaxKeys (slab, tile) histograms.
    const int64_t nu = a.dist_row / kUnit;
    const int64_t units = int64_t(a.B) * a.H_kv * a.zgroups * nu;
    const int64_t wave = int64_t(per_sm > 0 ? per_sm : 1) * sms;
    int64_t P = wave < units ? wave : units;
    while (P < units && (ceil_div(units, P) > kMaxRange ||
                         max_keys_per_range(units, P, nu, a.n_tiles) > kMaxKeys))
        P = P + wave < units ? P + wave : units;
    return launch_pdl(score_kernel<GB, W>, dim3(unsigned(P)), dim3(kScoreThreads), sizeof(ScoreSmem<GB>),
                      s, a);
}

// ------------------------------------------------------- r = 256 codes --
// The work is the flat sequence of 1024-token pieces of all (b, h_kv, group
// of <= 8 query heads) slabs; CTA c takes one contiguous range of about
// U / gridDim.x pieces (one CTA range per resident CTA, so the CTAs end
// together).  In a piece, thread t scores tokens 4t .. 4t+3: their 32-byte
// codes arrive by coalesced 16-byte asynchronous copies (each warp copies
// its own 4 KB) into a two-piece shared ring, one piece ahead, and are read
// once for all heads of the group.  The four distances of a head go out as one 32-bit word (a warp
// writes 128 consecutive bytes) and into a 257-bin shared histogram per
// head; the histograms go to the (slab, 36K-token tile) rows in global
// memory whenever the range moves to another tile, and at its end.
constexpr int kWideThreads = 256;
constexpr int kWidePiece = 4 * kWideThreads;                      // tokens per piece
constexpr size_t kWideRing = 2 * size_t(kWidePiece) * 2 * 16;    // two pieces of 32-byte codes
static_assert(kTile % kWidePiece == 0, "a piece lies in one histogram tile");

__global__ void __launch_bounds__(kWideThreads, 3) score_wide_kernel(ScoreArgs a)
{
    extern __shared__ __align__(16) uint4 ring[];  // [2][kWidePiece * 2]
    __shared__ uint32_t hist[kScoreHeads][kHistStrideWide];
    __shared__ uint4 qs[kScoreHeads][2];
    __shared__ uint2 qp[kScoreHeads][2];
    pdl_trigger();
    const int tid = threadIdx.x;
    const int64_t per_slab = a.dist_row / kWidePiece;
    const int64_t U = int64_t(a.B) * a.H_kv * a.zgroups * per_slab;
    const int64_t f_beg = int64_t(blockIdx.x) * U / gridDim.x;
    const int64_t f_end = int64_t(blockIdx.x + 1) * U / gridDim.x;
    for (int i = tid; i < kScoreHeads * kHistStrideWide; i += kWideThreads) (&hist[0][0])[i] = 0u;
    pdl_wait();  // query codes, the appended key code, cleared tile histograms

    // copy the warp's 128 codes of piece f (4 KB) into ring slot `slot`:
    // lane l takes 16-byte pieces l, l + 32, ... (coalesced), piece p of the
    // warp (token p / 2, half p % 2) lands in row p / 8 (the lane that reads
    // it: tokens 4 row .. 4 row + 3) at column (p % 8) ^ (row % 8), so each
    // lane's 128-byte row reads back without bank conflicts.  Always commits
    // one group; zero fill past the sequence end.
    const int lane = tid & 31, warp = tid >> 5;
    auto issue = [&](int64_t f, int slot) {
        asm volatile("" ::: "memory");  // earlier reads of the ring stay before the copies
        if (f < f_end) {
            const int64_t slab = f / per_slab;
            const int64_t tw0 = (f - slab * per_slab) * kWidePiece + 128 * warp;  // warp's tokens
            const int bhk = int(slab / a.zgroups), h = bhk % a.H_kv, b = bhk / a.H_kv;
            const int64_t len = clamp_len(__ldg(a.seq_len + b), a.max_seq_len, a.n_cap);
            const uint4 *src = reinterpret_cast<const uint4 *>(a.codes) +
                               ((int64_t(b) * a.H_kv + h) * a.n_cap + tw0) * 2;
            const uint32_t base = smem_addr(ring + size_t(slot) * kWidePiece * 2 + 256 * warp);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int p = lane + 32 * j, row = p >> 3;
                const bool in = tw0 + (p >> 1) < len;
                cp_async16_zfill(base + uint32_t(128 * row + 16 * ((p & 7) ^ (row & 7))),
                                 in ? static_cast<const void *>(src + p) : a.codes,
                                 in ? 16u : 0u);
            }
        }
        cp_async_commit();
    };

    int64_t key = -1;    // (slab, tile) of the histograms being counted
    int ng = 0;          // heads of that slab's group
    int64_t bh0 = 0;     // its first query head
    int64_t len = 0;
    auto flush = [&]() {  // the counts so far to the tile rows, then cleared
        __syncthreads();
        const int64_t tile = key % a.n_tiles;
        for (int i = tid; i < ng * kBinsWide; i += kWideThreads) {
            const int g = i / kBinsWide, t = i % kBinsWide;
            const uint32_t v = hist[g][t];
            if (v) {
                atomicAdd(a.hist + ((bh0 + g) * a.n_tiles + tile) * kHistStrideWide + t, v);
                hist[g][t] = 0u;
            }
        }
    };
    issue(f_beg, 0);
    for (int64_t f = f_beg; f < f_end; ++f) {
        const int slot = int((f - f_beg) & 1);
        __syncwarp();  // every lane is done reading the slot the next copies overwrite
        issue(f + 1, slot ^ 1);
        const int64_t slab = f / per_slab, piece = f - slab * per_slab;
        const int64_t t00 = piece * kWidePiece;
        const int64_t k = slab * a.n_tiles + t00 / kTile;
        if (k != key) {  // CTA-uniform
            if (key >= 0) flush();
            const int z = int(slab % a.zgroups), bhk = int(slab / a.zgroups);
            const int h = bhk % a.H_kv, b = bhk / a.H_kv;
            const int g0 = z * kScoreHeads;
            ng = min(kScoreHeads, a.G - g0);
            bh0 = int64_t(b) * a.H_q + int64_t(h) * a.G + g0;
            len = clamp_len(__ldg(a.seq_len + b), a.max_seq_len, a.n_cap);
            __syncthreads();  // the previous slab's query codes are no longer read
            if (tid < 2 * ng) {
                const int g = tid >> 1, half = tid & 1;
                const uint4 v =
                    __ldg(reinterpret_cast<const uint4 *>(a.qcodes + (bh0 + g) * 8) + half);
                qs[g][half] = v;
                qp[g][half] = make_uint2(v.x ^ v.y, v.z ^ v.w);
            }
            __syncthreads();
            key = k;
        }
        cp_async_wait<1>();                // this lane's copies of piece f have landed
        __syncwarp();                      // and so have the other lanes'
        const uint4 *mine = ring + size_t(slot) * kWidePiece * 2 + 8 * tid;  // row `lane`
        uint4 kc[4][2];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            kc[i][0] = mine[(2 * i) ^ (lane & 7)];
            kc[i][1] = mine[(2 * i + 1) ^ (lane & 7)];
        }
        uint32_t k01[4][2], k23[4][2];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                k01[i][hf] = kc[i][hf].x ^ kc[i][hf].y;
                k23[i][hf] = kc[i][hf].z ^ kc[i][hf].w;
            }
        // this thread's first token and how many of its four hold keys (32-bit:
        // rows are shorter than 2^31)
        const int t0 = int(t00) + 4 * tid;
        const int nv = int(len) - t0;
        uint8_t *drow = a.dist + bh0 * a.dist_row + t0;  // head g: + g * dist_row
        const uint32_t hbase = smem_addr(&hist[0][0]);
        for (int g = 0; g < ng; ++g) {
            const uint4 q0 = qs[g][0], q1 = qs[g][1];
            const uint2 p0 = qp[g][0], p1 = qp[g][1];
            const uint32_t hb = hbase + uint32_t(g * kHistStrideWide * 4);
            uint32_t word = 0u;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                // zero-filled codes past the sequence end are scored too and
                // then neither counted nor stored
                const uint32_t d =
                    uint32_t(hamming128(kc[i][0], k01[i][0], k23[i][0], q0, p0) +
                             hamming128(kc[i][1], k01[i][1], k23[i][1], q1, p1));
                const bool v = i < nv;
                if (v) asm volatile("red.shared.add.u32 [%0], 1;" ::"r"(hb + 4u * d) : "memory");
                word |= (v ? d - (d >> 8) : uint32_t(kDistPad)) << (8 * i);  // 256 saturates to 255
            }
            __stcg(reinterpret_cast<uint32_t *>(drow + g * a.dist_row), word);
        }
    }
    cp_async_wait<0>();
    if (key >= 0) flush();
}

}  // namespace

cudaError_t launch_score(const ScoreArgs &a, cudaStream_t s)
{
    if (a.words == 8) {
        if (cudaError_t e =
                ensure_smem_attr(reinterpret_cast<const void *>(score_wide_kernel), kWideRing))
            return e;
        int dev = 0, sms = 0, per_sm = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (e == cudaSuccess)
            e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, score_wide_kernel,
                                                              kWideThreads, kWideRing);
        if (e != cudaSuccess) return e;
        const int64_t U = int64_t(a.B) * a.H_kv * a.zgroups * (a.dist_row / kWidePiece);
        const int64_t wave = int64_t(per_sm > 0 ? per_sm : 1) * sms;
        return launch_pdl(score_wide_kernel, dim3(unsigned(U < wave ? U : wave)),
                          dim3(kWideThreads), kWideRing, s, a);
    }
    const int gb = a.G < kScoreHeads ? a.G : kScoreHeads;
    if (a.words == 4) {
        switch (gb) {
        case 1: return launch_score_t<1, 4>(a, s);
        case 2: return launch_score_t<2, 4>(a, s);
        case 3: return launch_score_t<3, 4>(a, s);
        case 4: return launch_score_t<4, 4>(a, s);
        case 5: return launch_score_t<5, 4>(a, s);
        case 6: return launch_score_t<6, 4>(a, s);
        case 7: return launch_score_t<7, 4>(a, s);
        default: return launch_score_t<8, 4>(a, s);
        }
    }
    // narrower codes: groups of 3, 5-7 heads take the next wider instance
    // (its unused head slots are skipped)
    if (a.words == 2) {
        if (gb == 1) return launch_score_t<1, 2>(a, s);
        if (gb == 2) return launch_score_t<2, 2>(a, s);
        if (gb <= 4) return launch_score_t<4, 2>(a, s);
        return launch_score_t<8, 2>(a, s);
    }
    if (a.words == 1) {
        if (gb == 1) return launch_score_t<1, 1>(a, s);
        if (gb == 2) return launch_score_t<2, 1>(a, s);
        if (gb <= 4) return launch_score_t<4, 1>(a, s);
        return launch_score_t<8, 1>(a, s);
    }
    return cudaErrorInvalidValue;
}

}  // namespace hata
