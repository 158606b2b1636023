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
// the shapes.  Within its range the CTA's eight warps take units in
// round-robin order (warp w: units w, w+8, ...) with no block-wide barrier:
// lane l owns tokens l, l+32, l+64, l+96 of a unit (four coalesced 16-byte
// loads per warp instruction).  The loads are asynchronous copies
// (cp.async) into a per-warp ring of kRing units in shared memory, issued
// kRing-1 units ahead; every lane reads back only the bytes it copied, so a
// lane's own wait_group is the only synchronisation, and the codes in
// flight cost no registers.  The code stream is read from HBM exactly once
// per KV head.  Each code is scored against every query head of the group:
//
//   x_w = code_w XOR q_w (w = 0..3)
//   (s, c)    = full-add(x0, x1, x2)    -- bitwise carry-save adder
//   (ones, c2) = half-add(s, x3)
//   dist = popc(ones) + 2 popc(c XOR c2) + 4 popc(c AND c2)
//
// i.e. three population counts instead of four: POPC issues at an eighth of
// the integer-logic rate on sm_100a, and it is what bounds the arithmetic.
//
// Per query head the kernel stores the u8 distance row (32 lanes write 32
// consecutive bytes per store; the row stays L2-resident for the selection
// kernel) and counts a 129-bin histogram per (head, 32K-token tile) in
// shared memory; a range touches at most kMaxKeys (slab, tile) pairs.  At
// the end of its range the CTA adds the non-zero bins into the tile
// histograms in global memory (zeroed by the prep kernel), one reduction
// per bin, so the selection kernel finds both the boundary distance and the
// counts before any tile from them.
#include "hata_internal.cuh"
#include "tma.cuh"

namespace hata {
namespace {

constexpr int kWarps = kScoreThreads / 32;  // 8
constexpr int kUnit = 128;                  // tokens per warp step
constexpr int kRing = 2;                    // units per warp ring
constexpr int kTileUnits = kTile / kUnit;   // 256
constexpr int kMaxKeys = 3;                 // (slab, tile) histograms per CTA range

__device__ __forceinline__ int64_t clamp_len(int32_t sl, int64_t max_len, int64_t n_cap)
{
    int64_t l = sl < 0 ? 0 : sl;
    l = l < max_len ? l : max_len;
    return l < n_cap ? l : n_cap;
}

__device__ __forceinline__ int hamming128(const uint4 &k, const uint4 &q)
{
    const uint32_t x0 = k.x ^ q.x, x1 = k.y ^ q.y, x2 = k.z ^ q.z, x3 = k.w ^ q.w;
    const uint32_t s = x0 ^ x1 ^ x2;
    const uint32_t c = (x0 & x1) | (x2 & (x0 ^ x1));
    const uint32_t ones = s ^ x3, c2 = s & x3;
    return __popc(ones) + 2 * __popc(c ^ c2) + 4 * __popc(c & c2);
}

// One (b, h_kv, head group) slab.
struct Slab {
    int b, h, ng;
    int64_t len;
    size_t bh0;  // b * H_q + first query head of the group
};

template <int GB>
struct ScoreSmem {
    uint4 ring[kWarps][kRing][kUnit];        // 32 KB of staged codes
    uint4 qs[kMaxKeys][GB];                  // query codes of each key's slab
    uint32_t hist[kMaxKeys][GB][kHistStride];
    uint8_t tile[kWarps][GB < 4 ? 4 : (GB + 3) / 4 * 4][kUnit];  // a unit's distances
};

// Histogram increment: one shared-memory reduction, no return value.
__device__ __forceinline__ void red_shared_add1(uint32_t addr)
{
    asm volatile("red.shared.add.u32 [%0], 1;" ::"r"(addr) : "memory");
}

// One unit's distances against the GB query heads of its group: byte
// g*128 + 32i of the warp's tile (base tb = tile + lane) and one count in
// bin d of head g (base hb).  kFull: all 128 tokens hold keys; otherwise the
// tokens from nv on get the pad byte and no count.
template <int GB, bool kFull>
__device__ __forceinline__ void score_unit(const uint4 (&cur)[4], const uint4 *qs, int ng,
                                           uint32_t tb, uint32_t hb, int lane, int nv)
{
#pragma unroll
    for (int g = 0; g < GB; ++g) {
        if (g < ng) {
            const uint4 q = qs[g];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const uint32_t d = uint32_t(hamming128(cur[i], q));
                const uint32_t t = tb + uint32_t(g * kUnit + 32 * i);
                if (kFull || lane + 32 * i < nv) {
                    asm volatile("st.shared.u8 [%0], %1;" ::"r"(t), "r"(d) : "memory");
                    red_shared_add1(hb + uint32_t(g * kHistStride * 4) + 4u * d);
                } else {
                    asm volatile("st.shared.u8 [%0], %1;" ::"r"(t), "r"(uint32_t(kDistPad))
                                 : "memory");
                }
            }
        }
    }
}

template <int GB>
__global__ void __launch_bounds__(kScoreThreads, 4) score_kernel(ScoreArgs a)
{
    extern __shared__ __align__(128) uint8_t smem_raw[];
    ScoreSmem<GB> &S = *reinterpret_cast<ScoreSmem<GB> *>(smem_raw);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    pdl_trigger();
    pdl_wait();  // query codes, the appended key code and cleared histograms

    const int nu = int(a.dist_row / kUnit);  // units per slab (pads included)
    const int n_tiles = int(a.n_tiles);
    const int n_units = int(int64_t(a.B) * a.H_kv * a.zgroups * nu);
    const int f_beg = int(int64_t(blockIdx.x) * n_units / gridDim.x);
    const int f_end = int(int64_t(blockIdx.x + 1) * n_units / gridDim.x);
    if (f_beg >= f_end) return;

    auto slab_of = [&](int s) {
        Slab r;
        const int z = s % a.zgroups;
        const int bh = s / a.zgroups;
        r.h = bh % a.H_kv;
        r.b = bh / a.H_kv;
        r.len = clamp_len(__ldg(a.seq_len + r.b), a.max_seq_len, a.n_cap);
        const int g0 = z * kScoreHeads;
        r.ng = min(GB, a.G - g0);
        r.bh0 = size_t(r.b) * a.H_q + size_t(r.h) * a.G + g0;
        return r;
    };
    auto key_of = [&](int slab, int uis) { return slab * n_tiles + uis / kTileUnits; };
    int k_lo, k_hi;
    {
        const int s0 = f_beg / nu, s1 = (f_end - 1) / nu;
        k_lo = key_of(s0, f_beg - s0 * nu);
        k_hi = key_of(s1, f_end - 1 - s1 * nu);
    }

    for (int i = tid; i < kMaxKeys * GB * kHistStride; i += kScoreThreads)
        (&S.hist[0][0][0])[i] = 0u;
    if (tid < kMaxKeys * GB * 4) {  // query codes of every key's slab
        const int kk = tid / (GB * 4), g = (tid / 4) % GB, w = tid & 3;
        uint32_t v = 0u;
        if (k_lo + kk <= k_hi) {
            const Slab r = slab_of((k_lo + kk) / n_tiles);
            if (g < r.ng) v = __ldg(a.qcodes + (r.bh0 + g) * kWords + w);
        }
        reinterpret_cast<uint32_t *>(&S.qs[kk][g])[w] = v;
    }
    __syncthreads();

    const uint4 *codes = reinterpret_cast<const uint4 *>(a.codes);
    const int my_first = f_beg + warp;
    const int my_n = my_first < f_end ? (f_end - 1 - my_first) / kWarps + 1 : 0;
    constexpr int kStep = kWarps * kUnit;  // tokens between a warp's units

    // ---- load side: unit j into ring slot j % kRing, kRing-1 units ahead.
    // l_src points at token t0 + lane of the next unit, l_left = len - t0;
    // both advance by kStep per unit and are rebuilt at a slab change.
    int l_slab = my_first / nu, l_uis = my_first - l_slab * nu;
    const uint4 *l_src = codes;
    int l_left = 0;
    auto l_rebuild = [&]() {
        const Slab r = slab_of(l_slab);
        l_src = codes + (int64_t(r.b) * a.H_kv + r.h) * a.n_cap + int64_t(l_uis) * kUnit + lane;
        l_left = int(r.len - int64_t(l_uis) * kUnit);
    };
    l_rebuild();
    auto issue = [&](int j) {
        asm volatile("" ::: "memory");  // earlier reads of the ring stay before the copies
        if (j < my_n) {
            const uint32_t dst = smem_addr(&S.ring[warp][j % kRing][lane]);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const bool ok = lane + 32 * i < l_left;  // zero fill past len, no read
                cp_async16_zfill(dst + 512u * i, ok ? l_src + 32 * i : codes, ok ? 16u : 0u);
            }
            l_uis += kWarps;
            l_src += kStep;
            l_left -= kStep;
            if (l_uis >= nu) {
                do {
                    l_uis -= nu;
                    ++l_slab;
                } while (l_uis >= nu);
                if (j + 1 < my_n) l_rebuild();
            }
        }
        cp_async_commit();
    };
    for (int j = 0; j < kRing - 1; ++j) issue(j);

    // ---- compute side: c_row = distance row of head 0 at t0, c_left = len - t0
    int c_slab = my_first / nu, c_uis = my_first - c_slab * nu;
    uint8_t *c_row = a.dist;
    int c_left = 0, c_ng = 0, c_kbase = 0;
    auto c_rebuild = [&]() {
        const Slab r = slab_of(c_slab);
        c_row = a.dist + r.bh0 * a.dist_row + int64_t(c_uis) * kUnit;
        c_left = int(r.len - int64_t(c_uis) * kUnit);
        c_ng = r.ng;
        c_kbase = c_slab * n_tiles - k_lo;
    };
    c_rebuild();
    // lane l stores 16 bytes of head (g0 + l / 8) of a unit: its offset in
    // the rows, fixed for the whole range
    const int64_t lane_off = int64_t(lane >> 3) * a.dist_row + (lane & 7) * 16;
    const uint32_t tb = smem_addr(&S.tile[warp][0][0]) + uint32_t(lane);

    for (int j = 0; j < my_n; ++j) {
        issue(j + kRing - 1);
        cp_async_wait<kRing - 1>();  // this lane's copies of unit j have landed
        uint4 cur[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) cur[i] = S.ring[warp][j % kRing][lane + 32 * i];
        const int kk = c_kbase + (c_uis >> 8);  // kTileUnits = 256 units per tile
        if (c_left <= 0) {
            // past seq_len: pad bytes only (4 per lane, 128 per head)
#pragma unroll
            for (int g = 0; g < GB; ++g)
                if (g < c_ng)
                    reinterpret_cast<uint32_t *>(c_row + g * a.dist_row)[lane] = 0xffffffffu;
        } else {
            const uint32_t hb = smem_addr(&S.hist[kk][0][0]);
            if (c_left >= kUnit)
                score_unit<GB, true>(cur, S.qs[kk], c_ng, tb, hb, lane, kUnit);
            else
                score_unit<GB, false>(cur, S.qs[kk], c_ng, tb, hb, lane, c_left);
            __syncwarp();
            // the tile to the rows: lane l stores 16 bytes of head g0 + l / 8
#pragma unroll
            for (int g0 = 0; g0 < GB; g0 += 4) {
                if (g0 + (lane >> 3) < c_ng) {
                    const uint4 v = *reinterpret_cast<const uint4 *>(
                        &S.tile[warp][g0 + (lane >> 3)][(lane & 7) * 16]);
                    __stcg(reinterpret_cast<uint4 *>(c_row + g0 * a.dist_row + lane_off), v);
                }
            }
            __syncwarp();  // the tile is rewritten by the next unit
        }
        c_uis += kWarps;
        c_row += kStep;
        c_left -= kStep;
        if (c_uis >= nu) {
            do {
                c_uis -= nu;
                ++c_slab;
            } while (c_uis >= nu);
            if (j + 1 < my_n) c_rebuild();
        }
    }
    cp_async_wait<0>();

    // ---- publish: add the non-zero bins of every touched (slab, tile) ----
    __syncthreads();
    const int n_keys = k_hi - k_lo + 1;
    for (int i = tid; i < n_keys * GB * kBins; i += kScoreThreads) {
        const int kk = i / (GB * kBins), g = (i / kBins) % GB, t = i % kBins;
        const uint32_t v = S.hist[kk][g][t];
        if (v == 0u) continue;
        const int key = k_lo + kk;
        const Slab r = slab_of(key / n_tiles);
        if (g < r.ng)
            atomicAdd(a.hist + ((r.bh0 + g) * size_t(n_tiles) + key % n_tiles) * kHistStride + t, v);
    }
}

template <int GB>
cudaError_t launch_score_t(const ScoreArgs &a, cudaStream_t s)
{
    const void *fn = reinterpret_cast<const void *>(score_kernel<GB>);
    if (cudaError_t e = ensure_smem_attr(fn, sizeof(ScoreSmem<GB>))) return e;
    int dev = 0, sms = 0, per_sm = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess)
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, score_kernel<GB>,
                                                          kScoreThreads, sizeof(ScoreSmem<GB>));
    if (e != cudaSuccess) return e;
    // One range per resident CTA, unless ranges would touch more than
    // kMaxKeys = 3 (slab, tile) pairs.  Slabs of >= kTileUnits units: a range
    // of <= kTileUnits units meets at most the end of one tile, a short last
    // tile and the start of the next slab.  Shorter slabs are one key each:
    // a range of <= 2 * nu units meets at most three of them.
    const int64_t nu = a.dist_row / kUnit;
    const int64_t units = int64_t(a.B) * a.H_kv * a.zgroups * nu;
    const int64_t max_range = nu >= kTileUnits ? kTileUnits : (kMaxKeys - 1) * nu;
    int64_t P = int64_t(per_sm > 0 ? per_sm : 1) * sms;
    if (P * max_range < units) P = ceil_div(units, max_range);
    if (P > units) P = units;
    return launch_pdl(score_kernel<GB>, dim3(unsigned(P)), dim3(kScoreThreads), sizeof(ScoreSmem<GB>),
                      s, a);
}

}  // namespace

cudaError_t launch_score(const ScoreArgs &a, cudaStream_t s)
{
    const int gb = a.G < kScoreHeads ? a.G : kScoreHeads;
    switch (gb) {
    case 1: return launch_score_t<1>(a, s);
    case 2: return launch_score_t<2>(a, s);
    case 3: return launch_score_t<3>(a, s);
    case 4: return launch_score_t<4>(a, s);
    case 5: return launch_score_t<5>(a, s);
    case 6: return launch_score_t<6>(a, s);
    case 7: return launch_score_t<7>(a, s);
    default: return launch_score_t<8>(a, s);
    }
}

}  // namespace hata
