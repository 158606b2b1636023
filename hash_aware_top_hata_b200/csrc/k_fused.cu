// k_fused.cu -- the selection and the gather + attention of a decode step
// as ONE persistent kernel, after the scoring kernel: selection warps turn
// the distance rows into index lists while attention warps already gather
// and attend the heads selected so far.
//
// HATA review page (arXiv 2506.02572), "What carries the argument": the top-k
// indices select K/V rows and exact attention runs over them; the page's
// implementation fuses kernels and gathers inside the attention.  Referee
// report, major comment 1 (Algorithm 3): the top-k runs over 129 possible
// scores; here the boundary bucket goes to the lower token indices, so the
// selected set is unique.
//
// As separate kernels, the selection (latency-bound: a threshold from the
// tile histograms, one block scan and an ordered compaction per 36K-token
// tile) runs while HBM idles, and the attention waits for all of it.  Here
// one CTA per SM runs three kinds of warps at once:
//
//   * kSW selection warps (288 threads): the CTA's selection tiles, statically
//     assigned (tile i of the flat (head, tile) sequence to CTA i mod P, in
//     head order), each the multi-kernel selection's arithmetic
//     (select_common.cuh); a finished tile is handed to the publisher.
//   * kAW attention warps.  Stage s of CTA c is attention item j = s*P + c:
//     kFSeg consecutive entries of one head's selected list, 16 per warp.  A
//     warp waits until the head is selected, gathers its 16 K and V rows and
//     the query through a private cp.async ring, runs the tensor-core stage
//     (attend_common.cuh) and leaves a partial (m, l, acc) in shared memory.
//   * one publisher warp.  It merges each attention item's kAW partials into
//     one, releases finished selection tiles and attention items to the other
//     CTAs through counters (one GPU-scope fence per batch), polls the
//     counters of the heads its attention warps will need next, and, when it
//     completes a head, merges the head's item partials into out.  Only this
//     warp fences at GPU scope, so the other warps never wait behind their
//     own copies in flight.
//
// Hand-offs inside a CTA use mbarriers (every waiter at most one phase
// behind) and monotonic counters; between CTAs counters with acquire /
// release.  Every wait is bounded by spin_limit_ns of wall time; a wait that
// gives up sets HATA_FLAG_TIMEOUT and the CTA abandons its remaining work
// (its warps keep their control flow, so every named barrier is still met).
#include <cuda_bf16.h>

#include "async_copy.cuh"
#include "attend_common.cuh"
#include "hata_internal.cuh"
#include "select_common.cuh"
#include "sync.cuh"

namespace hata {
namespace {

constexpr int kSW = 9;                     // selection warps
constexpr int kAW = 6;                     // attention warps
constexpr int kPubWarp = kSW + kAW;        // the publisher
constexpr int kThreads = 32 * (kSW + kAW + 1);
// 16 warps: four per SM sub-partition (each holds a quarter of the register
// file), so 128 registers per thread
constexpr int kRegs = (65536 / kThreads) / 8 * 8;
static_assert(kThreads == 512, "four warps per sub-partition");
constexpr int kST = 32 * kSW;              // selection threads = one tile pass
constexpr int kRingA = 3;                  // stages per attention-warp ring
constexpr int kPSlots = 3;                 // attention items in flight
constexpr int kQBytes = kD * 4;
constexpr int kSlotBytes = tc::kStageBytes + kQBytes;  // K, V rows (swizzled) + q
constexpr int kSelPer = kTile / kST;       // distances per selection thread in a tile
constexpr int kSelPieces = kSelPer / 16;
constexpr int kSelGroups = kSelPer / 32;
constexpr int kSelBar = 1;                 // named barrier of the selection warps
constexpr int kSelQ = 8;                   // selection hand-off queue
static_assert(kST * kSelPer == kTile, "a selection tile is one pass of the selection threads");
static_assert(kFSeg == tc::kSub * kAW, "an attention item is one stage of every attention warp");

struct FSmem {
    uint8_t aring[kAW][kRingA][kSlotBytes];         // attention stages
    float pslot[kPSlots][kAW][kPartStride];         // attention warp partials
    uint64_t mb_item[kPSlots];        // attention warps wrote the slot's partials
    uint64_t mb_item_free[kPSlots];   // the publisher merged them
    uint32_t vmask[kAW][kRingA];      // rows present in each attention stage
    int32_t selq[kSelQ];              // heads whose selection tile is done
    uint32_t selq_w, selq_r;          // written by selection thread 0 / by the publisher
    uint32_t a_ready;                 // this CTA's attention stages whose head is selected
                                      // (a prefix, posted by the publisher)
    int2 scan2[kSW + 1];
    int thr[4];
    uint32_t abort;                   // a wait of this CTA gave up
};
static_assert(sizeof(FSmem) <= 227 * 1024, "one CTA per SM: at most 227 KB of shared memory");

// ------------------------------------------------------------ waiting --

// This CTA gave up (a shared-memory read: cheap enough for hot loops).
__device__ __forceinline__ bool aborted_here(const FSmem &S)
{
    return *reinterpret_cast<const volatile uint32_t *>(&S.abort) != 0u;
}

// This CTA or any other gave up in this step (also reads the step's abort
// word in global memory: only for loops that are waiting anyway).
__device__ __forceinline__ bool aborted(const FusedArgs &a, const FSmem &S)
{
    return aborted_here(S) || ld_relaxed_gpu(a.abort_word) != 0u;
}

// Give up: this CTA stops its work, the other CTAs stop waiting (the step's
// abort word, cleared by prep every step) and the caller is told
// (HATA_FLAG_TIMEOUT, read by hata_workspace_check).
__device__ __noinline__ void give_up_impl(uint32_t *flags, uint32_t *step_abort, uint32_t *abort)
{
    *reinterpret_cast<volatile uint32_t *>(abort) = 1u;
    atomicOr(step_abort, 1u);
    atomicOr(flags, HATA_FLAG_TIMEOUT);
}
__device__ __forceinline__ void give_up(const FusedArgs &a, FSmem &S)
{
    give_up_impl(a.flags, a.abort_word, &S.abort);
}

// Wait (bounded) for the phase of parity `par` of an mbarrier.
__device__ __forceinline__ bool wait_mbar(const FusedArgs &a, FSmem &S, uint64_t *bar,
                                          uint32_t par)
{
    if (mbar_test(bar, par)) return true;
    const uint64_t t0 = global_ns();
    for (;;) {
        if (mbar_test(bar, par)) return true;
        if (aborted(a, S) || global_ns() - t0 > a.spin_limit_ns) {
            give_up(a, S);
            return false;
        }
        nanosleep_ns(64);
    }
}

// One test of an mbarrier phase by lane 0, the same answer for the whole
// warp (the publisher's decisions must be warp-uniform).
__device__ __forceinline__ bool poll_uniform(uint64_t *bar, uint32_t par)
{
    bool done = false;
    if ((threadIdx.x & 31) == 0) done = mbar_test(bar, par);
    return __shfl_sync(0xffffffffu, done, 0);
}

// -------------------------------------------------------------- layout --

__device__ __forceinline__ int seq_len_of(const FusedArgs &a, int b)
{
    return int(clamp_len(__ldg(a.seq_len + b), a.max_seq_len, a.n_cap));
}

struct Sched {
    int P, c;        // CTAs, this CTA
    int n_sel;       // selection tiles in all ((head, tile) pairs)
    int sel_items;   // of this CTA
    int J;           // attention items in all
    int stages;      // of this CTA
};

__device__ __forceinline__ int share(int n, int P, int c) { return c < n ? (n - c + P - 1) / P : 0; }

// Attention stage s of this CTA: item j = c + s P, kFSeg entries of one
// head's list.  Does the item hold any selected entry?
__device__ __forceinline__ bool stage_rows(const FusedArgs &a, const Sched &sc, int s,
                                           int64_t *bh_out)
{
    const int j = s * sc.P + sc.c;
    const int64_t bh = j / a.n_seg;
    const int seg = j - int(bh) * a.n_seg;
    const int len = seq_len_of(a, int(bh / a.H_q));
    const int k_eff = a.topk < len ? a.topk : len;
    *bh_out = bh;
    return seg * kFSeg < k_eff;
}

// --------------------------------------------------------- selection --

// Selection tile i = (head bh, tile) of the flat sequence, by the kST
// selection threads: the head's index entries of the tile, ascending, lower
// index first at the boundary distance -- the multi-kernel selection's
// arithmetic (select_common.cuh).  Ends by handing the head to the
// publisher.
__device__ __forceinline__ void select_tile(const FusedArgs &a, FSmem &S, int i, int tid)
{
    const int64_t bh = i / a.n_tiles;
    const int tile = i - int(bh) * a.n_tiles;
    const int len = seq_len_of(a, int(bh / a.H_q));
    const int k_eff = a.topk < len ? a.topk : len;
    int32_t *idx = a.idx + bh * a.topk;
    if (tile == 0)
        for (int x = k_eff + tid; x < a.topk; x += kST) idx[x] = -1;
    if (k_eff > 0 && int64_t(tile) * kTile < len) {  // uniform
        const uint8_t *drow = a.dist + bh * a.dist_row;
        const int lane = tid & 31;
        if (tid < 32)
            head_threshold<false, 8>(a.hist + bh * int64_t(a.n_tiles) * kHistStride, a.n_tiles,
                                     k_eff, tile, lane, S.thr);
        const int64_t my0 = int64_t(tile) * kTile + int64_t(tid) * kSelPer;
        uint4 dv[kSelPieces];
#pragma unroll
        for (int v = 0; v < kSelPieces; ++v)
            dv[v] = my0 + 16 * v < a.dist_len
                        ? __ldg(reinterpret_cast<const uint4 *>(drow + my0 + 16 * v))
                        : make_uint4(~0u, ~0u, ~0u, ~0u);
        named_bar_sync(kSelBar, kST);
        const int T = S.thr[0], n_less = S.thr[1], lp = S.thr[2], tp = S.thr[3];
        const int r_ties = k_eff - n_less;
        const int placed = lp + (tp < r_ties ? tp : r_ties);
        if (placed < k_eff) {  // uniform
            const uint32_t T4 = uint32_t(T) * 0x01010101u, T4p = T4 + 0x01010101u;
            uint32_t lt_bits[kSelGroups], eq_bits[kSelGroups];
            int n_lt = 0, n_eq = 0;
#pragma unroll
            for (int m = 0; m < kSelGroups; ++m) {
                const uint32_t dw[8] = {dv[2 * m].x,     dv[2 * m].y,     dv[2 * m].z,
                                        dv[2 * m].w,     dv[2 * m + 1].x, dv[2 * m + 1].y,
                                        dv[2 * m + 1].z, dv[2 * m + 1].w};
                if (T < 128)
                    group_masks<false>(dw, T4, T4p, lt_bits[m], eq_bits[m]);
                else
                    group_masks<true>(dw, T4, T4p, lt_bits[m], eq_bits[m]);
                n_lt += __popc(lt_bits[m]);
                n_eq += __popc(eq_bits[m]);
            }
            int tile_lt, tile_eq;
            const int2 before = block_exclusive_scan2<kST, kSelBar>(n_lt, n_eq, S.scan2, &tile_lt,
                                                                    &tile_eq);
            const int room = r_ties - tp > 0 ? r_ties - tp : 0;
            const int take_tile = room < tile_eq ? room : tile_eq;
            const int taken_before = before.y < take_tile ? before.y : take_tile;
            int my_take = take_tile - before.y;
            my_take = my_take < 0 ? 0 : (my_take > n_eq ? n_eq : my_take);
            const int pos = placed + before.x + taken_before;
            emit_selected(lt_bits, eq_bits, my_take, pos, int(my0), [&](int p, int tok) {
                if (p < a.topk) idx[p] = tok;
            });
        }
    }
    named_bar_sync(kSelBar, kST);  // every entry of the tile is written
    if (tid == 0) {
        // hand the head to the publisher (queue of kSelQ entries)
        const uint32_t w = S.selq_w;
        const uint64_t t0 = global_ns();
        while (w - ld_acquire_cta(&S.selq_r) >= kSelQ) {
            if (aborted(a, S) || global_ns() - t0 > a.spin_limit_ns) {
                give_up(a, S);
                break;
            }
            nanosleep_ns(64);
        }
        S.selq[w % kSelQ] = int32_t(bh);
        st_release_cta(&S.selq_w, w + 1);
    }
}

__device__ __forceinline__ void select_role(const FusedArgs &a, FSmem &S, const Sched &sc, int tid)
{
    for (int k = 0; k < sc.sel_items; ++k) select_tile(a, S, sc.c + k * sc.P, tid);
}

// --------------------------------------------------------- attention --

__device__ __forceinline__ void attend_role(const FusedArgs &a, FSmem &S, const Sched &sc, int aw,
                                            int lane)
{
    using namespace tc;
    const uint32_t ring = smem_addr(&S.aring[aw][0][0]);
    const int p = lane & 15, rh = lane >> 4;  // piece p of rows 8 rh .. 8 rh + 7
    uint32_t doff[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) doff[u] = swz(8 * rh + u, p);

    struct Item {
        int64_t bh;
        int b, h, len, x0, nr;  // rows x0 .. x0 + nr - 1 of the head's list
    };
    auto item_of = [&](int s) {
        Item it;
        const int j = s * sc.P + sc.c;
        it.bh = j / a.n_seg;
        const int seg = j - int(it.bh) * a.n_seg;
        it.b = int(it.bh / a.H_q);
        it.h = int(it.bh - int64_t(it.b) * a.H_q) / a.G;
        it.len = seq_len_of(a, it.b);
        const int k_eff = a.topk < it.len ? a.topk : it.len;
        it.x0 = seg * kFSeg + kSub * aw;
        it.nr = k_eff - it.x0 < 0 ? 0 : (k_eff - it.x0 > kSub ? kSub : k_eff - it.x0);
        return it;
    };
    // the stage's 16 indices (lane l < 16 holds entry x0 + l), once the head
    // is selected
    auto fetch = [&](int s) -> int32_t {
        if (s >= sc.stages) return -1;
        const Item it = item_of(s);
        if (it.nr <= 0) return -1;
        // the publisher posts, in order, the stages whose head is selected
        bool ok = ld_acquire_cta(&S.a_ready) > uint32_t(s);
        if (!ok) {
            const uint64_t t0 = global_ns();
            for (;;) {
                nanosleep_ns(128);
                if (ld_acquire_cta(&S.a_ready) > uint32_t(s)) {
                    ok = true;
                    break;
                }
                if (aborted(a, S) || global_ns() - t0 > a.spin_limit_ns) {
                    give_up(a, S);
                    break;
                }
            }
        }
        ok = __all_sync(0xffffffffu, ok);
        return ok && lane < it.nr ? __ldcg(a.idx + it.bh * a.topk + it.x0 + lane) : -1;
    };
    // gather stage s into ring slot s % kRingA (always one group)
    auto issue = [&](int s, int32_t v) {
        if (s < sc.stages) {
            const Item it = item_of(s);
            const int slot = s % kRingA;
            const uint32_t Ks = ring + uint32_t(slot * kSlotBytes), Vs = Ks + kSub * kRowB,
                           Qs = Ks + tc::kStageBytes;
            const int64_t slab = (int64_t(it.b) * a.H_kv + it.h) * a.n_cap;
            const uint8_t *Kp = static_cast<const uint8_t *>(a.K) + slab * kRowB + p * 16;
            const uint8_t *Vp = static_cast<const uint8_t *>(a.V) + slab * kRowB + p * 16;
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int32_t row = __shfl_sync(0xffffffffu, v, 8 * rh + u);
                // the selection never yields an index outside [0, len); the
                // check keeps a corrupted list from steering a copy outside
                // the cache.  Rows without a key are zero-filled.
                const bool ok = row >= 0 && row < it.len;
                const int64_t off = ok ? int64_t(row) * kRowB : 0;
                cp_async16_zfill(Ks + doff[u], Kp + off, ok ? 16u : 0u);
                cp_async16_zfill(Vs + doff[u], Vp + off, ok ? 16u : 0u);
            }
            const uint32_t vm = __ballot_sync(0xffffffffu, lane < kSub && v >= 0 && v < it.len);
            if (vm) cp_async16_zfill(Qs + 16u * lane, a.q + it.bh * kD + 4 * lane, 16u);
            if (lane == 0) S.vmask[aw][slot] = vm;
        }
        cp_async_commit();
    };

    // prologue: stages 0 .. kRingA-2 in flight, the indices of the next one
    // loaded
    int32_t v_next = -1;
#pragma unroll
    for (int s = 0; s < kRingA - 1; ++s) issue(s, fetch(s));
    v_next = fetch(kRingA - 1);
    const LaneOffsets lo(lane);
    for (int s = 0; s < sc.stages; ++s) {
        cp_async_wait<kRingA - 2>();  // stage s has landed
        __syncwarp();
        issue(s + kRingA - 1, v_next);  // into the slot of stage s - 1, computed last time
        v_next = fetch(s + kRingA);
        const int slot = s % kRingA;
        const uint32_t vm = S.vmask[aw][slot];
        float O[8][4];
#pragma unroll
        for (int j = 0; j < 8; ++j) O[j][0] = O[j][1] = O[j][2] = O[j][3] = 0.0f;
        float m_ref = -INFINITY, l_part = 0.0f;
        if (vm) {
            const uint32_t Ks = ring + uint32_t(slot * kSlotBytes);
            uint32_t qb[8][2];
            load_query<false>(reinterpret_cast<const float *>(&S.aring[aw][slot][tc::kStageBytes]),
                              a.scale_log2, lane, qb);
            attend_stage(vm, Ks, qb, lo, O, m_ref, l_part, lane);
        }
        const int ps = s % kPSlots;
        if (s >= kPSlots) wait_mbar(a, S, &S.mb_item_free[ps], uint32_t((s / kPSlots - 1) & 1));
        store_partial(S.pslot[ps][aw], O, m_ref, l_part, lane);
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.mb_item[ps]);
    }
    cp_async_wait<0>();
}

// --------------------------------------------------------- publisher --

// Merge the n partials (m, l, -, -, acc[128]) at pc (stride kPartStride,
// written by other CTAs) into out[128] = acc / l.  One warp; lane l owns
// dims l, l+32, l+64, l+96; rounds of 16 partials, all loads of a round
// issued together.
__device__ __forceinline__ void merge_partials(const float *pc, int n, float *out, int lane)
{
    constexpr int kRound = 16;
    float M = -INFINITY, L = 0.0f, A[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    for (int c0 = 0; c0 < n; c0 += kRound) {
        const int c = c0 + lane;
        const bool mine = lane < kRound && c < n;
        const float mc = mine ? __ldcg(pc + int64_t(c) * kPartStride) : -INFINITY;
        const float lc = mine ? __ldcg(pc + int64_t(c) * kPartStride + 1) : 0.0f;
        float acc[kRound][4];
#pragma unroll
        for (int j = 0; j < kRound; ++j) {
            const float *q = pc + int64_t(c0 + j) * kPartStride + 4 + lane;
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[j][i] = c0 + j < n ? __ldcg(q + 32 * i) : 0.0f;
        }
        float mr = mc;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mr = fmaxf(mr, __shfl_xor_sync(0xffffffffu, mr, o));
        const float Mn = fmaxf(M, mr);
        if (Mn == -INFINITY) continue;  // warp-uniform: no weight yet
        if (M != Mn) {
            const float r = M == -INFINITY ? 0.0f : exp2f(M - Mn);
            L *= r;
#pragma unroll
            for (int i = 0; i < 4; ++i) A[i] *= r;
            M = Mn;
        }
        const float wc = mc == -INFINITY ? 0.0f : exp2f(mc - M);
        float lw = lc * wc;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) lw += __shfl_xor_sync(0xffffffffu, lw, o);
        L += lw;
#pragma unroll
        for (int j = 0; j < kRound; ++j) {
            const float w = __shfl_sync(0xffffffffu, wc, j);
#pragma unroll
            for (int i = 0; i < 4; ++i) A[i] = fmaf(acc[j][i], w, A[i]);
        }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) out[lane + 32 * i] = L > 0.0f ? A[i] / L : 0.0f;
}

__device__ __forceinline__ void publisher_role(const FusedArgs &a, FSmem &S, const Sched &sc,
                                               int lane)
{
    int sa = 0, sr = 0;  // items merged, selections released
    int ardy = 0;        // attention stages known ready
    uint64_t t_idle = global_ns();
    const int n_stages = sc.stages, n_sel = sc.sel_items;
    while ((sa < n_stages || sr < n_sel || ardy < n_stages) && !aborted_here(S)) {
        bool progress = false;
        // ---- poll the heads of the next attention stages (lanes 0-7,
        // relaxed loads issued together; the fence below makes them acquire;
        // the item work below runs while they are in flight) ----
        bool rdy = true;
        if (lane < 8) {
            const int st = ardy + lane;
            int64_t bh;
            if (st < n_stages && stage_rows(a, sc, st, &bh))
                rdy = ld_relaxed_gpu(a.sel_done + bh) >= uint32_t(a.n_tiles);
        }
        // ---- finished attention items: merge the warps' partials ----
        int64_t items[2] = {-1, -1};
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            if (!(sa < n_stages && poll_uniform(&S.mb_item[sa % kPSlots],
                                                uint32_t((sa / kPSlots) & 1))))
                break;
            const int ps = sa % kPSlots;
            const int j = sa * sc.P + sc.c;
            const int64_t bh = j / a.n_seg;
            const int seg = j - int(bh) * a.n_seg;
            float M = -INFINITY;
#pragma unroll
            for (int w = 0; w < kAW; ++w) M = fmaxf(M, S.pslot[ps][w][0]);
            float L = 0.0f, A[4] = {0.0f, 0.0f, 0.0f, 0.0f};
            if (M != -INFINITY) {
#pragma unroll
                for (int w = 0; w < kAW; ++w) {
                    const float mw = S.pslot[ps][w][0];
                    const float wt = mw == -INFINITY ? 0.0f : exp2f(mw - M);
                    L = fmaf(S.pslot[ps][w][1], wt, L);
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        A[i] = fmaf(S.pslot[ps][w][4 + lane + 32 * i], wt, A[i]);
                }
            }
            float *pp = a.part + (bh * a.n_seg + seg) * kPartStride;
#pragma unroll
            for (int i = 0; i < 4; ++i) pp[4 + lane + 32 * i] = A[i];
            if (lane == 0) {
                pp[0] = M;
                pp[1] = L;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&S.mb_item_free[ps]);
            items[k] = bh;
            ++sa;
            progress = true;
        }
        const uint32_t rdy_mask = __ballot_sync(0xffffffffu, rdy);
        // the ready prefix (stages past the end count as ready)
        const int new_a = min(ardy + __ffs(~(rdy_mask & 0xffu) & 0x1ffu) - 1, n_stages);
        const bool newly_ready = new_a > ardy;
        // ---- finished selection tiles ----
        const uint32_t w = ld_acquire_cta(&S.selq_w);
        const uint32_t r0 = uint32_t(sr);
        const int n_heads = int(w - r0);
        if (n_heads > 0) progress = true;
        if (items[0] >= 0 || n_heads > 0 || newly_ready) {
            // everything above, and what the selection warps wrote before
            // handing it over, becomes visible before the counters move; the
            // polled counters act as acquires for what the attention warps
            // read next
            __syncwarp();
            fence_acq_rel_gpu();
            if (newly_ready) {
                progress = true;
                ardy = new_a;
                if (lane == 0) st_release_cta(&S.a_ready, uint32_t(ardy));
            }
            if (lane == 0)
                for (uint32_t e = r0; e < w; ++e) red_add_relaxed_gpu(a.sel_done + S.selq[e % kSelQ], 1u);
            sr += n_heads;
            __syncwarp();
            if (lane == 0) st_release_cta(&S.selq_r, uint32_t(sr));
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                if (items[k] < 0) continue;
                uint32_t old = 0;
                if (lane == 0) old = atom_add_acq_rel_gpu(a.head_cnt + items[k], 1u);
                old = __shfl_sync(0xffffffffu, old, 0);
                if (old + 1u == uint32_t(a.n_seg)) {  // the head's last item: merge it
                    fence_acq_rel_gpu();
                    merge_partials(a.part + items[k] * a.n_seg * kPartStride, a.n_seg,
                                   a.out + items[k] * kD, lane);
                }
            }
        }
        if (progress) {
            t_idle = global_ns();
        } else {
            if (aborted(a, S) || global_ns() - t_idle > a.spin_limit_ns) {
                give_up(a, S);
                break;
            }
            nanosleep_ns(64);
        }
    }
}

// ------------------------------------------------------------- kernel --

__global__ void __maxnreg__(kRegs) fused_select_attend_kernel(FusedArgs a)
{
    extern __shared__ __align__(128) uint8_t smem_raw[];
    FSmem &S = *reinterpret_cast<FSmem *>(smem_raw);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    pdl_trigger();

    Sched sc;
    sc.P = gridDim.x;
    sc.c = blockIdx.x;
    sc.n_sel = a.B * a.H_q * a.n_tiles;
    sc.sel_items = share(sc.n_sel, sc.P, sc.c);
    sc.J = a.B * a.H_q * a.n_seg;
    sc.stages = share(sc.J, sc.P, sc.c);

    if (tid == 0) {
        for (int i = 0; i < kPSlots; ++i) {
            mbar_init(&S.mb_item[i], kAW);
            mbar_init(&S.mb_item_free[i], 1);
        }
        S.selq_w = S.selq_r = 0u;
        S.abort = 0u;
        S.a_ready = 0u;
    }
    __syncthreads();
    pdl_wait();  // distance rows and tile histograms of the scoring kernel

    if (warp < kSW)
        select_role(a, S, sc, tid);
    else if (warp < kPubWarp)
        attend_role(a, S, sc, warp - kSW, lane);
    else
        publisher_role(a, S, sc, lane);
}

}  // namespace

cudaError_t launch_fused(const FusedArgs &a, cudaStream_t s)
{
    const void *fn = reinterpret_cast<const void *>(fused_select_attend_kernel);
    if (cudaError_t e = ensure_smem_attr(fn, sizeof(FSmem))) return e;
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    return launch_pdl(fused_select_attend_kernel, dim3(unsigned(sms)), dim3(kThreads),
                      sizeof(FSmem), s, a);
}

}  // namespace hata
