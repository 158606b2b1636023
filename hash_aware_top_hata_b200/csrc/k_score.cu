// k_score.cu -- Hamming scoring of every cached key code.
//
// HATA review page (arXiv 2506.02572), "What carries the argument": the query
// code is XOR-ed with every cached key code and a popcount reduction gives
// the Hamming score; major comment 1 (Algorithm 3): the top-k runs over
// these 129 possible scores.
//
// Persistent kernel.  Work items are (b, h_kv, group of <= 8 query heads,
// chunk of 4096 tokens); CTA k takes items k, k + gridDim.x, ...  Each item's
// 64 KB of 16-byte codes streams through a 3-deep ring of 16 KB shared-memory
// buffers filled by the bulk-copy engine (cp.async.bulk issued by one
// thread, mbarrier completion), so the code stream is read from HBM exactly
// once per KV head and its latency hides behind the arithmetic of the
// previous sub-block.  Every code is scored against all query heads of its
// group:
//
//   x_w = code_w XOR q_w (w = 0..3)
//   (s, c)    = full-add(x0, x1, x2)    -- bitwise carry-save adder
//   (ones, c2) = half-add(s, x3)
//   dist = popc(ones) + 2 popc(c XOR c2) + 4 popc(c AND c2)
//
// i.e. three population counts instead of four: POPC issues at a quarter of
// the integer rate on sm_100a, and it is what bounds this kernel.
//
// Per query head the kernel writes the u8 distance row (through a
// shared-memory tile and a bulk store; the row stays L2-resident for the
// selection kernel) and a 129-bin histogram per chunk (per-warp shared
// counters), published as a cumulative histogram per chunk plus atomic adds
// into the head's total histogram.
#include "block_scan.cuh"
#include "hata_internal.cuh"
#include "tma.cuh"

namespace hata {
namespace {

constexpr int kWarps = kScoreThreads / 32;
constexpr int kSub = 1024;                    // tokens per staged sub-block (16 KB)
constexpr int kSubsPerChunk = kChunk / kSub;  // 4
constexpr int kRing = 3;
constexpr int kTokPerThread = kSub / kScoreThreads;  // 4

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

struct Item {
    int b, h, z, c;
    int64_t len;
};
static_assert(kChunk % kSub == 0, "sub-blocks tile a chunk");

struct ScoreSmem {
    uint4 codes[kRing][kSub];               // 48 KB ring of staged codes
    uint8_t dist[2][kScoreHeads][kSub];     // 16 KB double-buffered distance tiles
    uint32_t hist[kWarps][kScoreHeads][kBins];
    uint32_t chist[kScoreHeads][kBins];
    uint64_t full[kRing];
};

template <int GB>
__global__ void __launch_bounds__(kScoreThreads, 2) score_kernel(ScoreArgs a)
{
    extern __shared__ __align__(128) uint8_t smem_raw[];
    ScoreSmem &S = *reinterpret_cast<ScoreSmem *>(smem_raw);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    // item -> (b, h_kv, head group, chunk): 32-bit arithmetic, once per item
    auto item_of = [&](int it) {
        Item r;
        r.c = it % int(a.n_chunks);
        int g = it / int(a.n_chunks);
        r.z = g % a.zgroups;
        g /= a.zgroups;
        r.h = g % a.H_kv;
        r.b = g / a.H_kv;
        r.len = clamp_len(__ldg(a.seq_len + r.b), a.max_seq_len, a.n_cap);
        return r;
    };
    // tokens of sub-block s of item r that hold real codes
    auto sub_valid = [&](const Item &r, int s) -> int {
        const int64_t v = r.len - (int64_t(r.c) * kChunk + int64_t(s) * kSub);
        return v <= 0 ? 0 : (v >= kSub ? kSub : int(v));
    };
    // sub-block j of this CTA's sequence into ring slot j % kRing (thread 0)
    auto issue = [&](int j) {
        const Item r = item_of(int(blockIdx.x) + (j / kSubsPerChunk) * int(gridDim.x));
        const int s = j % kSubsPerChunk;
        const int v = sub_valid(r, s);
        uint64_t *bar = &S.full[j % kRing];
        mbar_arrive_expect_tx(bar, uint32_t(v) * 16u);
        if (v > 0) {
            const uint4 *src = reinterpret_cast<const uint4 *>(a.codes) +
                               ((int64_t(r.b) * a.H_kv + r.h) * a.n_cap +
                                int64_t(r.c) * kChunk + int64_t(s) * kSub);
            bulk_g2s(S.codes[j % kRing], src, uint32_t(v) * 16u, bar);
        }
    };

    if (tid == 0) {
        for (int i = 0; i < kRing; ++i) mbar_init(&S.full[i], 1);
        fence_mbar_init();
    }
    for (int i = tid; i < kWarps * kScoreHeads * kBins; i += kScoreThreads)
        (&S.hist[0][0][0])[i] = 0u;
    __syncthreads();

    const int n_items = int(int64_t(a.B) * a.H_kv * a.zgroups * a.n_chunks);
    const int my_items =
        int(blockIdx.x) < n_items ? (n_items - 1 - int(blockIdx.x)) / int(gridDim.x) + 1 : 0;
    const int n_subs = my_items * kSubsPerChunk;
    if (tid == 0)
        for (int j = 0; j < kRing && j < n_subs; ++j) issue(j);

    Item r{};
    int ng = 0;
    size_t bh0 = 0;
    uint4 qc[GB];
    for (int j = 0; j < n_subs; ++j) {
        const int s = j % kSubsPerChunk;
        if (s == 0) {  // a new item: decode it and fetch its query codes once
            r = item_of(int(blockIdx.x) + (j / kSubsPerChunk) * int(gridDim.x));
            const int g0 = r.z * kScoreHeads;
            ng = min(GB, a.G - g0);
            bh0 = size_t(r.b) * a.H_q + size_t(r.h) * a.G + g0;
#pragma unroll
            for (int g = 0; g < GB; ++g)
                qc[g] = g < ng ? reinterpret_cast<const uint4 *>(a.qcodes)[bh0 + g]
                               : make_uint4(0, 0, 0, 0);
        }
        const int v = sub_valid(r, s);

        const bool landed = mbar_wait(&S.full[j % kRing], uint32_t((j / kRing) & 1));
        // the distance tile of sub-block j was last stored by bulk group j-2:
        // let it finish reading (it was issued a whole sub-block ago) before
        // the barrier that releases the tile writes
        if (tid == 0) bulk_wait_read<1>();
        if (__syncthreads_or(!landed)) {
            // a copy never completed: flag it and stop (the wait was bounded)
            if (tid == 0) atomicOr(a.flags + r.b, HATA_FLAG_TIMEOUT);
            break;
        }
        const uint4 *buf = S.codes[j % kRing];
        uint8_t(*tile)[kSub] = S.dist[j & 1];
#pragma unroll
        for (int u = 0; u < kTokPerThread; ++u) {
            const int t = u * kScoreThreads + tid;
            const bool valid = t < v;
            const uint4 cv = valid ? buf[t] : make_uint4(0, 0, 0, 0);
#pragma unroll
            for (int g = 0; g < GB; ++g) {
                if (g < ng) {
                    const int d = hamming128(cv, qc[g]);
                    tile[g][t] = valid ? uint8_t(d) : kDistPad;
                    if (valid) atomicAdd(&S.hist[warp][g][d], 1u);
                }
            }
        }
        fence_async_shared();          // tile writes -> visible to the bulk store
        __syncthreads();
        if (tid == 0) {
            const int64_t off = int64_t(r.c) * kChunk + int64_t(s) * kSub;
            for (int g = 0; g < ng; ++g)
                bulk_s2g(a.dist + (bh0 + g) * a.dist_row + off, tile[g], kSub);
            bulk_commit();
            if (j + kRing < n_subs) issue(j + kRing);
        }

        const int64_t nch = r.len > 0 ? ceil_div(r.len, kChunk) : 1;
        if (s == kSubsPerChunk - 1 && r.c < nch) {
            // ---- chunk done: publish its histogram ----
            for (int i = tid; i < ng * kBins; i += kScoreThreads) {
                const int g = i / kBins, t = i % kBins;
                uint32_t sum = 0;
#pragma unroll
                for (int w = 0; w < kWarps; ++w) {
                    sum += S.hist[w][g][t];
                    S.hist[w][g][t] = 0u;
                }
                S.chist[g][t] = sum;
            }
            __syncthreads();
            if (warp < ng) {
                const int g = warp;
                const size_t bh = bh0 + g;
                uint32_t vv[5];
                uint32_t run = 0;
#pragma unroll
                for (int e = 0; e < 5; ++e) {
                    const int t = lane * 5 + e;
                    vv[e] = t < kBins ? S.chist[g][t] : 0u;
                    run += vv[e];
                }
                uint32_t acc = uint32_t(warp_inclusive_scan(int(run))) - run;
                uint32_t *cp = a.cum + (bh * a.n_chunks + r.c) * kCumStride;
#pragma unroll
                for (int e = 0; e < 5; ++e) {
                    const int t = lane * 5 + e;
                    acc += vv[e];
                    if (t < kBins) {
                        cp[t] = acc;
                        if (vv[e]) atomicAdd(a.hist_total + bh * kHistStride + t, vv[e]);
                    }
                }
            }
            // chist is next rewritten only after four more sub-blocks, each
            // closed by a __syncthreads
        }
    }
    if (tid == 0) bulk_wait_all();
}

template <int GB>
cudaError_t launch_score_t(const ScoreArgs &a, cudaStream_t s)
{
    const void *fn = reinterpret_cast<const void *>(score_kernel<GB>);
    if (cudaError_t e = ensure_smem_attr(fn, sizeof(ScoreSmem))) return e;
    int dev = 0, sms = 0, per_sm = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess)
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, score_kernel<GB>,
                                                          kScoreThreads, sizeof(ScoreSmem));
    if (e != cudaSuccess) return e;
    const int64_t cap = int64_t(per_sm > 0 ? per_sm : 1) * sms;
    const int64_t items = int64_t(a.B) * a.H_kv * a.zgroups * a.n_chunks;
    score_kernel<GB><<<unsigned(items < cap ? items : cap), kScoreThreads, sizeof(ScoreSmem), s>>>(a);
    return cudaGetLastError();
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
