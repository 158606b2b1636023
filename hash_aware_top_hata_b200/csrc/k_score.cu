// k_score.cu -- Hamming scoring of every cached key code and the top-k plan.
//
// HATA review page (arXiv 2506.02572): "What carries the argument" (the query
// code is XOR-ed with all key codes; popcount / reduction gives the Hamming
// score) and major comment 1 (Algorithm 3: top-k over the 129 possible
// scores; the page leaves the boundary bucket open -- here it goes to the
// lower token index).
//
// Grid: (chunk of 4096 tokens, b * H_kv + h_kv, group of <= 8 query heads).
// Each CTA streams its chunk of 16-byte codes once (coalesced 128-bit loads,
// evict-first) and scores it against the codes of all query heads of the KV
// group that it holds in registers, so the code stream is read once per KV
// head, not once per query head.  Per query head it writes the u8 distance
// row (kept for the selection pass; it stays in L2) and a 129-bin histogram
// of the chunk (per-warp shared-memory counters), published as a
// cumulative histogram per chunk plus atomic adds into the head's total.
//
// The last CTA of a (b, h_kv, group) to finish -- found with a fence and an
// arrival counter, no waiting -- turns the totals into the selection plan:
//   T      = smallest distance with #(dist <= T) >= k_eff, k_eff = min(k, len)
//   n_less = #(dist < T), ties = k_eff - n_less taken from the T bucket
//   per chunk c: take_c = the part of the `ties` lowest-index T-keys lying in
//   chunk c, and off_c = the output slot of chunk c's first selected key.
// The selection kernel then needs no global sort and no second pass.
#include "block_scan.cuh"
#include "hata_internal.cuh"

namespace hata {
namespace {

constexpr int kWarps = kScoreThreads / 32;
constexpr int kPerThread = kChunk / kScoreThreads;  // 16 tokens per thread
constexpr int kLoadBatch = 8;

__device__ __forceinline__ int64_t clamp_len(int32_t sl, int64_t max_len, int64_t n_cap)
{
    int64_t l = sl < 0 ? 0 : sl;
    l = l < max_len ? l : max_len;
    return l < n_cap ? l : n_cap;
}

__device__ __forceinline__ int hamming128(const uint4 &a, const uint4 &b)
{
    return __popc(a.x ^ b.x) + __popc(a.y ^ b.y) + __popc(a.z ^ b.z) + __popc(a.w ^ b.w);
}

template <int GB>
__global__ void __launch_bounds__(kScoreThreads) score_kernel(ScoreArgs a)
{
    const int c = blockIdx.x;
    const int b = blockIdx.y / a.H_kv, h = blockIdx.y % a.H_kv;
    const int z = blockIdx.z;
    const int g0 = z * kScoreHeads;
    const int ng = min(GB, a.G - g0);
    const int64_t len = clamp_len(a.seq_len[b], a.max_seq_len, a.n_cap);
    const int64_t nch = len > 0 ? ceil_div(len, kChunk) : 1;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const size_t bh0 = size_t(b) * a.H_q + size_t(h) * a.G + g0;  // first query head
    if (c >= nch) {
        // chunk entirely past seq_len: only its distance padding
        static_assert(kChunk == 16 * kScoreThreads, "one 16-byte store per thread per head");
        const uint4 pad = make_uint4(0xffffffffu, 0xffffffffu, 0xffffffffu, 0xffffffffu);
        for (int g = 0; g < ng; ++g)
            reinterpret_cast<uint4 *>(a.dist + (bh0 + g) * a.dist_row + int64_t(c) * kChunk)[tid] = pad;
        return;
    }

    __shared__ uint32_t hist_s[kWarps][GB][kBins];
    __shared__ uint32_t chist[GB][kBins];
    __shared__ int scan_s[kWarps + 1];
    __shared__ int s_last;
    __shared__ uint32_t tot_s[kBins];
    __shared__ int s_T, s_ties;

    for (int i = tid; i < kWarps * GB * kBins; i += kScoreThreads)
        (&hist_s[0][0][0])[i] = 0u;

    uint4 qc[GB];
#pragma unroll
    for (int g = 0; g < GB; ++g)
        qc[g] = g < ng ? reinterpret_cast<const uint4 *>(a.qcodes)[bh0 + g] : make_uint4(0, 0, 0, 0);
    __syncthreads();

    const int64_t n0 = int64_t(c) * kChunk;
    const uint4 *crow = reinterpret_cast<const uint4 *>(a.codes) +
                        (int64_t(b) * a.H_kv + h) * a.n_cap;
    uint8_t *drow = a.dist + bh0 * a.dist_row;

#pragma unroll
    for (int m0 = 0; m0 < kPerThread; m0 += kLoadBatch) {
        uint4 cv[kLoadBatch];
#pragma unroll
        for (int u = 0; u < kLoadBatch; ++u) {
            const int64_t n = n0 + int64_t(m0 + u) * kScoreThreads + tid;
            cv[u] = n < len ? __ldcs(crow + n) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < kLoadBatch; ++u) {
            const int64_t n = n0 + int64_t(m0 + u) * kScoreThreads + tid;
            const bool valid = n < len;
#pragma unroll
            for (int g = 0; g < GB; ++g) {
                if (g < ng) {
                    const int d = hamming128(cv[u], qc[g]);
                    drow[g * a.dist_row + n] = valid ? uint8_t(d) : kDistPad;
                    if (valid) atomicAdd(&hist_s[warp][g][d], 1u);
                }
            }
        }
    }
    __syncthreads();

    for (int i = tid; i < ng * kBins; i += kScoreThreads) {
        const int g = i / kBins, t = i % kBins;
        uint32_t s = 0;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) s += hist_s[w][g][t];
        chist[g][t] = s;
    }
    __syncthreads();

    // Cumulative histogram of this chunk, one warp per query head; lane L owns
    // bins 5L .. 5L+4.
    if (warp < ng) {
        const int g = warp;
        const size_t bh = bh0 + g;
        uint32_t v[5];
        uint32_t run = 0;
#pragma unroll
        for (int e = 0; e < 5; ++e) {
            const int t = lane * 5 + e;
            v[e] = t < kBins ? chist[g][t] : 0u;
            run += v[e];
        }
        const uint32_t before = uint32_t(warp_inclusive_scan(int(run))) - run;
        uint32_t *cp = a.cum + (bh * a.n_chunks + c) * kCumStride;
        uint32_t acc = before;
#pragma unroll
        for (int e = 0; e < 5; ++e) {
            const int t = lane * 5 + e;
            acc += v[e];
            if (t < kBins) {
                cp[t] = acc;
                if (v[e]) atomicAdd(a.hist_total + bh * kHistStride + t, v[e]);
            }
        }
    }
    __threadfence();
    __syncthreads();
    if (tid == 0) {
        const uint32_t prev =
            atomicAdd(a.cnt_score + (size_t(blockIdx.y) * a.zgroups + z), 1u);
        s_last = prev == uint32_t(nch - 1);
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();

    // ---- plan (last CTA of this (b, h_kv, group)) ----
    const int k_eff = int(int64_t(a.topk) < len ? int64_t(a.topk) : len);
    for (int g = 0; g < ng; ++g) {
        const size_t bh = bh0 + g;
        for (int t = tid; t < kBins; t += kScoreThreads)
            tot_s[t] = __ldcg(a.hist_total + bh * kHistStride + t);
        __syncthreads();
        if (warp == 0) {
            uint32_t v[5];
            uint32_t run = 0;
#pragma unroll
            for (int e = 0; e < 5; ++e) {
                const int t = lane * 5 + e;
                v[e] = t < kBins ? tot_s[t] : 0u;
                run += v[e];
            }
            uint32_t acc = uint32_t(warp_inclusive_scan(int(run))) - run;
            int T = -1;
            uint32_t less_at_T = 0;
#pragma unroll
            for (int e = 0; e < 5; ++e) {
                const int t = lane * 5 + e;
                if (t < kBins && T < 0 && acc + v[e] >= uint32_t(k_eff)) {
                    T = t;
                    less_at_T = acc;
                }
                acc += v[e];
            }
            // cum is monotone, so the lowest lane that found a bin holds T
            const unsigned found = __ballot_sync(0xffffffffu, T >= 0);
            const int src = found ? __ffs(int(found)) - 1 : 0;
            int Tf = __shfl_sync(0xffffffffu, T, src);
            const int nless = __shfl_sync(0xffffffffu, int(less_at_T), src);
            if (!found || k_eff <= 0) Tf = -1;
            if (lane == 0) {
                PlanHead ph;
                ph.T = Tf;
                ph.k_eff = Tf >= 0 ? k_eff : 0;
                ph.n_less = Tf >= 0 ? nless : 0;
                ph.ties = Tf >= 0 ? k_eff - nless : 0;
                a.plan_head[bh] = ph;
                s_T = Tf;
                s_ties = ph.ties;
            }
        }
        __syncthreads();
        const int T = s_T, ties = s_ties;
        int carry_ties = 0, carry_sel = 0;
        for (int64_t cb = 0; cb < nch; cb += kScoreThreads) {
            const int64_t cc = cb + tid;
            int less = 0, tie = 0;
            if (cc < nch && T >= 0) {
                const uint32_t *cp = a.cum + (bh * a.n_chunks + cc) * kCumStride;
                less = T > 0 ? int(__ldcg(cp + T - 1)) : 0;
                tie = int(__ldcg(cp + T)) - less;
            }
            int tot_tie, tot_sel;
            const int P = block_exclusive_scan<kScoreThreads>(tie, scan_s, &tot_tie) + carry_ties;
            const int take = max(0, min(ties - P, tie));
            const int off =
                block_exclusive_scan<kScoreThreads>(less + take, scan_s, &tot_sel) + carry_sel;
            if (cc < nch) {
                PlanChunk pc;
                pc.off = off;
                pc.take = take;
                a.plan_chunk[bh * a.n_chunks + cc] = pc;
            }
            carry_ties += tot_tie;
            carry_sel += tot_sel;
        }
        if (a.sel_idx)
            for (int i = k_eff + tid; i < a.topk; i += kScoreThreads)
                a.sel_idx[bh * a.topk + i] = -1;
        __syncthreads();
    }
}

}  // namespace

cudaError_t launch_score(const ScoreArgs &a, cudaStream_t s)
{
    const dim3 grid(unsigned(a.n_chunks), unsigned(a.B * a.H_kv), unsigned(a.zgroups));
    const int gb = a.G < kScoreHeads ? a.G : kScoreHeads;
    switch (gb) {
    case 1: score_kernel<1><<<grid, kScoreThreads, 0, s>>>(a); break;
    case 2: score_kernel<2><<<grid, kScoreThreads, 0, s>>>(a); break;
    case 3: score_kernel<3><<<grid, kScoreThreads, 0, s>>>(a); break;
    case 4: score_kernel<4><<<grid, kScoreThreads, 0, s>>>(a); break;
    case 5: score_kernel<5><<<grid, kScoreThreads, 0, s>>>(a); break;
    case 6: score_kernel<6><<<grid, kScoreThreads, 0, s>>>(a); break;
    case 7: score_kernel<7><<<grid, kScoreThreads, 0, s>>>(a); break;
    default: score_kernel<8><<<grid, kScoreThreads, 0, s>>>(a); break;
    }
    return cudaGetLastError();
}

}  // namespace hata
