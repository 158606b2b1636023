// k_hash.cu -- the HATA hash h(x) = sign(x W_H) on sm_100a.
//
// HATA review page (arXiv 2506.02572): "Assumptions & free parameters"
// (h(x) = sign(x W_H), per-head W_H, rbit = 128), "What carries the
// argument" (queries and keys are hashed; the key codes are cached) and the
// Figure 2 caption (Algorithm 1: HashEncode(K) fills the code cache, rbit/32
// words per token).
//
// Every code bit j is the fp32 chain acc = fmaf(x_i, W[i][j], acc), i = 0..127
// ascending, then acc > 0.  The chain order is fixed, so codes are
// reproducible bit for bit by any implementation that follows the same
// order (the CPU oracle does).  r = 128 bits (the page's width), or 32 / 64 /
// 256 (the other widths of its ablation): r/32 code words per token.
//
// Two kernels: the prefill hash (register-blocked over 8 rows per warp, the
// head's W_H in shared memory) for hata_hash_keys, and the decode prep
// (one 32-bit code word of 8 rows per CTA) that hashes the step's queries,
// appends the new key's code (and optionally its K/V rows) and clears the
// per-step counters the scoring kernel accumulates into.  The projection
// is 16K FMAs per row at r = 128: on the FP32 pipes, not the tensor cores,
// whose accumulation order is unspecified and would break bit-exact codes.
#include "hata_internal.cuh"
#include "async_copy.cuh"

namespace hata {
namespace {


template <bool BF16>
__device__ __forceinline__ float load_x(const void *base, int64_t i)
{
    if (BF16) {
        const uint16_t u = reinterpret_cast<const uint16_t *>(base)[i];
        return __uint_as_float(uint32_t(u) << 16);
    }
    return reinterpret_cast<const float *>(base)[i];
}

// -------------------------------------------------------------- prefill --
// Register-blocked: a CTA stages its head's W_H in shared memory once and
// walks its rows in passes of kPfPass rows; warp w takes 8 rows of a pass,
// lane l the output bits 4l..4l+3 of each, so a lane holds 32 accumulators,
// each the fp32 chain acc = fmaf(x_i, W[i][j], acc) over i = 0..127 in order.
// Per step i a lane reads its 4 W values (one 16-byte load; the warp reads
// W's row i contiguously) and the 8 row values (two broadcast loads), then
// issues 16 paired FMAs over row pairs: fma.rn.f32x2 performs two IEEE fp32
// fused multiply-adds, each rounded to nearest, so every chain is the one
// the scalar form computes (it halves the issue slots, not the FMA work).
// 96 KB of shared memory: two CTAs, 16 warps, per SM.
constexpr int kPfWarps = 8;
constexpr int kPfThreads = 32 * kPfWarps;
constexpr int kPfRows = 8;                   // rows per warp and pass
constexpr int kPfPass = kPfWarps * kPfRows;  // rows per CTA and pass
constexpr int kPfRowsPerCta = 16 * kPfPass;  // 1024 rows per CTA

template <int R>
struct PfSmem {
    float W[kD * R];                         // this head's W_H, [i][j]
    float x[kPfWarps][kD][kPfRows];          // each warp's rows, [i][row]
};

// acc (two fp32 chains) += x (pair) * w (pair), element by element
__device__ __forceinline__ void ffma2(uint64_t &acc, uint64_t x, uint64_t w)
{
    asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(acc) : "l"(x), "l"(w));
}

__device__ __forceinline__ uint64_t dup2(float v)
{
    uint64_t r;
    asm("mov.b64 %0, {%1, %1};" : "=l"(r) : "f"(v));
    return r;
}

template <bool BF16, int R>
__global__ void __launch_bounds__(kPfThreads, 2) hash_prefill_kernel(const void *__restrict__ K,
                                                                    KStrides ks, int64_t n_cap,
                                                                    const float *__restrict__ W,
                                                                    uint32_t *__restrict__ codes,
                                                                    int H_kv, int64_t pos0, int64_t n)
{
    extern __shared__ __align__(16) uint8_t pf_raw[];
    PfSmem<R> &S = *reinterpret_cast<PfSmem<R> *>(pf_raw);
    constexpr int kBL = R / 32, kLPW = 32 / kBL;  // bits per lane, lanes per code word
    const int h = blockIdx.y, b = blockIdx.z, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t g_begin = int64_t(blockIdx.x) * kPfRowsPerCta;
    const int64_t g_end = min(g_begin + kPfRowsPerCta, n);
    const int64_t slab = (int64_t(b) * H_kv + h) * n_cap + pos0;  // code row of row 0
    const int64_t kbase = int64_t(b) * ks.b + int64_t(h) * ks.h + pos0 * ks.n;  // K element of row 0
    {
        const float *Wh = W + size_t(h) * kD * R;
        const uint32_t base = smem_addr(S.W);
        for (int c = tid; c < kD * R / 4; c += kPfThreads)
            cp_async16_zfill(base + 16u * c, Wh + 4 * c, 16u);
        cp_async_commit();
    }
    // staging: lane l holds row (l & 7) of its warp at steps i = 4k + (l >> 3)
    // (eight lanes write one 32-byte run); the next pass's values are loaded
    // into registers while a pass computes
    const int sr = lane & 7, si = lane >> 3;
    float xv[kD / 4];
    auto fetch = [&](int64_t g0) {
        const int64_t t = g0 + warp * kPfRows + sr;
        const bool ok = t < g_end;
#pragma unroll
        for (int k = 0; k < kD / 4; ++k) xv[k] = ok ? load_x<BF16>(K, kbase + t * ks.n + 4 * k + si) : 0.0f;
    };
    fetch(g_begin);
    for (int64_t g0 = g_begin; g0 < g_end; g0 += kPfPass) {
        __syncthreads();  // the previous pass is done with the rows
#pragma unroll
        for (int k = 0; k < kD / 4; ++k) S.x[warp][4 * k + si][sr] = xv[k];
        cp_async_wait<0>();
        __syncthreads();
        if (g0 + kPfPass < g_end) fetch(g0 + kPfPass);
        uint64_t acc[kPfRows / 2][kBL];  // [row pair][column]
#pragma unroll
        for (int p = 0; p < kPfRows / 2; ++p)
#pragma unroll
            for (int c = 0; c < kBL; ++c) acc[p][c] = 0ull;
        const float *wrow = S.W + kBL * lane;  // W[0][kBL l ..]
        const ulonglong2 *xrow = reinterpret_cast<const ulonglong2 *>(&S.x[warp][0][0]);
#pragma unroll 4
        for (int i = 0; i < kD; ++i) {
            // this lane's kBL values of W's row i (4- to 32-byte loads)
            float wv[kBL];
            if constexpr (kBL == 8) {
                const float4 w0 = *reinterpret_cast<const float4 *>(wrow + i * R);
                const float4 w1 = *reinterpret_cast<const float4 *>(wrow + i * R + 4);
                wv[0] = w0.x, wv[1] = w0.y, wv[2] = w0.z, wv[3] = w0.w;
                wv[4] = w1.x, wv[5] = w1.y, wv[6] = w1.z, wv[7] = w1.w;
            } else if constexpr (kBL == 4) {
                const float4 w = *reinterpret_cast<const float4 *>(wrow + i * R);
                wv[0] = w.x, wv[1] = w.y, wv[2] = w.z, wv[3] = w.w;
            } else if constexpr (kBL == 2) {
                const float2 w = *reinterpret_cast<const float2 *>(wrow + i * R);
                wv[0] = w.x, wv[1] = w.y;
            } else {
                wv[0] = wrow[i * R];
            }
            const ulonglong2 xa = xrow[i * 2], xb = xrow[i * 2 + 1];  // rows (0,1) (2,3) | (4,5) (6,7)
            const uint64_t xp[4] = {xa.x, xa.y, xb.x, xb.y};
#pragma unroll
            for (int c = 0; c < kBL; ++c) {
                const uint64_t w2 = dup2(wv[c]);
#pragma unroll
                for (int p = 0; p < kPfRows / 2; ++p) ffma2(acc[p][c], xp[p], w2);
            }
        }
        // bits kBL l .. kBL l + kBL - 1 of each row -> word l / kLPW, bit kBL (l % kLPW) + c
#pragma unroll
        for (int r = 0; r < kPfRows; ++r) {
            const int p = r >> 1, sh = 32 * (r & 1);
            uint32_t v = 0;
#pragma unroll
            for (int c = 0; c < kBL; ++c)
                v |= (__uint_as_float(uint32_t(acc[p][c] >> sh)) > 0.0f ? 1u : 0u) << c;
            v <<= kBL * (lane % kLPW);
#pragma unroll
            for (int o = 1; o < kLPW; o <<= 1) v |= __shfl_xor_sync(0xffffffffu, v, o);
            const int64_t t = g0 + warp * kPfRows + r;
            if (lane % kLPW == 0 && t < g_end) codes[(slab + t) * (R / 32) + lane / kLPW] = v;
        }
    }
}

// --------------------------------------------------------- decode prep --
// Rows of KV head h: B*G query rows (b-major), then B appended-key rows.
// A CTA takes kPrepRowsCta rows of one head and one 32-bit word of their
// codes: warp = row, lane = bit 32 cb + lane (cb = blockIdx.z), so the CTA
// stages only its 32 columns of the head's W_H (16 KB, asynchronous 16-byte
// copies by all threads) next to its rows, and a warp ballot gives the
// word.  Every step of a chain reads its two operands from shared memory at
// addresses known in advance: the loads run ahead of the dependent FMAs
// instead of exposing their latency at each of the 128 steps.  The side
// jobs of a row (the device copy of q, the appended K/V rows, the flags)
// fall to the CTAs of word 0; the histogram rows are cleared by all words.
constexpr int kPrepRowsCta = 8;
constexpr int kPrepThreads = 32 * kPrepRowsCta;

template <bool BF16, int R>
__global__ void __launch_bounds__(kPrepThreads) prep_kernel(PrepArgs a)
{
    pdl_trigger();  // the scoring kernel's setup (step inputs only) may start now
    const int h = blockIdx.y, cb = blockIdx.z;
    const int r = threadIdx.x >> 5, lane = threadIdx.x & 31, j = 32 * cb + lane;
    const int nq = a.q ? a.B * a.G : 0;
    const int nk = a.k_new ? a.B : 0;
    const int rows = nq + nk;
    const int r0 = blockIdx.x * kPrepRowsCta;
    const int row = r0 + r;

    if (a.ws_header && blockIdx.x == 0 && h == 0 && cb == 0 && threadIdx.x == 0) {
        a.ws_header[0] = kWsMagic;
        a.ws_header[1] = uint32_t(a.B);
    }
    if (r0 >= rows) return;

    __shared__ __align__(16) float ws[kD][32];             // columns 32 cb .. of W_H
    __shared__ __align__(16) float xs[kPrepRowsCta][kD];   // the rows
    {
        const float *Wh = a.W + size_t(h) * kD * R + 32 * cb;
        const uint32_t base = smem_addr(&ws[0][0]);
        for (int c = threadIdx.x; c < kD * 8; c += kPrepThreads)  // row c / 8, piece c % 8
            cp_async16_zfill(base + 16u * c, Wh + size_t(c >> 3) * R + 4 * (c & 7), 16u);
        cp_async_commit();
    }

    // the row itself: its warp reads it with 16-byte (q, fp32 keys) or
    // 8-byte (bf16 keys) loads -- q and k_new may be host memory, where few
    // wide requests cost much less than many narrow ones
    if (row < rows) {
        float4 v;
        if (row < nq) {
            const size_t bh = size_t(row / a.G) * a.H_q + h * a.G + row % a.G;
            v = reinterpret_cast<const float4 *>(a.q + bh * kD)[lane];
            if (a.q_copy && cb == 0) reinterpret_cast<float4 *>(a.q_copy + bh * kD)[lane] = v;
        } else {
            const int64_t e0 = (int64_t(row - nq) * a.H_kv + h) * kD;
            if (BF16) {
                const uint2 u = reinterpret_cast<const uint2 *>(static_cast<const uint16_t *>(a.k_new) + e0)[lane];
                v = make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xffff0000u),
                                __uint_as_float(u.y << 16), __uint_as_float(u.y & 0xffff0000u));
            } else {
                v = reinterpret_cast<const float4 *>(static_cast<const float *>(a.k_new) + e0)[lane];
            }
        }
        reinterpret_cast<float4 *>(&xs[r][0])[lane] = v;
    }
    if (row < nq) {
        const int b = row / a.G, g = row % a.G, hq = h * a.G + g;
        const size_t bh = size_t(b) * a.H_q + hq;
        if (a.hist)
            for (int64_t t = j; t < a.hist_row_words; t += R) a.hist[bh * a.hist_row_words + t] = 0u;
        if (a.sync && cb == 0 && lane == 0) {
            // the fused step's counters: selection tiles done and attention
            // items published of this head
            const size_t BH = size_t(a.B) * a.H_q;
            a.sync[bh] = 0u;
            a.sync[BH + bh] = 0u;
            if (bh == 0) a.sync[2 * BH] = 0u;  // the step's abort word
        }
        if (a.flags && h == 0 && g == 0 && cb == 0 && lane == 0) {
            const int64_t sl = a.seq_len[b];
            uint32_t f = 0;
            if (sl < 0 || sl > a.max_seq_len || sl > a.n_cap) f |= HATA_FLAG_SEQ_LEN_RANGE;
            if (a.k_new && (sl - 1 < 0 || sl - 1 >= a.n_cap)) f |= HATA_FLAG_POS_RANGE;
            a.flags[b] = f;
        }
    }
    cp_async_wait<0>();
    __syncthreads();
    if (row >= rows) return;  // warp-uniform; no barrier follows

    // the fixed-order chain acc = fmaf(x_i, W[i][j], acc), i = 0..127
    // (operands of block i0 + 16 are loaded before block i0 is multiplied in)
    constexpr int kBlk = 16;
    const float4 *xr = reinterpret_cast<const float4 *>(&xs[r][0]);
    float xa[kBlk], wa[kBlk], xb[kBlk], wb[kBlk];
    auto fetch = [&](int i0, float (&xv)[kBlk], float (&wv)[kBlk]) {
#pragma unroll
        for (int k = 0; k < kBlk / 4; ++k) {
            const float4 v = xr[i0 / 4 + k];
            xv[4 * k] = v.x, xv[4 * k + 1] = v.y, xv[4 * k + 2] = v.z, xv[4 * k + 3] = v.w;
        }
#pragma unroll
        for (int k = 0; k < kBlk; ++k) wv[k] = ws[i0 + k][lane];
    };
    float acc = 0.0f;
    fetch(0, xa, wa);
#pragma unroll
    for (int i0 = 0; i0 < kD; i0 += 2 * kBlk) {
        fetch(i0 + kBlk, xb, wb);
#pragma unroll
        for (int k = 0; k < kBlk; ++k) acc = __fmaf_rn(xa[k], wa[k], acc);
        if (i0 + 2 * kBlk < kD) fetch(i0 + 2 * kBlk, xa, wa);
#pragma unroll
        for (int k = 0; k < kBlk; ++k) acc = __fmaf_rn(xb[k], wb[k], acc);
    }
    const uint32_t word = __ballot_sync(0xffffffffu, acc > 0.0f);

    if (row < nq) {
        if (lane == 0) {
            const int b = row / a.G, g = row % a.G;
            const size_t bh = size_t(b) * a.H_q + h * a.G + g;
            a.q_out[bh * (R / 32) + cb] = word;
        }
    } else {
        const int b = row - nq;
        const int64_t pos = a.pos ? int64_t(a.pos[b]) : int64_t(a.seq_len[b]) - 1;
        if (pos >= 0 && pos < a.n_cap) {
            const int64_t crow = (int64_t(b) * a.H_kv + h) * a.n_cap + pos;
            if (lane == 0) a.codes[crow * (R / 32) + cb] = word;
            if (a.v_new && cb == 0) {
                // K from the staged row (a bf16 key is the upper half of its
                // fp32 widening: exact); V copied by the row's warp
#pragma unroll
                for (int e = lane; e < kD; e += 32) {
                    const float xk = xs[r][e];
                    if (BF16)
                        static_cast<uint16_t *>(a.K)[crow * kD + e] =
                            uint16_t(__float_as_uint(xk) >> 16);
                    else
                        static_cast<float *>(a.K)[crow * kD + e] = xk;
                }
                const int64_t e0 = (int64_t(b) * a.H_kv + h) * kD;
                if (BF16)
                    reinterpret_cast<uint2 *>(static_cast<uint16_t *>(a.V) + crow * kD)[lane] =
                        reinterpret_cast<const uint2 *>(static_cast<const uint16_t *>(a.v_new) + e0)[lane];
                else
                    reinterpret_cast<float4 *>(static_cast<float *>(a.V) + crow * kD)[lane] =
                        reinterpret_cast<const float4 *>(static_cast<const float *>(a.v_new) + e0)[lane];
            }
        } else if (a.err_word && cb == 0 && lane == 0) {
            atomicOr(a.err_word, HATA_FLAG_POS_RANGE);
        }
    }
}

}  // namespace

template <bool BF16, int R>
cudaError_t launch_hash_prefill_t(const void *K, KStrides ks, int64_t n_cap, const float *W,
                                  uint32_t *codes, int B, int H_kv, int64_t pos0, int64_t n,
                                  cudaStream_t s)
{
    constexpr size_t kSmem = sizeof(PfSmem<R>);
    if (cudaError_t e = ensure_smem_attr(
            reinterpret_cast<const void *>(hash_prefill_kernel<BF16, R>), kSmem))
        return e;
    const dim3 grid(unsigned(ceil_div(n, kPfRowsPerCta)), unsigned(H_kv), unsigned(B));
    hash_prefill_kernel<BF16, R><<<grid, kPfThreads, kSmem, s>>>(K, ks, n_cap, W, codes, H_kv, pos0, n);
    return cudaGetLastError();
}

cudaError_t launch_hash_prefill(const void *K, bool bf16, KStrides ks, int64_t n_cap,
                                const float *W, uint32_t *codes, int B, int H_kv, int64_t pos0,
                                int64_t n, int words, cudaStream_t s)
{
    switch (words * 2 + (bf16 ? 1 : 0)) {
    case 16 + 1: return launch_hash_prefill_t<true, 256>(K, ks, n_cap, W, codes, B, H_kv, pos0, n, s);
    case 16: return launch_hash_prefill_t<false, 256>(K, ks, n_cap, W, codes, B, H_kv, pos0, n, s);
    case 8 + 1: return launch_hash_prefill_t<true, 128>(K, ks, n_cap, W, codes, B, H_kv, pos0, n, s);
    case 8: return launch_hash_prefill_t<false, 128>(K, ks, n_cap, W, codes, B, H_kv, pos0, n, s);
    case 4 + 1: return launch_hash_prefill_t<true, 64>(K, ks, n_cap, W, codes, B, H_kv, pos0, n, s);
    case 4: return launch_hash_prefill_t<false, 64>(K, ks, n_cap, W, codes, B, H_kv, pos0, n, s);
    case 2 + 1: return launch_hash_prefill_t<true, 32>(K, ks, n_cap, W, codes, B, H_kv, pos0, n, s);
    case 2: return launch_hash_prefill_t<false, 32>(K, ks, n_cap, W, codes, B, H_kv, pos0, n, s);
    default: return cudaErrorInvalidValue;
    }
}

template <bool BF16, int R>
cudaError_t launch_prep_t(const PrepArgs &a, int rows_per_head, cudaStream_t s)
{
    const dim3 grid(unsigned(ceil_div(rows_per_head, kPrepRowsCta)), unsigned(a.H_kv),
                    unsigned(R / 32));
    prep_kernel<BF16, R><<<grid, kPrepThreads, 0, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_prep(const PrepArgs &a, int rows_per_head, cudaStream_t s)
{
    switch (a.words * 2 + (a.kv_bf16 ? 1 : 0)) {
    case 16 + 1: return launch_prep_t<true, 256>(a, rows_per_head, s);
    case 16: return launch_prep_t<false, 256>(a, rows_per_head, s);
    case 8 + 1: return launch_prep_t<true, 128>(a, rows_per_head, s);
    case 8: return launch_prep_t<false, 128>(a, rows_per_head, s);
    case 4 + 1: return launch_prep_t<true, 64>(a, rows_per_head, s);
    case 4: return launch_prep_t<false, 64>(a, rows_per_head, s);
    case 2 + 1: return launch_prep_t<true, 32>(a, rows_per_head, s);
    case 2: return launch_prep_t<false, 32>(a, rows_per_head, s);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace hata
