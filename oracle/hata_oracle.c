/*
 * hata_oracle.c -- plain, slow, single-threaded CPU statement of the HATA
 * decode-step path.  TEST INFRASTRUCTURE ONLY: it exists so that the CUDA
 * library can be checked against it.  Only tests/, __graft_entry__.smoke()
 * and bench.py's cpu_baseline / reference legs may load it.  It shares no
 * code, header, table or helper with the CUDA library under
 * hash_aware_top_hata_b200/ and includes nothing from it.
 *
 * Source of every step: the Pith review page of "HATA: Trainable and
 * Hardware-Efficient Hash-Aware Top-k Attention for Scalable Large Model
 * Inference" (arXiv 2506.02572):
 *   - "What carries the argument": a per-head projection x W_H gives r = 128
 *     bits; a query code is XOR-ed with every cached key code and a popcount
 *     gives the Hamming score; the top-k keys feed attention.
 *   - "Assumptions & free parameters": the inference hash is h(x)=sign(x W_H),
 *     rbit = 128.
 *   - Figure 2 caption (Algorithm 1, prefill): HashEncode(K) fills the key
 *     code cache, which holds rbit/32 32-bit words per token.
 *   - Referee report, major comment 1 (Algorithm 3): the top-k runs over
 *     Hamming scores that take only rbit+1 distinct values; the paper leaves
 *     the choice inside the boundary bucket open.
 *
 * Readings taken where the page is silent:
 *   - bit j of a code is 1 iff the projection is > +0 (zero, -0 and NaN give 0);
 *   - the projection of bit j is the fp32 chain acc = fma(x_i, W[i][j], acc)
 *     over i = 0..d-1 ascending, starting from acc = +0 (the same precision and
 *     order the GPU kernel uses, so that both sides take the same decision);
 *   - W_H is stored [d][r] row-major (x is a row vector, h = sign(x W_H));
 *   - bit j lives in word j/32 at bit position j%32 (least significant first);
 *   - "top-k" means the k smallest Hamming distances; ties in the boundary
 *     bucket go to the lower token index; the selected indices are reported in
 *     ascending token order; when k >= n every key is selected;
 *   - attention over the selected keys is exact softmax attention, computed
 *     here in fp64 from the stored (bf16 or fp32) K and V values;
 *   - attention over an empty key set returns the zero vector.
 *
 * Build: gcc -O3 -ffp-contract=off -fno-fast-math -shared -fPIC, plus -mfma
 * where the host CPU has it (see __init__.py).  fmaf() is the correctly
 * rounded C99 fused multiply-add with or without -mfma.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_DT_BF16 0
#define ORACLE_DT_F32 1

/* bf16 is the upper half of an IEEE binary32: widening is exact. */
static float widen_bf16(uint16_t h)
{
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

static float load_elem(const void *base, int dtype, int64_t i)
{
    if (dtype == ORACLE_DT_BF16)
        return widen_bf16(((const uint16_t *)base)[i]);
    return ((const float *)base)[i];
}

/* ---------------------------------------------------------------- hash ---
 * h(x) = sign(x W_H): one bit per column j of W_H. */
void oracle_hash_f32(const float *x, const float *W, int d, int r, uint32_t *code)
{
    /* acc[j] is bit j's projection; every acc[j] runs its own chain over
     * i = 0, 1, ..., d-1 (the loops are nested i-outer only so that the r
     * independent chains advance side by side). */
    float *acc = (float *)malloc(sizeof(float) * (size_t)r);
    for (int j = 0; j < r; ++j)
        acc[j] = 0.0f;
    for (int i = 0; i < d; ++i)
        for (int j = 0; j < r; ++j)
            acc[j] = fmaf(x[i], W[(int64_t)i * r + j], acc[j]);
    for (int w = 0; w < r / 32; ++w)
        code[w] = 0u;
    for (int j = 0; j < r; ++j)
        if (acc[j] > 0.0f)
            code[j / 32] |= 1u << (j % 32);
    free(acc);
}

/* Same hash for a vector stored in bf16 or fp32 (widened exactly first). */
void oracle_hash_vec(const void *x, int dtype, const float *W, int d, int r, uint32_t *code)
{
    float *xf = (float *)malloc(sizeof(float) * (size_t)d);
    for (int i = 0; i < d; ++i)
        xf[i] = load_elem(x, dtype, i);
    oracle_hash_f32(xf, W, d, r, code);
    free(xf);
}

/* Prefill (Algorithm 1): code every key of positions [pos0, pos0+n) of a
 * [B][H][n_cap][d] key cache into a [B][H][n_cap][r/32] code cache. */
void oracle_hash_keys(const void *K, int dtype, const float *W_H, uint32_t *codes,
                      int64_t n_cap, int B, int H, int64_t pos0, int64_t n, int d, int r)
{
    int words = r / 32;
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h)
            for (int64_t t = pos0; t < pos0 + n; ++t) {
                int64_t row = ((int64_t)b * H + h) * n_cap + t;
                const char *xp = (const char *)K +
                    row * d * (dtype == ORACLE_DT_BF16 ? 2 : 4);
                oracle_hash_vec(xp, dtype, W_H + (int64_t)h * d * r, d, r,
                                codes + row * words);
            }
}

/* ------------------------------------------------------------- hamming ---
 * Number of bit positions where the two codes differ (XOR, then count). */
int oracle_hamming(const uint32_t *a, const uint32_t *b, int r)
{
    int dist = 0;
    for (int j = 0; j < r; ++j) {
        uint32_t x = a[j / 32] ^ b[j / 32];
        dist += (int)((x >> (j % 32)) & 1u);
    }
    return dist;
}

void oracle_hamming_all(const uint32_t *qcode, const uint32_t *codes, int64_t n, int r,
                        int32_t *dist)
{
    int words = r / 32;
    for (int64_t t = 0; t < n; ++t)
        dist[t] = oracle_hamming(qcode, codes + t * words, r);
}

/* ---------------------------------------------------------------- top-k ---
 * Sort (distance, index) ascending -- a total order, so the result is what a
 * stable sort on distance gives -- keep the first min(k, n), then report the
 * kept indices in ascending order.  Unused slots of idx_out[0..k) get -1.
 * Returns the number selected. */
typedef struct {
    int32_t d;
    int64_t i;
} pair_t;

static int cmp_pair(const void *pa, const void *pb)
{
    const pair_t *a = (const pair_t *)pa, *b = (const pair_t *)pb;
    if (a->d != b->d)
        return a->d < b->d ? -1 : 1;
    if (a->i != b->i)
        return a->i < b->i ? -1 : 1;
    return 0;
}

static int cmp_i32(const void *pa, const void *pb)
{
    int32_t a = *(const int32_t *)pa, b = *(const int32_t *)pb;
    return (a > b) - (a < b);
}

int64_t oracle_topk(const int32_t *dist, int64_t n, int64_t k, int32_t *idx_out)
{
    int64_t m = k < n ? k : n;
    if (m < 0)
        m = 0;
    pair_t *p = (pair_t *)malloc(sizeof(pair_t) * (size_t)(n > 0 ? n : 1));
    for (int64_t t = 0; t < n; ++t) {
        p[t].d = dist[t];
        p[t].i = t;
    }
    qsort(p, (size_t)n, sizeof(pair_t), cmp_pair);
    for (int64_t t = 0; t < m; ++t)
        idx_out[t] = (int32_t)p[t].i;
    qsort(idx_out, (size_t)m, sizeof(int32_t), cmp_i32);
    for (int64_t t = m; t < k; ++t)
        idx_out[t] = -1;
    free(p);
    return m;
}

/* ------------------------------------------------------------ attention ---
 * Exact softmax attention of one query over the listed rows, in fp64:
 *   s_t = scale * <q, K[t]>, p = exp(s - max s) / sum, out = sum_t p_t V[t].
 * K and V are [n][d] row-major (bf16 or fp32).  An empty list gives 0. */
void oracle_attend(const float *q, const void *K, const void *V, int dtype, int d,
                   const int32_t *idx, int64_t m, double scale, double *out)
{
    for (int i = 0; i < d; ++i)
        out[i] = 0.0;
    if (m <= 0)
        return;
    double *s = (double *)malloc(sizeof(double) * (size_t)m);
    double smax = -INFINITY;
    for (int64_t t = 0; t < m; ++t) {
        int64_t row = idx[t];
        double acc = 0.0;
        for (int i = 0; i < d; ++i)
            acc += (double)q[i] * (double)load_elem(K, dtype, row * d + i);
        s[t] = scale * acc;
        if (s[t] > smax)
            smax = s[t];
    }
    double l = 0.0;
    for (int64_t t = 0; t < m; ++t) {
        s[t] = exp(s[t] - smax);
        l += s[t];
    }
    for (int64_t t = 0; t < m; ++t) {
        int64_t row = idx[t];
        for (int i = 0; i < d; ++i)
            out[i] += s[t] * (double)load_elem(V, dtype, row * d + i);
    }
    for (int i = 0; i < d; ++i)
        out[i] /= l;
    free(s);
}

/* Dense softmax attention over rows 0..n-1 (the baseline the sparse path is
 * compared with; with k >= n the two must agree). */
void oracle_dense(const float *q, const void *K, const void *V, int dtype, int d, int64_t n,
                  double scale, double *out)
{
    int32_t *idx = (int32_t *)malloc(sizeof(int32_t) * (size_t)(n > 0 ? n : 1));
    for (int64_t t = 0; t < n; ++t)
        idx[t] = (int32_t)t;
    oracle_attend(q, K, V, dtype, d, idx, n, scale, out);
    free(idx);
}

/* ---------------------------------------------------------- decode step ---
 * One query head's decode step (Figure 2): hash q with its KV head's W_H,
 * score the n cached codes, keep the top-k, attend over them.
 *   q      [d] fp32          W       [d][r] fp32 (this KV head's)
 *   codes  [n][r/32]         K, V    [n][d] (this KV head's rows)
 * Outputs: qcode [r/32], dist [n], idx [k] (ascending, -1 pad), out [d].
 * Returns the number of selected keys. */
int64_t oracle_decode_head(const float *q, const float *W, const uint32_t *codes,
                           const void *K, const void *V, int dtype, int64_t n, int d, int r,
                           int64_t k, double scale, uint32_t *qcode, int32_t *dist,
                           int32_t *idx, double *out)
{
    oracle_hash_f32(q, W, d, r, qcode);
    oracle_hamming_all(qcode, codes, n, r, dist);
    int64_t m = oracle_topk(dist, n, k, idx);
    oracle_attend(q, K, V, dtype, d, idx, m, scale, out);
    return m;
}
