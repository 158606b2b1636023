/*
 * hata.h -- C ABI of the B200 (sm_100a) hash-aware top-k attention (HATA)
 * decode path.
 *
 * The method (HATA review page, arXiv 2506.02572):
 *   "What carries the argument": every query and key is hashed per attention
 *     head to r = 128 bits; the query code is XOR-ed with every cached key
 *     code and a popcount gives the Hamming score; the top-k keys are
 *     gathered and attention runs over them only ("fused gather-attention").
 *   "Assumptions & free parameters": inference hash h(x) = sign(x W_H),
 *     W_H per head, rbit = 128.
 *   Figure 2 caption, Algorithm 1 (prefill): HashEncode(K) fills the key code
 *     cache Kcache_H, rbit/32 32-bit words per token; K and V fill the KV cache.
 *   Referee report, major comment 1 (Algorithm 3): top-k over 129 possible
 *     Hamming values; the choice inside the boundary bucket is left open.
 *   "Assumptions & free parameters": rbit is a free parameter chosen by
 *     ablation (accuracy grows from 32 to 128 bits, then levels off).
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are DEVICE pointers, allocated and owned by the
 *     caller; the library never allocates, frees or keeps them.  Work is
 *     enqueued on `stream` (a cudaStream_t; NULL = legacy default stream)
 *     and the call returns without synchronising, except where noted.
 *   - d (head_dim) must be 128; r (hash bits) 128, the page's width, or 32,
 *     64 or 256, the other widths of its ablation (HATA_ERR_UNSUPPORTED
 *     otherwise).  At r = 256 the distances run 0..256; selections use them
 *     exactly, while the optional byte-wide distance rows store min(d, 255).
 *   - Layouts are dense row-major:
 *       W_H    [H_kv][d][r]        fp32, 16-byte aligned; bit j of a code is
 *                                   [sum_i x_i W_H[i][j] > 0]
 *       K, V   [B][H_kv][n_cap][d] bf16 or fp32 (kv_dtype), 16-byte aligned
 *       codes  [B][H_kv][n_cap][r/32] uint32, bit j in word j/32 at bit j%32
 *                                   (least significant first), 16-byte aligned
 *       q, out [B][H_q][d] fp32, 16-byte aligned
 *       k_new, v_new [B][H_kv][d] (kv_dtype), 16-byte aligned
 *     Query head h_q uses KV head h_q / (H_q / H_kv) (grouped-query attention);
 *     its code is made with that KV head's W_H so that codes are comparable.
 *   - Hash arithmetic: the projection of bit j is the fp32 chain
 *     acc = fmaf(x_i, W_H[i][j], acc) over i = 0..127 ascending from acc = +0;
 *     bf16 inputs are widened exactly.  A projection of exactly 0 (or NaN)
 *     gives bit 0.
 *   - Argument checks run on the host before anything is launched; a failed
 *     check returns HATA_ERR_INVALID_ARG / HATA_ERR_UNSUPPORTED and enqueues
 *     nothing.  A failed launch returns HATA_ERR_CUDA.  Device-side range
 *     checks (a seq_len beyond max_seq_len or n_cap, an append position
 *     outside the cache) never fault: the kernel clamps or skips, records a
 *     flag, and hata_workspace_check / the err_flags word reports it.
 *   - Nothing throws across the ABI.  Calls are thread-safe; calls that share
 *     a workspace must be ordered on one stream.
 */
#ifndef HATA_H
#define HATA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum hata_status {
    HATA_OK = 0,
    HATA_ERR_INVALID_ARG = 1,   /* null pointer, bad size, misalignment, small workspace */
    HATA_ERR_UNSUPPORTED = 2,   /* d != 128, r not 32/64/128/256, H_q not a multiple of H_kv */
    HATA_ERR_CUDA = 3,          /* a CUDA launch or copy failed */
    HATA_ERR_DEVICE_CHECK = 4   /* a device-side range check fired (see the flags) */
} hata_status_t;

typedef enum hata_dtype {
    HATA_DT_BF16 = 0,
    HATA_DT_F32 = 1
} hata_dtype_t;

/* Device-side check flags (OR-ed into the error word). */
#define HATA_FLAG_SEQ_LEN_RANGE 1u  /* seq_len[b] < 0, > max_seq_len or > n_cap: clamped */
#define HATA_FLAG_POS_RANGE     2u  /* an append position outside [0, n_cap): skipped  */
#define HATA_FLAG_TIMEOUT       4u  /* a bounded wait of the fused decode step gave up:
                                       its results are not valid (see
                                       hata_set_wait_limit_ns)                         */

/* ABI revision; bumps whenever a signature below changes. */
int hata_abi_version(void);

/* Static text for a status code. */
const char *hata_status_string(int status);

/* Text describing the most recent failed call on this host thread
 * (thread-local; "" if none). */
const char *hata_last_error(void);

/* ------------------------------------------------------------------------
 * hata_hash_keys -- prefill (Algorithm 1: KH <- HashEncode(K); Kcache_H <- KH).
 * Hashes the keys of positions [pos0, pos0 + n) of every (b, h_kv) of the
 * key cache K with W_H[h_kv] and writes codes[b][h_kv][pos0 .. pos0+n).
 *   K      (kv_dtype) read: element [b][h][t][i] at
 *          K + b*k_stride_b + h*k_stride_h + t*k_stride_n + i (element
 *          strides; i contiguous), so a strided or paged view of a larger
 *          cache is hashed in place.  The dense [B][H_kv][n_cap][d] cache is
 *          (n_cap*H_kv*d, n_cap*d, d).  Aligned to its element size.
 *   W_H    [H_kv][d][r] fp32                read
 *   codes  [B][H_kv][n_cap][r/32] uint32    written at the hashed positions only
 * Requires 0 <= pos0, n >= 0, pos0 + n <= n_cap, strides >= 0 and
 * k_stride_n >= d.  n == 0 enqueues nothing. */
hata_status_t hata_hash_keys(const void *K, hata_dtype_t kv_dtype, int64_t k_stride_b,
                             int64_t k_stride_h, int64_t k_stride_n, const float *W_H,
                             uint32_t *codes, int64_t n_cap, int B, int H_kv, int64_t pos0,
                             int64_t n, int d, int r, void *stream);

/* ------------------------------------------------------------------------
 * hata_append_code -- decode-time growth of the key code cache (the decode
 * stage extends Kcache_H by one token per step): hashes k_new[b][h] with
 * W_H[h] and writes it to codes[b][h][pos[b]].
 *   k_new     [B][H_kv][d] (kv_dtype)   read
 *   pos       [B] int32, device         read; a position outside [0, n_cap)
 *                                       is skipped and flagged
 *   err_flags optional device uint32    HATA_FLAG_POS_RANGE is OR-ed in
 */
hata_status_t hata_append_code(const void *k_new, hata_dtype_t kv_dtype, const float *W_H,
                               uint32_t *codes, int64_t n_cap, const int32_t *pos, int B,
                               int H_kv, int d, int r, uint32_t *err_flags, void *stream);

/* ------------------------------------------------------------------------
 * Workspace of hata_decode_step: device memory of at least this many bytes,
 * 256-byte aligned, owned by the caller.  It needs no initialisation and
 * carries no state between calls.  Returns 0 for invalid sizes. */
size_t hata_decode_workspace_size(int B, int H_q, int H_kv, int64_t max_seq_len, int topk);

/* Row length (bytes) that an optional caller-provided distance buffer must
 * have at least: max_seq_len rounded up to the scoring chunk (4096). */
int64_t hata_dist_row_bytes(int64_t max_seq_len);

/* Number of kernels one hata_decode_step with these sizes launches on the
 * current device in the current mode (hata_set_decode_mode): 1 for the
 * cluster step; 3 for the fused step (prep, score, the persistent selection
 * + attention kernel); for the multi-kernel step prep, score, select,
 * attention and, unless the heads are merged inside the attention CTAs, the
 * combine kernel: 4 or 5.  Returns -1 (hata_last_error says why) for
 * invalid sizes or if a device query fails.  Host-only; launches nothing. */
int hata_decode_kernel_launches(int B, int H_q, int H_kv, int64_t max_seq_len, int topk,
                                hata_dtype_t kv_dtype, int r);

/* ------------------------------------------------------------------------
 * Step implementation.  Three implementations give the same codes, distances
 * and indices bit for bit (outputs agree within the attention tolerance):
 *   the multi-kernel step  prep, score, select, attention and (unless every
 *                          head is merged inside its attention CTA) combine;
 *   the fused step         prep, score, then ONE persistent kernel with one
 *                          CTA per SM in which selection warps build the
 *                          index lists while attention warps already gather
 *                          and attend the heads selected so far (bf16 caches
 *                          and r <= 128 only);
 *   the cluster step       ONE kernel: a thread-block cluster per (b, h_kv)
 *                          of up to 8 CTAs of up to 16384 tokens each hashes,
 *                          scores, selects and attends, the CTAs meeting
 *                          through distributed shared memory (r = 128,
 *                          H_q / H_kv of 1, 2 or 4, max_seq_len up to
 *                          131072, every cluster resident at once).
 * A step whose sizes the chosen implementation does not serve takes the
 * multi-kernel step.
 *   HATA_MODE_AUTO          the library's choice (default): the cluster step
 *                           where it serves, else the multi-kernel step
 *   HATA_MODE_MULTI_KERNEL  always the multi-kernel step
 *   HATA_MODE_FUSED         the fused step
 *   HATA_MODE_CLUSTER       the cluster step
 * The mode is process-wide and read when a step is enqueued. */
#define HATA_MODE_AUTO 0
#define HATA_MODE_MULTI_KERNEL 1
#define HATA_MODE_FUSED 2
#define HATA_MODE_CLUSTER 3
hata_status_t hata_set_decode_mode(int mode);
int hata_get_decode_mode(void);

/* Bound, in nanoseconds of wall time, of every wait of the fused step's
 * persistent kernel on another warp or CTA (default 1 s; process-wide, read
 * when a step is enqueued).  A wait that reaches it gives up: the kernel sets
 * HATA_FLAG_TIMEOUT (reported by hata_workspace_check) and finishes without
 * valid results instead of staying resident.  Its CTAs must all be resident
 * at once to make progress, so a GPU shared with long-running kernels of
 * other streams may need a longer bound. */
hata_status_t hata_set_wait_limit_ns(uint64_t ns);

/* ------------------------------------------------------------------------
 * hata_decode_step -- one decode step of HATA for every (b, h_q) (Figure 2):
 *   0. optional append: if k_new != NULL its rows are hashed into
 *      codes[b][h][seq_len[b]-1]; if v_new (and k_new) are given, k_new and
 *      v_new are also copied into K/V at that position;
 *   1. q_code[b][h_q] = h(q[b][h_q]) with W_H of its KV head;
 *   2. dist[b][h_q][n] = popcount(q_code XOR codes[b][h_kv][n]), n < seq_len[b];
 *   3. S = the min(topk, seq_len[b]) keys of smallest distance, ties in the
 *      boundary bucket to the lower token index;
 *   4. out[b][h_q] = sum_{n in S} softmax_n(scale * q.K[n]) V[n]  (fp32
 *      accumulation, exact softmax over S only).  seq_len[b] == 0 gives 0.
 * Arguments (q, k_new, v_new and out may be device memory or page-locked host
 * memory that the device can address (any cudaHostAlloc / cudaMallocHost
 * block under unified addressing): each is read, or written, once per step by
 * the kernels themselves, so a step with host inputs and output needs no
 * separate copy operations.  K and V may be page-locked host memory too (the
 * caches kept off the device): a step then reads only the selected rows,
 * 2 * topk rows per query head, across the bus.  Every other buffer is
 * device memory):
 *   q         [B][H_q][d] fp32
 *   W_H       [H_kv][d][r] fp32, 16-byte aligned
 *   codes     [B][H_kv][n_cap][r/32]; written only by the optional append
 *   K, V      [B][H_kv][n_cap][d] kv_dtype; written only when v_new is given
 *   seq_len   [B] int32, device: keys 0 .. seq_len[b]-1 take part
 *   max_seq_len  host upper bound of every seq_len[b] (sizes the grids;
 *                1 <= max_seq_len <= n_cap)
 *   topk      >= 1 (k >= seq_len[b] selects every key)
 *   scale     softmax scale (1/sqrt(d) for standard attention)
 *   workspace, workspace_bytes   see hata_decode_workspace_size
 *   out       [B][H_q][d] fp32, written
 *   sel_idx   optional [B][H_q][topk] int32: S in ascending token order,
 *             slots past |S| set to -1
 *   q_codes   optional [B][H_q][r/32] uint32: the query codes
 *   dist, dist_row_bytes  optional [B][H_q][dist_row_bytes] uint8: the
 *             Hamming distances (0..r; min(d, 255) at r = 256); positions
 *             seq_len[b] ..
 *             hata_dist_row_bytes(max_seq_len)-1 hold 255;
 *             dist_row_bytes >= hata_dist_row_bytes(max_seq_len), multiple of 16
 *   events    optional array of 6 cudaEvent_t recorded on `stream` before the
 *             first kernel and after each of the five kernels (prep, score,
 *             select, attend, combine) -- a profiling hook (an event between
 *             two kernels keeps the second from starting early).  In the
 *             fused step events 3..5 are all recorded after the step kernel,
 *             in the cluster step events 1..5 after its one kernel.
 */
hata_status_t hata_decode_step(const float *q, const float *W_H, uint32_t *codes, void *K,
                               void *V, hata_dtype_t kv_dtype, int64_t n_cap,
                               const int32_t *seq_len, int64_t max_seq_len, const void *k_new,
                               const void *v_new, int B, int H_q, int H_kv, int d, int r,
                               int topk, float scale, void *workspace, size_t workspace_bytes,
                               float *out, int32_t *sel_idx, uint32_t *q_codes, uint8_t *dist,
                               int64_t dist_row_bytes, void *const *events, void *stream);

/* ------------------------------------------------------------------------
 * hata_decode_step_noalloc -- hata_decode_step for callers that cannot
 * allocate device memory (no counterpart in the HATA paper: this is a
 * deployment convenience).  Some callers may not call cudaMalloc -- a plugin
 * inside a serving engine that hands all device memory to its own pool, or
 * code on a latency-critical path where cudaMalloc's implicit device
 * synchronisation is not allowed.  They still pass every input and output;
 * the decode scratch comes from a fixed array of
 * HATA_NOALLOC_WORKSPACE_BYTES in the library's device image, which every
 * GPU that loads the library holds until the process exits.
 *   - Arguments and results are those of hata_decode_step without
 *     workspace / workspace_bytes.
 *   - Sizes whose scratch (hata_decode_workspace_size) exceeds the fixed
 *     buffer are rejected with HATA_ERR_INVALID_ARG before anything runs.
 *   - The first call on each device looks the buffer's device address up
 *     (cudaGetSymbolAddress, with that device current) and caches it; make
 *     that first call before any stream capture.
 *   - Nothing in the buffer needs to start at zero: every step rebuilds the
 *     counters and histograms it uses.  All calls on a device share the one
 *     buffer, so calls that may overlap on the GPU (different streams
 *     without ordering between them) race: order them on one stream.
 *   - hata_workspace_check cannot see this buffer; device-side flags of
 *     this entry point are not reported.
 *   - The cached address belongs to the device's current context: after
 *     cudaDeviceReset (or any other teardown of the primary context) the
 *     library's device image is loaded again and the array may move, so
 *     this entry point must not be called again in that process.
 * The call allocates nothing (no cudaMalloc / cudaFree / allocating
 * library routine). */
#define HATA_NOALLOC_WORKSPACE_BYTES (64u << 20)
hata_status_t hata_decode_step_noalloc(const float *q, const float *W_H, uint32_t *codes,
                                       void *K, void *V, hata_dtype_t kv_dtype, int64_t n_cap,
                                       const int32_t *seq_len, int64_t max_seq_len,
                                       const void *k_new, const void *v_new, int B, int H_q,
                                       int H_kv, int d, int r, int topk, float scale, float *out,
                                       int32_t *sel_idx, uint32_t *q_codes, uint8_t *dist,
                                       int64_t dist_row_bytes, void *const *events, void *stream);

/* ------------------------------------------------------------------------
 * Sequence-parallel decode step (one head's keys sharded over ranks).
 * The cached tokens of every (b, h_kv) are split into contiguous shards, one
 * per rank, in rank order (rank w holds global tokens o_w .. o_w + len_w - 1
 * with o_0 = 0 and o_{w+1} = o_w + len_w); each rank keeps its shard as an
 * ordinary cache (positions 0 .. len_w - 1, seq_len[b] = len_w).  Algorithm
 * 3's threshold top-k (referee report, major comment 1) needs only the
 * shards' histograms of the r + 1 Hamming values, so a step is two local
 * phases around two small exchanges that the caller runs (all-gathers over
 * NCCL, for instance):
 *   1. hata_sp_score   hash q (and append), score this shard, write its
 *                      per-head histogram [B][H_q][HATA_SP_HIST_WORDS];
 *      exchange        all-gather the histograms of every rank, rank-major:
 *                      hist_all [world][B][H_q][HATA_SP_HIST_WORDS];
 *   2. hata_sp_attend  from hist_all: the global threshold and this shard's
 *                      share of the boundary ties (lower ranks, i.e. lower
 *                      tokens, first), then the shard's selection and the
 *                      attention over it, written as an unnormalised partial
 *                      [B][H_q][HATA_SP_PART_WORDS] fp32: {m, l, -, -,
 *                      acc[128]} with m in log2 units (scale * log2 e), the
 *                      weights 2^(s - m), l their sum, acc the weighted sum
 *                      of V rows (m = -inf, l = 0, acc = 0 when empty);
 *      exchange        all-gather the partials: part_all [world][B][H_q][132];
 *   3. hata_sp_merge   out = the log-sum-exp merge of the world partials.
 * The union of the ranks' selections (shard positions + o_w) is the
 * single-GPU selection of the whole sequence bit for bit, and out agrees
 * with the single-GPU output within the attention tolerance.
 * Phases 1 and 2 of a step use the same workspace (hata_decode_workspace_size
 * of the same B, H_q, H_kv, max_seq_len, topk) and must be ordered on one
 * stream; phase 2 reads the query codes, distances and tile histograms
 * phase 1 left there.  A rank whose shard is empty passes seq_len 0.
 * Only the rank that holds the newest token passes k_new / v_new. */
#define HATA_SP_HIST_WORDS 260
#define HATA_SP_PART_WORDS 132
hata_status_t hata_sp_score(const float *q, const float *W_H, uint32_t *codes, void *K, void *V,
                            hata_dtype_t kv_dtype, int64_t n_cap, const int32_t *seq_len,
                            int64_t max_seq_len, const void *k_new, const void *v_new, int B,
                            int H_q, int H_kv, int d, int r, int topk, void *workspace,
                            size_t workspace_bytes, uint32_t *hist_out, void *stream);
/* sel_idx: optional [B][H_q][topk] int32, this shard's selected positions
 * (shard-local, ascending), -1 after the last. */
hata_status_t hata_sp_attend(const uint32_t *hist_all, int world, int rank,
                             const uint32_t *codes, const void *K, const void *V,
                             hata_dtype_t kv_dtype, int64_t n_cap, const int32_t *seq_len,
                             int64_t max_seq_len, int B, int H_q, int H_kv, int d, int r,
                             int topk, float scale, void *workspace, size_t workspace_bytes,
                             float *part_out, int32_t *sel_idx, void *stream);
hata_status_t hata_sp_merge(const float *part_all, int world, int B, int H_q, float *out,
                            void *stream);

/* ------------------------------------------------------------------------
 * hata_workspace_check -- synchronises `stream`, reads and clears the
 * device-side check flags of a decode workspace.  Returns HATA_OK if none
 * fired, HATA_ERR_DEVICE_CHECK otherwise (flags, if non-NULL, receives them). */
hata_status_t hata_workspace_check(void *workspace, size_t workspace_bytes, uint32_t *flags,
                                   void *stream);

/* ------------------------------------------------------------------------
 * hata_dense_decode -- dense decode attention over all keys 0..seq_len[b]-1
 * (the full-attention baseline HATA is compared with; with topk >= seq_len
 * hata_decode_step must agree with it).  Same layouts as hata_decode_step.
 * workspace: hata_dense_workspace_size bytes, 256-byte aligned. */
size_t hata_dense_workspace_size(int B, int H_q, int H_kv, int64_t max_seq_len);
hata_status_t hata_dense_decode(const float *q, const void *K, const void *V,
                                hata_dtype_t kv_dtype, int64_t n_cap, const int32_t *seq_len,
                                int64_t max_seq_len, int B, int H_q, int H_kv, int d,
                                float scale, void *workspace, size_t workspace_bytes,
                                float *out, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* HATA_H */
