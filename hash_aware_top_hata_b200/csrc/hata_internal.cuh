// hata_internal.cuh -- constants, workspace layout and launch declarations
// shared by the CUDA translation units of libhata.  Not part of the ABI.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "../../include/hata.h"

namespace hata {

constexpr int kD = 128;         // head_dim (the page's models all use 128)
constexpr int kRbit = 128;      // the page's hash width (rbit = 128)
constexpr int kRbitWide = 256;  // widest hash of its ablation (32, 64 and 256 too)
constexpr int kBins = kRbit + 1;        // Hamming distances 0..128 (fewer bins used below)
constexpr int kBinsWide = kRbitWide + 1;  // distances 0..256 of the 256-bit codes
constexpr int kChunk = 4096;            // tokens per scoring / selection chunk
constexpr int kScoreThreads = 1024;
constexpr int kScoreHeads = 8;          // query heads scored per code load (one CTA)
constexpr int kAttnThreads = 128;
constexpr int kHistStride = 132;        // u32 per (head, tile) histogram row (129 bins)
constexpr int kHistStrideWide = 260;    // the same at r = 256 (257 bins); the workspace
                                        // reserves rows of this size for every width
constexpr int kTile = 36864;            // tokens per histogram tile / selection tile (9 x 4096)
constexpr int kPartStride = 132;        // f32 per (head, chunk) partial: m, l, -, -, acc[128]
constexpr int kFSeg = 96;               // selected rows per attention item, fused step
                                        // (16 per attention warp)
constexpr uint8_t kDistPad = 255;       // distance stored past seq_len; at r = 256 the
                                        // stored distance saturates at 255 too
constexpr int kSpHistWords = 260;       // sequence-parallel histogram row (HATA_SP_HIST_WORDS)
constexpr uint32_t kWsMagic = 0x48415441u;  // "HATA"

__host__ __device__ inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// A batch row's sequence length as the kernels use it: seq_len[b] clamped to
// [0, min(max_len, n_cap)] (an out-of-range length is also flagged by prep).
__device__ __forceinline__ int64_t clamp_len(int32_t sl, int64_t max_len, int64_t n_cap)
{
    int64_t l = sl < 0 ? 0 : sl;
    l = l < max_len ? l : max_len;
    return l < n_cap ? l : n_cap;
}
inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

constexpr int kAttnMaxWorkers = 4096;   // upper bound of the attention stream-K workers

// Most attention workers that can share one head: each of the P <= T
// workers owns at least floor(T / P) >= r_min rows of the flat row space.
inline int attn_max_contributors(int64_t BH, int topk)
{
    const int64_t T = BH * topk;
    const int64_t r_min = T >= kAttnMaxWorkers ? T / kAttnMaxWorkers : 1;
    const int64_t c = (topk + r_min - 1) / r_min + 1;
    return int(c < kAttnMaxWorkers ? c : kAttnMaxWorkers);
}

// Decode workspace.  The first 256 B hold a header {magic, B}; one flag word
// per batch row follows.  Everything else is rebuilt by every decode step.
struct DecodeLayout {
    int64_t n_chunks = 0;   // 4096-token chunks of max_seq_len
    int64_t dist_row = 0;   // bytes per (b, h_q) distance row
    int64_t n_tiles = 0;    // 36K-token histogram / selection tiles of a distance row
    int zgroups = 0;        // ceil(G / kScoreHeads)
    int n_split = 0;        // attention partial slots per head (multi-kernel step)
    int n_seg = 0;          // attention items per head (fused step)
    size_t off_flags = 0, off_qcodes = 0, off_q = 0, off_dist = 0, off_hist = 0, off_idx = 0,
           off_part = 0, off_sync = 0, off_khead = 0, total = 0;
};

// Words per (head, tile) histogram row for r/32 = words code words.
inline int hist_stride(int words) { return words == 8 ? kHistStrideWide : kHistStride; }

inline bool decode_layout(int B, int H_q, int H_kv, int64_t max_seq_len, int topk,
                          DecodeLayout *L)
{
    if (B <= 0 || H_q <= 0 || H_kv <= 0 || max_seq_len <= 0 || topk <= 0) return false;
    if (H_q % H_kv != 0) return false;
    if (max_seq_len > (int64_t(1) << 31) - kChunk) return false;
    const int64_t BH = int64_t(B) * H_q;
    if (BH > (int64_t(1) << 24) || int64_t(B) * H_kv > (int64_t(1) << 24)) return false;
    const int G = H_q / H_kv;
    L->n_chunks = ceil_div(max_seq_len, kChunk);
    L->dist_row = L->n_chunks * kChunk;
    L->n_tiles = ceil_div(L->dist_row, kTile);
    L->zgroups = int(ceil_div(G, kScoreHeads));
    // the scoring kernel numbers its 128-token units with 32-bit integers
    if (int64_t(B) * H_kv * L->zgroups * (L->dist_row / 128) >= (int64_t(1) << 31)) return false;
    L->n_split = attn_max_contributors(BH, topk);
    L->n_seg = int(ceil_div(topk, kFSeg));
    // the fused step numbers its selection and attention items with 32-bit
    // integers too
    if (BH * L->n_seg >= (int64_t(1) << 31) || BH * L->n_tiles >= (int64_t(1) << 31)) return false;
    const int64_t parts = L->n_split > L->n_seg ? L->n_split : L->n_seg;
    size_t o = 256;
    L->off_flags = o;      o = align_up(o + 4 * size_t(B), 256);
    L->off_qcodes = o;     o = align_up(o + 32 * size_t(BH), 256);  // up to 8 words a head
    L->off_q = o;          o = align_up(o + 4 * kD * size_t(BH), 256);  // q, read once per step
    L->off_dist = o;       o = align_up(o + size_t(BH) * L->dist_row, 256);
    L->off_hist = o;       o = align_up(o + 4 * size_t(BH) * L->n_tiles * kHistStrideWide, 256);
    L->off_idx = o;        o = align_up(o + 4 * size_t(BH) * topk, 256);
    L->off_part = o;       o = align_up(o + 4 * size_t(BH) * parts * kPartStride, 256);
    // fused-step counters: selection tiles done and attention items published
    // per head, then the step's abort word (all zeroed by prep every step)
    L->off_sync = o;       o = align_up(o + 4 * size_t(2 * BH + 1), 256);
    // sequence-parallel step: the keys each head selects from this shard
    L->off_khead = o;      o = align_up(o + 4 * size_t(BH), 256);
    L->total = o;
    return true;
}

// ------------------------------------------------------------------ args --
struct PrepArgs {
    const float *q;          // [B][H_q][128] or null (append only); device or mapped host
    float *q_copy;           // [B][H_q][128] device copy of q for the attention, or null
    const void *k_new;       // [B][H_kv][128] or null
    const void *v_new;       // [B][H_kv][128] or null
    const float *W;          // [H_kv][128][r]
    uint32_t *codes;         // [B][H_kv][n_cap][r/32]
    void *K, *V;             // caches, written only if v_new
    const int32_t *pos;      // explicit append positions [B] (append API) or null
    const int32_t *seq_len;  // decode: append at seq_len[b]-1, flags
    uint32_t *q_out;         // [B][H_q][r/32]
    uint32_t *flags;         // per-b flag words (decode) or null
    uint32_t *err_word;      // single OR-ed word (append API) or null
    uint32_t *hist;          // [B][H_q][hist_row_words] zeroed (decode) or null
    int64_t hist_row_words;  // n_tiles * hist_stride(words)
    uint32_t *sync;          // fused-step counters zeroed (decode, fused step) or null:
                             // [B][H_q] twice, then one abort word
    uint32_t *ws_header;     // {magic, B} written (decode) or null
    int64_t n_cap, max_seq_len;
    int B, H_q, H_kv, G;
    int kv_bf16;
    int words;               // r / 32: code words per token (1, 2 or 4)
};

struct ScoreArgs {
    const uint32_t *qcodes;  // [B][H_q][r/32]
    const uint32_t *codes;   // [B][H_kv][n_cap][r/32]
    const int32_t *seq_len;
    uint8_t *dist;           // [B][H_q][dist_row]
    int64_t dist_row;
    uint32_t *hist;          // [B][H_q][n_tiles][hist_stride(words)], zeroed by prep
    int64_t n_cap, max_seq_len, n_tiles;
    int B, H_q, H_kv, G, zgroups;
    int words;               // r / 32 (1, 2, 4 or 8)
};

struct SelectArgs {
    const int32_t *seq_len;
    const uint8_t *dist;
    int64_t dist_row;
    const uint32_t *hist;    // [B][H_q][n_tiles][hist_stride(words)]
    int32_t *idx;            // [B][H_q][topk] ascending, -1 padded
    const int32_t *k_head;   // [B][H_q] keys to select per head (sequence-parallel step;
                             // written by the kernel before) or null: min(topk, len)
    const uint32_t *qcodes;  // r = 256 only: [B][H_q][8] query codes and the key codes
    const uint32_t *codes;   //   [B][H_kv][n_cap][8], for exact distances at 255 / 256
    int64_t n_cap, max_seq_len, n_tiles;
    int B, H_q, H_kv, G, topk;
    int words;
};

struct AttendArgs {
    const float *q;
    const void *K, *V;
    const int32_t *seq_len;
    const int32_t *idx;      // [B][H_q][topk]
    float *part;             // [B][H_q][n_split][kPartStride]
    uint32_t *flags;
    float *out;
    int64_t n_cap, max_seq_len;
    int B, H_q, H_kv, G, topk, n_split;
    int64_t n_workers;       // stream-K workers (set by the launcher)
    int head_per_cta;        // 1: a CTA's warps cover one whole head and merge it in shared
                             // memory (no combine launch); set by the launcher
    int head_split;          // > 0: head_split CTAs per head (the sequence-parallel step);
                             // set by the launcher
    const int32_t *k_head;   // [B][H_q] selected keys per head, or null: min(topk, len)
    float *part_out;         // [B][H_q][kPartStride]: unnormalised (m, l, acc) per head
                             // instead of out (the sequence-parallel step), or null
    float scale_log2;        // scale * log2(e)
};

// The fused step's selection + attention kernel (after prep and the scoring
// kernel): selection warps turn the distance rows into index lists, attention
// warps gather and attend the heads selected so far, one publisher warp per
// CTA hands results between CTAs.
struct FusedArgs {
    const int32_t *seq_len;
    const float *q;          // [B][H_q][128] device copy written by prep
    const void *K, *V;       // bf16 [B][H_kv][n_cap][128]
    const uint8_t *dist;     // [B][H_q][dist_row] (scoring kernel)
    const uint32_t *hist;    // [B][H_q][n_tiles][kHistStride] (scoring kernel)
    int32_t *idx;            // [B][H_q][topk]
    float *part;             // [B][H_q][n_seg][kPartStride]
    float *out;              // [B][H_q][128]
    uint32_t *sel_done;      // [B][H_q] selection tiles done, zeroed by prep
    uint32_t *head_cnt;      // [B][H_q] attention items published, zeroed by prep
    uint32_t *flags;         // per-b flag words: a wait that gives up ORs TIMEOUT into [0]
    uint32_t *abort_word;    // this step's "someone gave up" word, zeroed by prep
    int64_t dist_row;        // stride of the distance rows (bytes)
    int64_t dist_len;        // bytes of each row the scoring kernel wrote: max_seq_len
                             // rounded up to kChunk
    int64_t n_cap, max_seq_len;
    int n_tiles;             // kTile tiles of dist_len
    int B, H_q, H_kv, G, topk, n_seg;
    float scale_log2;
    uint64_t spin_limit_ns;  // bound of every wait
};

// The cluster step (one kernel per decode step for heads whose cache fits a
// thread-block cluster of up to kClusterMaxC CTAs of 8192 tokens each).
constexpr int kClusterMaxG = 4;   // query heads per KV head it serves (1, 2 or 4)
constexpr int kClusterMaxC = 8;   // CTAs per cluster (portable cluster size)

struct ClusterArgs {
    const float *q;          // [B][H_q][128]; device or mapped host
    const float *W;          // [H_kv][128][128]
    uint32_t *codes;         // [B][H_kv][n_cap][4]; the new key's code is written
    void *K, *V;             // bf16 or fp32 caches; the new rows written if v_new
    const void *k_new;       // [B][H_kv][128] (cache dtype) or null
    const void *v_new;       // [B][H_kv][128] (cache dtype) or null
    const int32_t *seq_len;
    uint32_t *q_out;         // [B][H_q][4] or null
    uint8_t *dist;           // caller's distance rows or null
    int64_t dist_row;
    int32_t *idx;            // [B][H_q][topk]
    float *out;              // [B][H_q][128]; device or mapped host
    uint32_t *flags;         // per-b flag words
    uint32_t *ws_header;     // {magic, B}
    int64_t n_cap, max_seq_len;
    int B, H_q, H_kv, G, topk;
    int tok_per_cta;         // tokens of a CTA's range (a multiple of 32; the plan's)
    int kv_bf16;             // 1: bf16 caches, 0: fp32
    float scale_log2;
};

// How the cluster step covers a head: kM = 0 (it does not), else CTAs of up
// to 8192 kM tokens, C of them per (b, h_kv), tok_per_cta tokens each.
struct ClusterPlan {
    int kM = 0, C = 0, tok_per_cta = 0;
};

struct DenseArgs {
    const float *q;
    const void *K, *V;
    const int32_t *seq_len;
    float *part;             // [B][H_q][n_chunks][kPartStride]
    uint32_t *cnt;           // [B][H_kv][zgroups]
    float *out;
    int64_t n_cap, max_seq_len, n_chunks;
    int B, H_q, H_kv, G, zgroups;
    float scale_log2;
};

constexpr int kDenseChunk = 2048;       // tokens per dense CTA
constexpr int kDenseHeads = 4;          // query heads sharing one K/V row load

inline bool dense_layout(int B, int H_q, int H_kv, int64_t max_seq_len, int64_t *n_chunks,
                         size_t *off_part, size_t *off_cnt, size_t *total)
{
    if (B <= 0 || H_q <= 0 || H_kv <= 0 || max_seq_len <= 0 || H_q % H_kv) return false;
    if (max_seq_len > (int64_t(1) << 31) - kDenseChunk) return false;
    const int64_t BH = int64_t(B) * H_q;
    if (BH > (int64_t(1) << 24)) return false;
    const int G = H_q / H_kv;
    *n_chunks = ceil_div(max_seq_len, kDenseChunk);
    size_t o = 256;
    *off_part = o;  o = align_up(o + 4 * size_t(BH) * (*n_chunks) * kPartStride, 256);
    *off_cnt = o;   o = align_up(o + 4 * size_t(B) * H_kv * ceil_div(G, kDenseHeads), 256);
    *total = o;
    return true;
}

// ------------------------------------------- programmatic dependent launch --
// The kernels after the first of a decode step are launched with programmatic
// stream serialization: a dependent grid may be scheduled while its
// predecessor still runs, so its launch latency hides behind that kernel.
// Every such kernel lets its own dependent go (pdl_trigger) and then waits
// for its predecessor to complete, with all its memory writes visible
// (pdl_wait), before it reads anything the predecessor produced.  Both are
// no-ops for a kernel launched without the attribute.
__device__ __forceinline__ void pdl_trigger()
{
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t s, Args &&...args)
{
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Records msg as hata_last_error() of this thread and returns st.
hata_status_t report_error(hata_status_t st, const char *msg);

// Opt a kernel into `bytes` of dynamic shared memory (more than 48 KB needs
// it) and the largest shared-memory carveout, once per device.
cudaError_t ensure_smem_attr(const void *func, size_t bytes);

// Launchers (each returns the cudaGetLastError() of its launch).
// Element strides of a key cache K[b][h][t][i] (i contiguous).
struct KStrides {
    int64_t b, h, n;
};
cudaError_t launch_hash_prefill(const void *K, bool bf16, KStrides ks, int64_t n_cap,
                                const float *W, uint32_t *codes, int B, int H_kv, int64_t pos0,
                                int64_t n, int words, cudaStream_t s);
cudaError_t launch_prep(const PrepArgs &a, int rows_per_head, cudaStream_t s);
cudaError_t launch_score(const ScoreArgs &a, cudaStream_t s);
cudaError_t launch_select(const SelectArgs &a, cudaStream_t s);
cudaError_t launch_attend(AttendArgs &a, bool bf16, cudaStream_t s);  // sets a.n_workers
cudaError_t launch_combine(const AttendArgs &a, cudaStream_t s);
// Kernels launch_attend + launch_combine issue for these sizes on the current
// device: 1 when the heads are merged inside the attention CTAs, else 2.
cudaError_t attend_launch_count(int B, int H_q, int topk, bool bf16, int *n);
cudaError_t launch_dense(const DenseArgs &a, bool bf16, cudaStream_t s);
cudaError_t launch_fused(const FusedArgs &a, cudaStream_t s);
// The cluster step's plan for these sizes on this device (r = 128 is the
// caller's check); plan->kM == 0 when it does not serve them.
cudaError_t cluster_step_plan(int B, int H_q, int H_kv, int64_t max_seq_len, int topk, bool bf16,
                              ClusterPlan *plan);
cudaError_t launch_cluster_step(const ClusterArgs &a, const ClusterPlan &p, cudaStream_t s);
// Sequence-parallel step: the attention of one shard's selected keys split
// over several CTAs per head (bf16; fp32 caches take launch_attend with
// a.k_head), partials merged by launch_combine into a.part_out.
cudaError_t launch_attend_split(AttendArgs &a, cudaStream_t s);  // sets a.head_split
// The per-head sum of the tile histograms: out[bh][0 .. kSpHistWords).
cudaError_t launch_sp_hist(const uint32_t *hist, int64_t n_tiles, int stride, int64_t BH,
                           uint32_t *out, cudaStream_t s);
// Keys each head selects from shard `rank` of `world`, from every shard's
// histogram (hist_all: [world][BH][kSpHistWords], `bins` = r + 1 used).
cudaError_t launch_sp_quota(const uint32_t *hist_all, int world, int rank, int64_t BH, int topk,
                            int bins, int32_t *k_head, cudaStream_t s);
// out[bh] = merge of the world partials part_all[w][bh][kPartStride].
cudaError_t launch_sp_merge(const float *part_all, int world, int64_t BH, float *out,
                            cudaStream_t s);

}  // namespace hata
