// hata_internal.cuh -- constants, workspace layout and launch declarations
// shared by the CUDA translation units of libhata.  Not part of the ABI.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/hata.h"

namespace hata {

constexpr int kD = 128;         // head_dim (the page's models all use 128)
constexpr int kRbit = 128;      // hash bits (rbit = 128 on the HATA page)
constexpr int kWords = kRbit / 32;
constexpr int kBins = kRbit + 1;        // Hamming distances 0..128
constexpr int kChunk = 4096;            // tokens per scoring / selection chunk
constexpr int kScoreThreads = 256;
constexpr int kScoreHeads = 8;          // query heads scored per code load (one CTA)
constexpr int kAttnThreads = 128;
constexpr int kCumStride = 132;         // u32 per (head, chunk) cumulative histogram
constexpr int kHistStride = 132;        // u32 per head total histogram
constexpr int kPartStride = 132;        // f32 per (head, chunk) partial: m, l, -, -, acc[128]
constexpr int kPrepRows = 4;            // rows hashed together by one prep CTA
constexpr uint8_t kDistPad = 255;       // distance stored past seq_len
constexpr uint32_t kWsMagic = 0x48415441u;  // "HATA"

__host__ __device__ inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Decode workspace.  The first 256 B hold a header {magic, B}; one flag word
// per batch row follows.  Everything else is rebuilt by every decode step.
struct DecodeLayout {
    int64_t n_chunks = 0;   // chunks of max_seq_len
    int64_t dist_row = 0;   // bytes per (b, h_q) distance row
    int zgroups = 0;        // ceil(G / kScoreHeads)
    size_t off_flags = 0, off_qcodes = 0, off_dist = 0, off_cum = 0, off_hist = 0,
           off_plan_head = 0, off_plan_chunk = 0, off_part = 0, off_cnt_score = 0,
           off_cnt_attn = 0, total = 0;
};

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
    L->zgroups = int(ceil_div(G, kScoreHeads));
    size_t o = 256;
    L->off_flags = o;      o = align_up(o + 4 * size_t(B), 256);
    L->off_qcodes = o;     o = align_up(o + 16 * size_t(BH), 256);
    L->off_dist = o;       o = align_up(o + size_t(BH) * L->dist_row, 256);
    L->off_cum = o;        o = align_up(o + 4 * size_t(BH) * L->n_chunks * kCumStride, 256);
    L->off_hist = o;       o = align_up(o + 4 * size_t(BH) * kHistStride, 256);
    L->off_plan_head = o;  o = align_up(o + 16 * size_t(BH), 256);
    L->off_plan_chunk = o; o = align_up(o + 8 * size_t(BH) * L->n_chunks, 256);
    L->off_part = o;       o = align_up(o + 4 * size_t(BH) * L->n_chunks * kPartStride, 256);
    L->off_cnt_score = o;  o = align_up(o + 4 * size_t(B) * H_kv * L->zgroups, 256);
    L->off_cnt_attn = o;   o = align_up(o + 4 * size_t(BH), 256);
    L->total = o;
    return true;
}

// Per-head plan written by the last scoring CTA of a (b, kv-head) group.
struct PlanHead {
    int32_t T;       // boundary distance (-1: nothing selected)
    int32_t k_eff;   // min(topk, seq_len)
    int32_t n_less;  // keys with distance < T
    int32_t ties;    // keys taken from the boundary bucket
};

struct PlanChunk {
    int32_t off;     // first output slot of this chunk's selected keys
    int32_t take;    // boundary-bucket keys this chunk contributes
};

// ------------------------------------------------------------------ args --
struct PrepArgs {
    const float *q;          // [B][H_q][128] or null (append only)
    const void *k_new;       // [B][H_kv][128] or null
    const void *v_new;       // [B][H_kv][128] or null
    const float *W;          // [H_kv][128][128]
    uint32_t *codes;         // [B][H_kv][n_cap][4]
    void *K, *V;             // caches, written only if v_new
    const int32_t *pos;      // explicit append positions [B] (append API) or null
    const int32_t *seq_len;  // decode: append at seq_len[b]-1, flags
    uint32_t *q_out;         // [B][H_q][4]
    uint32_t *flags;         // per-b flag words (decode) or null
    uint32_t *err_word;      // single OR-ed word (append API) or null
    uint32_t *hist_total;    // zeroed for every query row (decode) or null
    uint32_t *cnt_attn;      // zeroed for every query row (decode) or null
    uint32_t *cnt_score;     // zeroed [B][H_kv][zgroups] (decode) or null
    uint32_t *ws_header;     // {magic, B} written (decode) or null
    int64_t n_cap, max_seq_len;
    int B, H_q, H_kv, G, zgroups;
    int kv_bf16;
};

struct ScoreArgs {
    const uint32_t *qcodes;  // [B][H_q][4]
    const uint32_t *codes;   // [B][H_kv][n_cap][4]
    const int32_t *seq_len;
    uint8_t *dist;           // [B][H_q][dist_row]
    int64_t dist_row;
    uint32_t *cum;           // [B][H_q][n_chunks][kCumStride]
    uint32_t *hist_total;    // [B][H_q][kHistStride]
    PlanHead *plan_head;     // [B][H_q]
    PlanChunk *plan_chunk;   // [B][H_q][n_chunks]
    uint32_t *cnt_score;     // [B][H_kv][zgroups]
    int32_t *sel_idx;        // optional [B][H_q][topk] (only -1 padding written here)
    int64_t n_cap, max_seq_len, n_chunks;
    int B, H_q, H_kv, G, zgroups, topk;
};

struct AttendArgs {
    const float *q;
    const void *K, *V;
    const int32_t *seq_len;
    const uint8_t *dist;
    int64_t dist_row;
    const PlanHead *plan_head;
    const PlanChunk *plan_chunk;
    float *part;             // [B][H_q][n_chunks][kPartStride]
    uint32_t *cnt_attn;      // [B][H_q]
    float *out;
    int32_t *sel_idx;
    int64_t n_cap, max_seq_len, n_chunks;
    int B, H_q, H_kv, G, topk;
    float scale_log2;        // scale * log2(e)
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

// Launchers (each returns the cudaGetLastError() of its launch).
cudaError_t launch_hash_prefill(const void *K, bool bf16, int64_t n_cap, const float *W,
                                uint32_t *codes, int B, int H_kv, int64_t pos0, int64_t n,
                                cudaStream_t s);
cudaError_t launch_prep(const PrepArgs &a, int rows_per_head, cudaStream_t s);
cudaError_t launch_score(const ScoreArgs &a, cudaStream_t s);
cudaError_t launch_attend(const AttendArgs &a, bool bf16, cudaStream_t s);
cudaError_t launch_dense(const DenseArgs &a, bool bf16, cudaStream_t s);

}  // namespace hata
