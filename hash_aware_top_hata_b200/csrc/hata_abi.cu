// hata_abi.cu -- the extern "C" boundary of libhata: argument checks on the
// host, workspace carving, and the launch sequence of each entry point on the
// caller's stream.  Every check runs before anything is enqueued.
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <unordered_map>

#include "hata_internal.cuh"

using namespace hata;

namespace {

thread_local char g_err[512];

// Process-wide settings (hata_set_decode_mode / hata_set_wait_limit_ns).
std::atomic<int> g_mode{HATA_MODE_AUTO};
std::atomic<uint64_t> g_wait_ns{1000000000ull};

// Which steps HATA_MODE_AUTO picks for bf16 caches (the faster ones on B200).
constexpr bool kAutoFused = false;
constexpr bool kAutoCluster = true;

// The fused step serves bf16 K/V caches with codes of up to 128 bits when
// asked for (or chosen by AUTO); fp32 caches and 256-bit codes always take
// the multi-kernel step.
bool use_fused(hata_dtype_t kv_dtype, int r)
{
    const int m = g_mode.load();
    return kv_dtype == HATA_DT_BF16 && r <= kRbit &&
           (m == HATA_MODE_FUSED || (m == HATA_MODE_AUTO && kAutoFused));
}

// The cluster step serves 128-bit codes when the mode asks for it (or AUTO
// picks it) and the sizes fit (cluster_step_plan).
bool want_cluster(hata_dtype_t kv_dtype, int r)
{
    const int m = g_mode.load();
    (void)kv_dtype;
    return r == kRbit && (m == HATA_MODE_CLUSTER || (m == HATA_MODE_AUTO && kAutoCluster));
}

hata_status_t fail(hata_status_t st, const char *fmt, ...)
{
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof g_err, fmt, ap);
    va_end(ap);
    return st;
}

hata_status_t ok()
{
    g_err[0] = '\0';
    return HATA_OK;
}

hata_status_t cuda_fail(cudaError_t e, const char *what)
{
    return fail(HATA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool valid_dtype(hata_dtype_t t) { return t == HATA_DT_BF16 || t == HATA_DT_F32; }

hata_status_t check_dims(int d, int r)
{
    if (d != kD) return fail(HATA_ERR_UNSUPPORTED, "head_dim d=%d: only %d is supported", d, kD);
    if (r != 32 && r != 64 && r != kRbit && r != kRbitWide)
        return fail(HATA_ERR_UNSUPPORTED, "hash bits r=%d: 32, 64, %d or %d are supported", r,
                    kRbit, kRbitWide);
    return HATA_OK;
}

hata_status_t check_heads(int B, int H_q, int H_kv)
{
    if (B <= 0 || H_q <= 0 || H_kv <= 0)
        return fail(HATA_ERR_INVALID_ARG, "B=%d H_q=%d H_kv=%d must be positive", B, H_q, H_kv);
    if (H_q % H_kv != 0)
        return fail(HATA_ERR_UNSUPPORTED, "H_q=%d is not a multiple of H_kv=%d", H_q, H_kv);
    if (int64_t(B) * H_q > 65535 || int64_t(B) * H_kv > 65535)
        return fail(HATA_ERR_UNSUPPORTED, "B*H_q=%lld exceeds 65535",
                    (long long)(int64_t(B) * H_q));
    return HATA_OK;
}

struct Events {
    void *const *ev;
    cudaStream_t s;
    cudaError_t record(int i) const
    {
        return ev ? cudaEventRecord(static_cast<cudaEvent_t>(ev[i]), s) : cudaSuccess;
    }
};

}  // namespace

namespace hata {

hata_status_t report_error(hata_status_t st, const char *msg) { return fail(st, "%s", msg); }

cudaError_t ensure_smem_attr(const void *func, size_t bytes)
{
    static std::mutex mu;
    static std::unordered_map<const void *, uint64_t> done;  // bit d: set on device d
    int dev = 0;
    if (cudaError_t e = cudaGetDevice(&dev)) return e;
    const uint64_t bit = dev < 64 ? uint64_t(1) << dev : 0;
    std::lock_guard<std::mutex> lock(mu);
    if (bit && (done[func] & bit)) return cudaSuccess;
    cudaError_t e =
        cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, int(bytes));
    // every kernel of the step prefers the largest shared-memory carveout, so
    // the SMs keep one L1/shared split from kernel to kernel
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(func, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 int(cudaSharedmemCarveoutMaxShared));
    if (e == cudaSuccess) done[func] |= bit;
    return e;
}

}  // namespace hata

extern "C" {

int hata_abi_version(void) { return 4; }

const char *hata_status_string(int status)
{
    switch (status) {
    case HATA_OK: return "HATA_OK";
    case HATA_ERR_INVALID_ARG: return "HATA_ERR_INVALID_ARG";
    case HATA_ERR_UNSUPPORTED: return "HATA_ERR_UNSUPPORTED";
    case HATA_ERR_CUDA: return "HATA_ERR_CUDA";
    case HATA_ERR_DEVICE_CHECK: return "HATA_ERR_DEVICE_CHECK";
    default: return "HATA_ERR_UNKNOWN";
    }
}

const char *hata_last_error(void) { return g_err; }

hata_status_t hata_set_decode_mode(int mode)
{
    if (mode != HATA_MODE_AUTO && mode != HATA_MODE_MULTI_KERNEL && mode != HATA_MODE_FUSED &&
        mode != HATA_MODE_CLUSTER)
        return fail(HATA_ERR_INVALID_ARG, "decode mode %d", mode);
    g_mode.store(mode);
    return ok();
}

int hata_get_decode_mode(void) { return g_mode.load(); }

hata_status_t hata_set_wait_limit_ns(uint64_t ns)
{
    g_wait_ns.store(ns);
    return ok();
}

hata_status_t hata_hash_keys(const void *K, hata_dtype_t kv_dtype, int64_t k_stride_b,
                             int64_t k_stride_h, int64_t k_stride_n, const float *W_H,
                             uint32_t *codes, int64_t n_cap, int B, int H_kv, int64_t pos0,
                             int64_t n, int d, int r, void *stream)
{
    if (hata_status_t st = check_dims(d, r)) return st;
    if (!K || !W_H || !codes) return fail(HATA_ERR_INVALID_ARG, "null pointer argument");
    if (!valid_dtype(kv_dtype)) return fail(HATA_ERR_INVALID_ARG, "bad kv_dtype %d", int(kv_dtype));
    if (B <= 0 || H_kv <= 0 || B > 65535 || H_kv > 65535)
        return fail(HATA_ERR_INVALID_ARG, "B=%d H_kv=%d out of range", B, H_kv);
    if (n_cap <= 0 || pos0 < 0 || n < 0 || pos0 > n_cap || n > n_cap - pos0)
        return fail(HATA_ERR_INVALID_ARG, "positions [%lld, %lld) outside the cache of %lld",
                    (long long)pos0, (long long)(pos0 + n), (long long)n_cap);
    if (k_stride_b < 0 || k_stride_h < 0 || k_stride_n < d)
        return fail(HATA_ERR_INVALID_ARG,
                    "K strides (%lld, %lld, %lld): non-negative, and rows of d elements must not "
                    "overlap (k_stride_n >= d)",
                    (long long)k_stride_b, (long long)k_stride_h, (long long)k_stride_n);
    const size_t elt = kv_dtype == HATA_DT_BF16 ? 2 : 4;
    if (!aligned(K, elt) || !aligned(codes, 16) || !aligned(W_H, 16))  // 16-byte copies of W_H
        return fail(HATA_ERR_INVALID_ARG,
                    "K must be aligned to its element, codes and W_H to 16 bytes");
    if (n == 0) return ok();
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    const KStrides ks{k_stride_b, k_stride_h, k_stride_n};
    const cudaError_t e = launch_hash_prefill(K, kv_dtype == HATA_DT_BF16, ks, n_cap, W_H, codes,
                                              B, H_kv, pos0, n, r / 32, s);
    return e == cudaSuccess ? ok() : cuda_fail(e, "hash_keys launch");
}

hata_status_t hata_append_code(const void *k_new, hata_dtype_t kv_dtype, const float *W_H,
                               uint32_t *codes, int64_t n_cap, const int32_t *pos, int B,
                               int H_kv, int d, int r, uint32_t *err_flags, void *stream)
{
    if (hata_status_t st = check_dims(d, r)) return st;
    if (!k_new || !W_H || !codes || !pos) return fail(HATA_ERR_INVALID_ARG, "null pointer argument");
    if (!valid_dtype(kv_dtype)) return fail(HATA_ERR_INVALID_ARG, "bad kv_dtype %d", int(kv_dtype));
    if (B <= 0 || H_kv <= 0 || int64_t(B) * H_kv > (int64_t(1) << 24) || H_kv > 65535)
        return fail(HATA_ERR_INVALID_ARG, "B=%d H_kv=%d out of range", B, H_kv);
    if (n_cap <= 0) return fail(HATA_ERR_INVALID_ARG, "n_cap=%lld", (long long)n_cap);
    if (!aligned(k_new, 16) || !aligned(codes, 16) || !aligned(pos, 4) || !aligned(W_H, 16) ||
        (err_flags && !aligned(err_flags, 4)))
        return fail(HATA_ERR_INVALID_ARG, "misaligned pointer (k_new, codes, W_H: 16 B)");
    PrepArgs a{};
    a.k_new = k_new;
    a.W = W_H;
    a.codes = codes;
    a.pos = pos;
    a.err_word = err_flags;
    a.n_cap = n_cap;
    a.max_seq_len = n_cap;
    a.B = B;
    a.H_q = H_kv;
    a.H_kv = H_kv;
    a.G = 1;
    a.kv_bf16 = kv_dtype == HATA_DT_BF16;
    a.words = r / 32;
    const cudaError_t e = launch_prep(a, B, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? ok() : cuda_fail(e, "append_code launch");
}

size_t hata_decode_workspace_size(int B, int H_q, int H_kv, int64_t max_seq_len, int topk)
{
    DecodeLayout L;
    return decode_layout(B, H_q, H_kv, max_seq_len, topk, &L) ? L.total : 0;
}

int64_t hata_dist_row_bytes(int64_t max_seq_len)
{
    return max_seq_len <= 0 ? 0 : ceil_div(max_seq_len, kChunk) * kChunk;
}

int hata_decode_kernel_launches(int B, int H_q, int H_kv, int64_t max_seq_len, int topk,
                                hata_dtype_t kv_dtype, int r)
{
    if (B <= 0 || H_q <= 0 || H_kv <= 0 || H_q % H_kv || max_seq_len <= 0 || topk <= 0 ||
        !valid_dtype(kv_dtype) || (r != 32 && r != 64 && r != kRbit && r != kRbitWide)) {
        fail(HATA_ERR_INVALID_ARG, "B=%d H_q=%d H_kv=%d max_seq_len=%lld topk=%d kv_dtype=%d r=%d",
             B, H_q, H_kv, (long long)max_seq_len, topk, int(kv_dtype), r);
        return -1;
    }
    if (use_fused(kv_dtype, r)) return 3;  // prep, score, the selection + attention kernel
    if (want_cluster(kv_dtype, r)) {
        ClusterPlan plan;
        if (cudaError_t e = cluster_step_plan(B, H_q, H_kv, max_seq_len, topk,
                                              kv_dtype == HATA_DT_BF16, &plan)) {
            cuda_fail(e, "cluster occupancy query");
            return -1;
        }
        if (plan.kM) return 1;
    }
    int n = 0;
    if (cudaError_t e = attend_launch_count(B, H_q, topk, kv_dtype == HATA_DT_BF16, &n)) {
        cuda_fail(e, "occupancy query");
        return -1;
    }
    return 3 + n;
}

}  // extern "C"

namespace {

// The checks every step entry point shares: sizes, the caches, the
// workspace.  Fills the workspace layout.
hata_status_t check_step(const uint32_t *codes, const void *K, const void *V,
                         hata_dtype_t kv_dtype, int64_t n_cap, const int32_t *seq_len,
                         int64_t max_seq_len, int B, int H_q, int H_kv, int d, int r, int topk,
                         void *workspace, size_t workspace_bytes, DecodeLayout *L)
{
    if (hata_status_t st = check_dims(d, r)) return st;
    if (hata_status_t st = check_heads(B, H_q, H_kv)) return st;
    if (!codes || !K || !V || !seq_len || !workspace)
        return fail(HATA_ERR_INVALID_ARG, "null pointer argument");
    if (!valid_dtype(kv_dtype)) return fail(HATA_ERR_INVALID_ARG, "bad kv_dtype %d", int(kv_dtype));
    if (topk <= 0) return fail(HATA_ERR_INVALID_ARG, "topk=%d must be >= 1", topk);
    if (n_cap <= 0 || n_cap >= (int64_t(1) << 31))
        return fail(HATA_ERR_INVALID_ARG, "n_cap=%lld out of range", (long long)n_cap);
    if (max_seq_len <= 0 || max_seq_len > n_cap)
        return fail(HATA_ERR_INVALID_ARG, "max_seq_len=%lld must be in [1, n_cap=%lld]",
                    (long long)max_seq_len, (long long)n_cap);
    if (!aligned(K, 16) || !aligned(V, 16) || !aligned(codes, 16) || !aligned(seq_len, 4))
        return fail(HATA_ERR_INVALID_ARG, "misaligned pointer (K, V, codes: 16 B)");
    if (!aligned(workspace, 256)) return fail(HATA_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
    if (!decode_layout(B, H_q, H_kv, max_seq_len, topk, L))
        return fail(HATA_ERR_INVALID_ARG, "sizes out of range");
    if (workspace_bytes < L->total)
        return fail(HATA_ERR_INVALID_ARG, "workspace of %zu bytes < required %zu", workspace_bytes,
                    L->total);
    return HATA_OK;
}

hata_status_t check_scale(float scale)
{
    if (!(scale == scale) || scale > 3.0e38f || scale < -3.0e38f)
        return fail(HATA_ERR_INVALID_ARG, "scale must be finite");
    return HATA_OK;
}

// Where a step's intermediate results live.
struct StepBufs {
    uint32_t *qc;      // query codes [B][H_q][r/32]
    uint8_t *dist;     // distance rows
    int64_t drow;      // their stride
    int32_t *idx;      // index lists [B][H_q][topk]
    uint32_t *flags, *hist;
    float *q_dev;      // device copy of q
};

StepBufs step_bufs(char *ws, const DecodeLayout &L, uint32_t *q_codes, uint8_t *dist,
                   int64_t dist_row_bytes, int32_t *sel_idx)
{
    StepBufs sb;
    sb.qc = q_codes ? q_codes : reinterpret_cast<uint32_t *>(ws + L.off_qcodes);
    sb.dist = dist ? dist : reinterpret_cast<uint8_t *>(ws + L.off_dist);
    sb.drow = dist ? dist_row_bytes : L.dist_row;
    sb.idx = sel_idx ? sel_idx : reinterpret_cast<int32_t *>(ws + L.off_idx);
    sb.flags = reinterpret_cast<uint32_t *>(ws + L.off_flags);
    sb.hist = reinterpret_cast<uint32_t *>(ws + L.off_hist);
    sb.q_dev = reinterpret_cast<float *>(ws + L.off_q);
    return sb;
}

// The front of a step: prep (hash q, append, clear the histograms, flags),
// then the scoring kernel.  Events 0..2 around them.
hata_status_t enqueue_front(const float *q, const float *W_H, uint32_t *codes, void *K, void *V,
                            hata_dtype_t kv_dtype, int64_t n_cap, const int32_t *seq_len,
                            int64_t max_seq_len, const void *k_new, const void *v_new, int B,
                            int H_q, int H_kv, int r, const DecodeLayout &L, const StepBufs &sb,
                            char *ws, uint32_t *sync, const Events &ev)
{
    const cudaStream_t s = ev.s;
    const int G = H_q / H_kv;
    cudaError_t e;
    if ((e = ev.record(0)) != cudaSuccess) return cuda_fail(e, "event record");
    PrepArgs p{};
    p.q = q;
    p.q_copy = sb.q_dev;
    p.k_new = k_new;
    p.v_new = v_new;
    p.W = W_H;
    p.codes = codes;
    p.K = K;
    p.V = V;
    p.seq_len = seq_len;
    p.q_out = sb.qc;
    p.flags = sb.flags;
    p.hist = sb.hist;
    p.hist_row_words = L.n_tiles * hist_stride(r / 32);
    p.sync = sync;
    p.ws_header = reinterpret_cast<uint32_t *>(ws);
    p.n_cap = n_cap;
    p.max_seq_len = max_seq_len;
    p.B = B;
    p.H_q = H_q;
    p.H_kv = H_kv;
    p.G = G;
    p.kv_bf16 = kv_dtype == HATA_DT_BF16;
    p.words = r / 32;
    if ((e = launch_prep(p, B * G + (k_new ? B : 0), s)) != cudaSuccess)
        return cuda_fail(e, "prep launch");
    if ((e = ev.record(1)) != cudaSuccess) return cuda_fail(e, "event record");

    ScoreArgs sa{};
    sa.qcodes = sb.qc;
    sa.codes = codes;
    sa.seq_len = seq_len;
    sa.dist = sb.dist;
    sa.dist_row = sb.drow;
    sa.hist = sb.hist;
    sa.n_cap = n_cap;
    sa.max_seq_len = max_seq_len;
    sa.n_tiles = L.n_tiles;
    sa.B = B;
    sa.H_q = H_q;
    sa.H_kv = H_kv;
    sa.G = G;
    sa.zgroups = L.zgroups;
    sa.words = r / 32;
    if ((e = launch_score(sa, s)) != cudaSuccess) return cuda_fail(e, "score launch");
    if ((e = ev.record(2)) != cudaSuccess) return cuda_fail(e, "event record");
    return HATA_OK;
}

SelectArgs select_args(const StepBufs &sb, const uint32_t *codes, const int32_t *seq_len,
                       int64_t n_cap, int64_t max_seq_len, const DecodeLayout &L, int B, int H_q,
                       int H_kv, int r, int topk)
{
    SelectArgs se{};
    se.seq_len = seq_len;
    se.dist = sb.dist;
    se.dist_row = sb.drow;
    se.hist = sb.hist;
    se.idx = sb.idx;
    se.qcodes = sb.qc;
    se.codes = codes;
    se.n_cap = n_cap;
    se.max_seq_len = max_seq_len;
    se.n_tiles = L.n_tiles;
    se.B = B;
    se.H_q = H_q;
    se.H_kv = H_kv;
    se.G = H_q / H_kv;
    se.topk = topk;
    se.words = r / 32;
    return se;
}

AttendArgs attend_args(const StepBufs &sb, const void *K, const void *V, const int32_t *seq_len,
                       int64_t n_cap, int64_t max_seq_len, char *ws, const DecodeLayout &L, int B,
                       int H_q, int H_kv, int topk, float scale, float *out)
{
    AttendArgs aa{};
    aa.q = sb.q_dev;
    aa.K = K;
    aa.V = V;
    aa.seq_len = seq_len;
    aa.idx = sb.idx;
    aa.part = reinterpret_cast<float *>(ws + L.off_part);
    aa.flags = sb.flags;
    aa.out = out;
    aa.n_cap = n_cap;
    aa.max_seq_len = max_seq_len;
    aa.B = B;
    aa.H_q = H_q;
    aa.H_kv = H_kv;
    aa.G = H_q / H_kv;
    aa.topk = topk;
    aa.n_split = L.n_split;
    aa.scale_log2 = scale * 1.4426950408889634f;
    return aa;
}

}  // namespace

extern "C" {

hata_status_t hata_decode_step(const float *q, const float *W_H, uint32_t *codes, void *K,
                               void *V, hata_dtype_t kv_dtype, int64_t n_cap,
                               const int32_t *seq_len, int64_t max_seq_len, const void *k_new,
                               const void *v_new, int B, int H_q, int H_kv, int d, int r,
                               int topk, float scale, void *workspace, size_t workspace_bytes,
                               float *out, int32_t *sel_idx, uint32_t *q_codes, uint8_t *dist,
                               int64_t dist_row_bytes, void *const *events, void *stream)
{
    DecodeLayout L;
    if (hata_status_t st = check_step(codes, K, V, kv_dtype, n_cap, seq_len, max_seq_len, B, H_q,
                                      H_kv, d, r, topk, workspace, workspace_bytes, &L))
        return st;
    if (!q || !W_H || !out) return fail(HATA_ERR_INVALID_ARG, "null pointer argument");
    if (v_new && !k_new) return fail(HATA_ERR_INVALID_ARG, "v_new given without k_new");
    if (hata_status_t st = check_scale(scale)) return st;
    if (!aligned(q, 16) || !aligned(out, 16) || !aligned(W_H, 16) ||
        (k_new && !aligned(k_new, 16)) || (v_new && !aligned(v_new, 16)) ||
        (sel_idx && !aligned(sel_idx, 4)) || (q_codes && !aligned(q_codes, 16)))
        return fail(HATA_ERR_INVALID_ARG,
                    "misaligned pointer (q, W_H, K, V, codes, out, k_new, v_new, q_codes: 16 B)");
    if (dist) {
        if (!aligned(dist, 16) || dist_row_bytes % 16 || dist_row_bytes < L.dist_row)
            return fail(HATA_ERR_INVALID_ARG,
                        "dist must be 16-byte aligned with dist_row_bytes >= %lld, multiple of 16",
                        (long long)L.dist_row);
    }

    char *ws = static_cast<char *>(workspace);
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    const StepBufs sb = step_bufs(ws, L, q_codes, dist, dist_row_bytes, sel_idx);
    const Events ev{events, s};
    cudaError_t e;
    if (want_cluster(kv_dtype, r)) {
        ClusterPlan plan;
        if ((e = cluster_step_plan(B, H_q, H_kv, max_seq_len, topk, kv_dtype == HATA_DT_BF16,
                                   &plan)) != cudaSuccess)
            return cuda_fail(e, "cluster occupancy query");
        if (plan.kM) {
            ClusterArgs ca{};
            ca.q = q;
            ca.W = W_H;
            ca.codes = codes;
            ca.K = K;
            ca.V = V;
            ca.k_new = k_new;
            ca.v_new = v_new;
            ca.seq_len = seq_len;
            ca.q_out = q_codes;
            ca.dist = dist;
            ca.dist_row = dist_row_bytes;
            ca.idx = sb.idx;
            ca.out = out;
            ca.flags = sb.flags;
            ca.ws_header = reinterpret_cast<uint32_t *>(ws);
            ca.n_cap = n_cap;
            ca.max_seq_len = max_seq_len;
            ca.B = B;
            ca.H_q = H_q;
            ca.H_kv = H_kv;
            ca.G = H_q / H_kv;
            ca.topk = topk;
            ca.tok_per_cta = plan.tok_per_cta;
            ca.kv_bf16 = kv_dtype == HATA_DT_BF16;
            ca.scale_log2 = scale * 1.4426950408889634f;
            if ((e = ev.record(0)) != cudaSuccess) return cuda_fail(e, "event record");
            if ((e = launch_cluster_step(ca, plan, s)) != cudaSuccess)
                return cuda_fail(e, "cluster step launch");
            // one kernel does the work of all five: its end is recorded for each
            for (int i = 1; i <= 5; ++i)
                if ((e = ev.record(i)) != cudaSuccess) return cuda_fail(e, "event record");
            return ok();
        }
    }
    const bool fused = use_fused(kv_dtype, r);
    uint32_t *sync = reinterpret_cast<uint32_t *>(ws + L.off_sync);
    if (hata_status_t st = enqueue_front(q, W_H, codes, K, V, kv_dtype, n_cap, seq_len,
                                         max_seq_len, k_new, v_new, B, H_q, H_kv, r, L, sb, ws,
                                         fused ? sync : nullptr, ev))
        return st;

    if (fused) {
        FusedArgs fa{};
        fa.seq_len = seq_len;
        fa.q = sb.q_dev;
        fa.K = K;
        fa.V = V;
        fa.dist = sb.dist;
        fa.hist = sb.hist;
        fa.idx = sb.idx;
        fa.part = reinterpret_cast<float *>(ws + L.off_part);
        fa.out = out;
        fa.sel_done = sync;
        fa.head_cnt = sync + int64_t(B) * H_q;
        fa.flags = sb.flags;
        fa.abort_word = sync + 2 * int64_t(B) * H_q;
        fa.dist_row = sb.drow;
        fa.dist_len = L.dist_row;
        fa.n_cap = n_cap;
        fa.max_seq_len = max_seq_len;
        fa.n_tiles = int(L.n_tiles);
        fa.B = B;
        fa.H_q = H_q;
        fa.H_kv = H_kv;
        fa.G = H_q / H_kv;
        fa.topk = topk;
        fa.n_seg = L.n_seg;
        fa.scale_log2 = scale * 1.4426950408889634f;
        fa.spin_limit_ns = g_wait_ns.load();
        if ((e = launch_fused(fa, s)) != cudaSuccess) return cuda_fail(e, "fused launch");
        // one kernel does the work of the select, attend and combine kernels:
        // its end is recorded for all three
        for (int i = 3; i <= 5; ++i)
            if ((e = ev.record(i)) != cudaSuccess) return cuda_fail(e, "event record");
        return ok();
    }

    const SelectArgs se =
        select_args(sb, codes, seq_len, n_cap, max_seq_len, L, B, H_q, H_kv, r, topk);
    if ((e = launch_select(se, s)) != cudaSuccess) return cuda_fail(e, "select launch");
    if ((e = ev.record(3)) != cudaSuccess) return cuda_fail(e, "event record");

    AttendArgs aa = attend_args(sb, K, V, seq_len, n_cap, max_seq_len, ws, L, B, H_q, H_kv, topk,
                                scale, out);
    if ((e = launch_attend(aa, kv_dtype == HATA_DT_BF16, s)) != cudaSuccess)
        return cuda_fail(e, "attend launch");
    if ((e = ev.record(4)) != cudaSuccess) return cuda_fail(e, "event record");
    if ((e = launch_combine(aa, s)) != cudaSuccess) return cuda_fail(e, "combine launch");
    if ((e = ev.record(5)) != cudaSuccess) return cuda_fail(e, "event record");
    return ok();
}

hata_status_t hata_sp_score(const float *q, const float *W_H, uint32_t *codes, void *K, void *V,
                            hata_dtype_t kv_dtype, int64_t n_cap, const int32_t *seq_len,
                            int64_t max_seq_len, const void *k_new, const void *v_new, int B,
                            int H_q, int H_kv, int d, int r, int topk, void *workspace,
                            size_t workspace_bytes, uint32_t *hist_out, void *stream)
{
    DecodeLayout L;
    if (hata_status_t st = check_step(codes, K, V, kv_dtype, n_cap, seq_len, max_seq_len, B, H_q,
                                      H_kv, d, r, topk, workspace, workspace_bytes, &L))
        return st;
    if (!q || !W_H || !hist_out) return fail(HATA_ERR_INVALID_ARG, "null pointer argument");
    if (v_new && !k_new) return fail(HATA_ERR_INVALID_ARG, "v_new given without k_new");
    if (!aligned(q, 16) || !aligned(W_H, 16) || !aligned(hist_out, 4) ||
        (k_new && !aligned(k_new, 16)) || (v_new && !aligned(v_new, 16)))
        return fail(HATA_ERR_INVALID_ARG, "misaligned pointer (q, W_H, k_new, v_new: 16 B)");
    char *ws = static_cast<char *>(workspace);
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    const StepBufs sb = step_bufs(ws, L, nullptr, nullptr, 0, nullptr);
    const Events ev{nullptr, s};
    if (hata_status_t st = enqueue_front(q, W_H, codes, K, V, kv_dtype, n_cap, seq_len,
                                         max_seq_len, k_new, v_new, B, H_q, H_kv, r, L, sb, ws,
                                         nullptr, ev))
        return st;
    const cudaError_t e = launch_sp_hist(sb.hist, L.n_tiles, hist_stride(r / 32),
                                         int64_t(B) * H_q, hist_out, s);
    return e == cudaSuccess ? ok() : cuda_fail(e, "histogram launch");
}

hata_status_t hata_sp_attend(const uint32_t *hist_all, int world, int rank,
                             const uint32_t *codes, const void *K, const void *V,
                             hata_dtype_t kv_dtype, int64_t n_cap, const int32_t *seq_len,
                             int64_t max_seq_len, int B, int H_q, int H_kv, int d, int r,
                             int topk, float scale, void *workspace, size_t workspace_bytes,
                             float *part_out, int32_t *sel_idx, void *stream)
{
    DecodeLayout L;
    if (hata_status_t st = check_step(codes, K, V, kv_dtype, n_cap, seq_len, max_seq_len, B, H_q,
                                      H_kv, d, r, topk, workspace, workspace_bytes, &L))
        return st;
    if (!hist_all || !part_out) return fail(HATA_ERR_INVALID_ARG, "null pointer argument");
    if (world < 1 || rank < 0 || rank >= world)
        return fail(HATA_ERR_INVALID_ARG, "rank %d of world %d", rank, world);
    if (hata_status_t st = check_scale(scale)) return st;
    if (!aligned(hist_all, 4) || !aligned(part_out, 16) || (sel_idx && !aligned(sel_idx, 4)))
        return fail(HATA_ERR_INVALID_ARG, "misaligned pointer (part_out: 16 B)");
    char *ws = static_cast<char *>(workspace);
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    const StepBufs sb = step_bufs(ws, L, nullptr, nullptr, 0, sel_idx);
    int32_t *k_head = reinterpret_cast<int32_t *>(ws + L.off_khead);
    const int64_t BH = int64_t(B) * H_q;
    cudaError_t e = launch_sp_quota(hist_all, world, rank, BH, topk, r + 1, k_head, s);
    if (e != cudaSuccess) return cuda_fail(e, "quota launch");
    SelectArgs se =
        select_args(sb, codes, seq_len, n_cap, max_seq_len, L, B, H_q, H_kv, r, topk);
    se.k_head = k_head;
    if ((e = launch_select(se, s)) != cudaSuccess) return cuda_fail(e, "select launch");
    AttendArgs aa = attend_args(sb, K, V, seq_len, n_cap, max_seq_len, ws, L, B, H_q, H_kv, topk,
                                scale, nullptr);
    aa.k_head = k_head;
    aa.part_out = part_out;
    aa.n_split = L.n_split > L.n_seg ? L.n_split : L.n_seg;  // partial slots per head
    e = kv_dtype == HATA_DT_BF16 ? launch_attend_split(aa, s) : launch_attend(aa, false, s);
    if (e != cudaSuccess) return cuda_fail(e, "attend launch");
    if ((e = launch_combine(aa, s)) != cudaSuccess) return cuda_fail(e, "combine launch");
    return ok();
}

hata_status_t hata_sp_merge(const float *part_all, int world, int B, int H_q, float *out,
                            void *stream)
{
    if (!part_all || !out) return fail(HATA_ERR_INVALID_ARG, "null pointer argument");
    if (world < 1 || B <= 0 || H_q <= 0 || int64_t(B) * H_q > 65535)
        return fail(HATA_ERR_INVALID_ARG, "world=%d B=%d H_q=%d", world, B, H_q);
    if (!aligned(part_all, 16) || !aligned(out, 16))
        return fail(HATA_ERR_INVALID_ARG, "part_all and out must be 16-byte aligned");
    const cudaError_t e =
        launch_sp_merge(part_all, world, int64_t(B) * H_q, out, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? ok() : cuda_fail(e, "merge launch");
}

hata_status_t hata_workspace_check(void *workspace, size_t workspace_bytes, uint32_t *flags,
                                   void *stream)
{
    if (flags) *flags = 0;
    if (!workspace || workspace_bytes < 512 || !aligned(workspace, 256))
        return fail(HATA_ERR_INVALID_ARG, "bad workspace");
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint32_t hdr[2] = {0, 0};
    cudaError_t e = cudaMemcpyAsync(hdr, workspace, sizeof hdr, cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(e, "workspace header read");
    if (hdr[0] != kWsMagic) return ok();  // no decode step has run on it
    const uint32_t B = hdr[1];
    if (B == 0 || 256 + 4 * size_t(B) > workspace_bytes)
        return fail(HATA_ERR_INVALID_ARG, "workspace header does not match its size");
    uint32_t acc = 0;
    char *fl = static_cast<char *>(workspace) + 256;
    for (uint32_t b0 = 0; b0 < B; b0 += 256) {
        uint32_t buf[256];
        const uint32_t cnt = B - b0 < 256 ? B - b0 : 256;
        e = cudaMemcpyAsync(buf, fl + 4 * size_t(b0), 4 * size_t(cnt), cudaMemcpyDeviceToHost, s);
        if (e == cudaSuccess) e = cudaStreamSynchronize(s);
        if (e != cudaSuccess) return cuda_fail(e, "workspace flag read");
        for (uint32_t i = 0; i < cnt; ++i) acc |= buf[i];
    }
    e = cudaMemsetAsync(fl, 0, 4 * size_t(B), s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(e, "workspace flag clear");
    if (flags) *flags = acc;
    if (acc) return fail(HATA_ERR_DEVICE_CHECK, "device-side check flags 0x%x", acc);
    return ok();
}

size_t hata_dense_workspace_size(int B, int H_q, int H_kv, int64_t max_seq_len)
{
    int64_t nch;
    size_t op, oc, tot;
    return dense_layout(B, H_q, H_kv, max_seq_len, &nch, &op, &oc, &tot) ? tot : 0;
}

hata_status_t hata_dense_decode(const float *q, const void *K, const void *V,
                                hata_dtype_t kv_dtype, int64_t n_cap, const int32_t *seq_len,
                                int64_t max_seq_len, int B, int H_q, int H_kv, int d,
                                float scale, void *workspace, size_t workspace_bytes, float *out,
                                void *stream)
{
    if (hata_status_t st = check_dims(d, kRbit)) return st;
    if (hata_status_t st = check_heads(B, H_q, H_kv)) return st;
    if (!q || !K || !V || !seq_len || !workspace || !out)
        return fail(HATA_ERR_INVALID_ARG, "null pointer argument");
    if (!valid_dtype(kv_dtype)) return fail(HATA_ERR_INVALID_ARG, "bad kv_dtype %d", int(kv_dtype));
    if (n_cap <= 0 || n_cap >= (int64_t(1) << 31) || max_seq_len <= 0 || max_seq_len > n_cap)
        return fail(HATA_ERR_INVALID_ARG, "max_seq_len=%lld n_cap=%lld out of range",
                    (long long)max_seq_len, (long long)n_cap);
    if (!aligned(q, 16) || !aligned(K, 16) || !aligned(V, 16) || !aligned(out, 4) ||
        !aligned(seq_len, 4) || !aligned(workspace, 256))
        return fail(HATA_ERR_INVALID_ARG, "misaligned pointer");
    int64_t nch;
    size_t off_part, off_cnt, total;
    if (!dense_layout(B, H_q, H_kv, max_seq_len, &nch, &off_part, &off_cnt, &total))
        return fail(HATA_ERR_INVALID_ARG, "sizes out of range");
    if (workspace_bytes < total)
        return fail(HATA_ERR_INVALID_ARG, "workspace of %zu bytes < required %zu", workspace_bytes,
                    total);
    char *ws = static_cast<char *>(workspace);
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    DenseArgs a{};
    a.q = q;
    a.K = K;
    a.V = V;
    a.seq_len = seq_len;
    a.part = reinterpret_cast<float *>(ws + off_part);
    a.cnt = reinterpret_cast<uint32_t *>(ws + off_cnt);
    a.out = out;
    a.n_cap = n_cap;
    a.max_seq_len = max_seq_len;
    a.n_chunks = nch;
    a.B = B;
    a.H_q = H_q;
    a.H_kv = H_kv;
    a.G = H_q / H_kv;
    a.zgroups = int(ceil_div(a.G, kDenseHeads));
    a.scale_log2 = scale * 1.4426950408889634f;
    cudaError_t e = cudaMemsetAsync(a.cnt, 0, total - off_cnt, s);
    if (e != cudaSuccess) return cuda_fail(e, "dense counter clear");
    e = launch_dense(a, kv_dtype == HATA_DT_BF16, s);
    return e == cudaSuccess ? ok() : cuda_fail(e, "dense launch");
}

}  // extern "C"
