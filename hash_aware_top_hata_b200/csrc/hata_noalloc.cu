// hata_noalloc.cu -- hata_decode_step for callers that cannot allocate.
//
// Some callers may not call cudaMalloc: a plugin inside a serving engine
// that hands all device memory to its own pool, or code on a latency-critical
// path where cudaMalloc's implicit device synchronisation is not allowed.
// They can still pass their inputs and outputs; this entry point supplies the
// decode scratch from a fixed array in the library's own device image.
//
// The array is a file-scope static __device__ buffer of
// HATA_NOALLOC_WORKSPACE_BYTES; every GPU that loads the library holds it
// until the process exits.  Host code must not use the array's name as a
// device address (in host code it is only a stand-in symbol), so the first
// call on each device looks the real address up with cudaGetSymbolAddress,
// with that device current, and caches it.
#include <cstdio>
#include <mutex>

#include "hata_internal.cuh"

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[HATA_NOALLOC_WORKSPACE_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_scratch_ptr[kMaxDevices] = {};

thread_local char g_msg[256];

}  // namespace

extern "C" hata_status_t hata_decode_step_noalloc(
    const float *q, const float *W_H, uint32_t *codes, void *K, void *V, hata_dtype_t kv_dtype,
    int64_t n_cap, const int32_t *seq_len, int64_t max_seq_len, const void *k_new,
    const void *v_new, int B, int H_q, int H_kv, int d, int r, int topk, float scale, float *out,
    int32_t *sel_idx, uint32_t *q_codes, uint8_t *dist, int64_t dist_row_bytes,
    void *const *events, void *stream)
{
    const size_t need = hata_decode_workspace_size(B, H_q, H_kv, max_seq_len, topk);
    if (need == 0) return hata::report_error(HATA_ERR_INVALID_ARG, "sizes out of range");
    if (need > size_t(HATA_NOALLOC_WORKSPACE_BYTES)) {
        snprintf(g_msg, sizeof g_msg,
                 "decode scratch of %zu bytes exceeds the fixed no-alloc buffer of %u bytes",
                 need, unsigned(HATA_NOALLOC_WORKSPACE_BYTES));
        return hata::report_error(HATA_ERR_INVALID_ARG, g_msg);
    }
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return hata::report_error(HATA_ERR_CUDA, "no usable current device");
    void *ws = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_mu);
        if (!g_scratch_ptr[dev]) {
            void *p = nullptr;
            if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p)
                return hata::report_error(HATA_ERR_CUDA, "cudaGetSymbolAddress of the scratch failed");
            g_scratch_ptr[dev] = p;
        }
        ws = g_scratch_ptr[dev];
    }
    return hata_decode_step(q, W_H, codes, K, V, kv_dtype, n_cap, seq_len, max_seq_len, k_new,
                            v_new, B, H_q, H_kv, d, r, topk, scale, ws,
                            size_t(HATA_NOALLOC_WORKSPACE_BYTES), out, sel_idx, q_codes, dist,
                            dist_row_bytes, events, stream);
}
