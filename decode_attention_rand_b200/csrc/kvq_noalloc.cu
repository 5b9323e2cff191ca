// kvq_noalloc.cu - kvq_decode_attn_noalloc: decode attention for callers that
// cannot allocate device memory.
//
// kvq_decode_attn needs a caller-provided workspace (split partials and
// completion counters).  Some callers cannot call cudaMalloc to get one: a
// serving loop that has handed all device memory to its own pooling
// allocator, a plain C host program with no allocator of its own, or code
// that must not risk the device-wide synchronisation or the out-of-memory
// failure a fresh allocation can bring.  This entry point takes its scratch
// from a fixed array compiled into the library instead.
//
// The array lives in device memory of every GPU that loads the library and
// stays there until the process exits.  Host code cannot use the array's name
// as a device address, so the first call on each device (with that device
// current) looks the address up once with cudaGetSymbolAddress and keeps it;
// make that first call before any stream capture.  Every call shares the one
// array and finds the previous call's contents there: each call clears the
// completion counters at its start (an asynchronous memset on `stream`), and
// calls whose kernels overlap on the GPU (different streams, or two threads)
// race on the array and must be ordered by the caller.
#include <mutex>
#include <stdio.h>

#include "kvq_internal.h"

namespace {

__device__ __align__(256) unsigned char g_kvq_scratch[KVQ_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_lock;
void* g_scratch_ptr[kMaxDevices] = {};

}  // namespace

extern "C" {

int kvq_decode_attn_noalloc(const void* q, const kvq_codec* kc, const kvq_codec* vc,
                            const int8_t* signs_k, const int8_t* signs_v, const kvq_plane* K,
                            const kvq_plane* V, const int32_t* ctx_len, int32_t B, int32_t H_q,
                            int32_t H_kv, int64_t max_ctx, float softmax_scale, int32_t num_splits,
                            int32_t* err_word, void* out, int32_t out_dtype, void* stream) {
    char msg[256];
    if (!kc) return kvq::record_error(KVQ_EINVAL, "kvq_decode_attn_noalloc: codec is NULL");
    const int64_t need = kvq_decode_workspace_bytes(B, H_q, kc->head_dim, num_splits);
    if (need > (int64_t)KVQ_NOALLOC_SCRATCH_BYTES) {
        snprintf(msg, sizeof(msg),
                 "kvq_decode_attn_noalloc: this call needs %lld bytes of scratch, more than the "
                 "%lld bytes built into the library; use fewer splits or kvq_decode_attn",
                 (long long)need, (long long)KVQ_NOALLOC_SCRATCH_BYTES);
        return kvq::record_error(KVQ_EINVAL, msg);
    }
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        snprintf(msg, sizeof(msg), "kvq_decode_attn_noalloc: no usable current device (%s)",
                 cudaGetErrorName(e));
        return kvq::record_error(KVQ_ECUDA, msg);
    }
    void* ptr = nullptr;
    {
        std::lock_guard<std::mutex> guard(g_lock);
        if (!g_scratch_ptr[dev]) {
            void* p = nullptr;
            e = cudaGetSymbolAddress(&p, g_kvq_scratch);
            if (e != cudaSuccess || !p) {
                snprintf(msg, sizeof(msg),
                         "kvq_decode_attn_noalloc: cudaGetSymbolAddress of the scratch failed (%s)",
                         cudaGetErrorName(e));
                return kvq::record_error(KVQ_ECUDA, msg);
            }
            g_scratch_ptr[dev] = p;
        }
        ptr = g_scratch_ptr[dev];
    }
    if (B > 0 && H_q > 0 && need > 0) {
        // the completion counters (first bytes of the workspace) must start at zero
        const size_t counter_bytes = (size_t)(((int64_t)B * H_q + 3) / 4) * 16;
        e = cudaMemsetAsync(ptr, 0, counter_bytes, static_cast<cudaStream_t>(stream));
        if (e != cudaSuccess) {
            snprintf(msg, sizeof(msg), "kvq_decode_attn_noalloc: clearing the counters failed (%s)",
                     cudaGetErrorName(e));
            return kvq::record_error(KVQ_ECUDA, msg);
        }
    }
    return kvq_decode_attn(q, kc, vc, signs_k, signs_v, K, V, ctx_len, B, H_q, H_kv, max_ctx,
                           softmax_scale, num_splits, ptr, (int64_t)KVQ_NOALLOC_SCRATCH_BYTES,
                           err_word, out, out_dtype, stream);
}

}  // extern "C"
