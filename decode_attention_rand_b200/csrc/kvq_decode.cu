// kvq_decode.cu - dispatch of the decode-attention kernels: the staged kernel
// (kvq_decode_impl.cuh) for head_dim 64/128, G 1/2/4/8, L up to 256 and the
// 8-bit linear K / 4-bit log V norms; the generic kernel
// (kvq_decode_generic.cu) for every other codec.
#include "kvq_internal.h"

#include <atomic>

namespace kvq {

int device_sm_count() {
    static std::atomic<int> cache[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    int n = cache[dev].load();
    if (n <= 0) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            return 148;
        cache[dev].store(n);
    }
    return n;
}

bool decode_fast_supported(int d, int G, int LK, int LV, int mode_k, int mode_v) {
    if (d != 64 && d != 128) return false;
    if (G != 1 && G != 2 && G != 4 && G != 8) return false;
    if (mode_k != KVQ_NORM_LIN8 || mode_v != KVQ_NORM_LOG4) return false;
    return LK >= 2 && LK <= 256 && LV >= 2 && LV <= 256;
}

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t stream) {
    const int G = a.H_q / a.H_kv;
    if (!decode_fast_supported(a.kc.d, G, a.kc.L, a.vc.L, a.kc.mode, a.vc.mode))
        return launch_decode_generic(a, stream);
#define KVQ_DEC_CASE(DD, GG) \
    if (a.kc.d == DD && G == GG) return launch_decode_d##DD##_g##GG(a, stream);
    KVQ_DEC_CASE(64, 1) KVQ_DEC_CASE(64, 2) KVQ_DEC_CASE(64, 4) KVQ_DEC_CASE(64, 8)
    KVQ_DEC_CASE(128, 1) KVQ_DEC_CASE(128, 2) KVQ_DEC_CASE(128, 4) KVQ_DEC_CASE(128, 8)
#undef KVQ_DEC_CASE
    return cudaErrorInvalidValue;
}

}  // namespace kvq
