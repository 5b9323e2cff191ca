// Decode-attention kernels for head_dim 64, G = 1 query heads per KV head
// (fast code widths 5..8 plus the runtime-width kernel); see kvq_decode_impl.cuh.
#include "kvq_decode_impl.cuh"

namespace kvq {
cudaError_t launch_decode_d64_g1(const DecodeArgs& a, cudaStream_t stream) {
    return launch_decode_dg<64, 1>(a, stream);
}
}  // namespace kvq
