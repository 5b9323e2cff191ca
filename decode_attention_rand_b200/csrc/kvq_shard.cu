// kvq_shard.cu - the merge of context-sharded decode attention.
//
// When the cached context of a sequence is spread over several GPUs (each
// holding a range of its tokens), each GPU runs the split-K decode over its
// own range and stops before the combine (kvq_decode_attn_partials): its
// workspace then holds, per (batch entry, query head, split), the running
// maximum m (log2 units: scores times softmax_scale times log2 e), the
// softmax denominator l = sum 2^(s - m) and the rotated-domain accumulator
// acc = sum 2^(s - m) z^_V.  After an exchange of the workspaces, this kernel
// merges the splits of every part exactly as the single-GPU combine merges
// the splits of one launch:
//     M = max m,  L = sum l 2^(m - M),  z = sum acc 2^(m - M) / L,
// and finishes with the inverse rotation o = D_V H z / sqrt(d) (the
// decode-attention formulas of the codec, "TurboAngle: Near-Lossless KV
// Cache Compression via Uniform Angle Quantization", Abstract).
#include "kvq_internal.h"

namespace kvq {
namespace {

constexpr int kMergeWarpsMax = 8;

// One CTA per (batch entry, query head): warp 0 finds M, L and each split's
// weight 2^(m - M); every thread sums its elements over the splits; the
// Walsh-Hadamard transform runs in shared memory (d <= 256 elements).
__global__ void merge_partials_kernel(const float* __restrict__ parts, int n_parts,
                                      int64_t part_floats, int B, int H_q, int d, int S,
                                      const int8_t* __restrict__ signs_v, void* out,
                                      int out_dtype) {
    extern __shared__ float sh[];
    const int NS = n_parts * S;
    float* w = sh;           // [NS] weights 2^(m - M)
    float* vec = sh + NS;    // [d]
    float* Ls = vec + d;     // [1] L
    const int bq = blockIdx.x;  // b * H_q + h
    const int tid = threadIdx.x, lane = tid & 31;
    const int64_t stat0 = ws_counter_floats(B, H_q);
    const int64_t acc0 = stat0 + ws_stat_floats(B, H_q, S);
    if (tid < 32) {
        float mx = -INFINITY;
        for (int i = lane; i < NS; i += 32) {
            const int p = i / S, s = i % S;
            mx = fmaxf(mx, parts[p * part_floats + stat0 + ((int64_t)bq * S + s) * 2]);
        }
        mx = group_max<32>(mx);
        float sl = 0.f;
        for (int i = lane; i < NS; i += 32) {
            const int p = i / S, s = i % S;
            const float* st = parts + p * part_floats + stat0 + ((int64_t)bq * S + s) * 2;
            const float wi = mx == -INFINITY ? 0.f : exp2f(st[0] - mx);
            w[i] = wi;
            sl = fmaf(wi, st[1], sl);
        }
        sl = group_sum<32>(sl);
        if (lane == 0) Ls[0] = sl;
    }
    __syncthreads();
    const float L = Ls[0];
    const float inv = L > 0.f ? 1.f / L : 0.f;
    for (int j = tid; j < d; j += blockDim.x) {
        float a = 0.f;
        for (int i = 0; i < NS; i++) {
            const int p = i / S, s = i % S;
            a = fmaf(w[i], parts[p * part_floats + acc0 + ((int64_t)bq * S + s) * d + j], a);
        }
        vec[j] = a * inv;
    }
    // inverse rotation: unnormalised Walsh-Hadamard transform, then D_V / sqrt(d)
    for (int h = 1; h < d; h <<= 1) {
        __syncthreads();
        float x[256 / 32];
        int n = 0;
        for (int j = tid; j < d; j += blockDim.x, n++) {
            const float a = vec[j], b = vec[j ^ h];
            x[n] = (j & h) ? b - a : a + b;
        }
        __syncthreads();
        n = 0;
        for (int j = tid; j < d; j += blockDim.x, n++) vec[j] = x[n];
    }
    __syncthreads();
    const float isd = rsqrtf((float)d);
    for (int j = tid; j < d; j += blockDim.x) {
        float o = vec[j] * isd;
        o = signs_v[j] < 0 ? -o : o;
        if (out_dtype == 0)
            reinterpret_cast<__half*>(out)[(int64_t)bq * d + j] = __float2half_rn(o);
        else
            reinterpret_cast<float*>(out)[(int64_t)bq * d + j] = o;
    }
}

}  // namespace

cudaError_t launch_merge_partials(const float* parts, int n_parts, int64_t part_floats, int B,
                                  int H_q, int d, int S, const int8_t* signs_v, void* out,
                                  int out_dtype, cudaStream_t stream) {
    if (B == 0 || H_q == 0) return cudaSuccess;
    int threads = d < 32 ? 32 : d;
    if (threads > 32 * kMergeWarpsMax) threads = 32 * kMergeWarpsMax;
    const size_t smem = sizeof(float) * ((size_t)n_parts * S + d + 1);
    if (smem > 48 * 1024) {
        const cudaError_t e = cudaFuncSetAttribute(
            merge_partials_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    merge_partials_kernel<<<(unsigned)((int64_t)B * H_q), threads, smem, stream>>>(
        parts, n_parts, part_floats, B, H_q, d, S, signs_v, out, out_dtype);
    return cudaGetLastError();
}

}  // namespace kvq
