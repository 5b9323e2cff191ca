// kvq_internal.h - declarations shared between the kvq kernels and the C ABI
// layer (not installed; the public interface is include/kvq.h).
#pragma once

#include "kvq_common.cuh"

namespace kvq {

cudaError_t launch_encode(const CodecDev& c, const int8_t* signs, const __half* x, int64_t n_vec,
                          int64_t T, int64_t pos0, const PlaneDev& out, int sm_count,
                          cudaStream_t stream);

// One tensor's share of an encode launch.
struct EncodeJob {
    CodecDev c;
    const int8_t* signs;
    const __half* x;
    int64_t n_vec;  // B * H_kv * T
    int64_t T;
    int64_t pos0;
    PlaneDev out;
    int32_t* err_word;  // device error bits, or NULL
};

// One launch for one or two jobs of the same head_dim (K and V appended
// together); a job with n_vec 0 is skipped.
cudaError_t launch_encode_jobs(const EncodeJob* jobs, int n_jobs, int sm_count,
                               cudaStream_t stream);

cudaError_t launch_dequant(const CodecDev& c, const int8_t* signs, const PlaneDev& in,
                           int64_t n_vec, int64_t T, int64_t pos0, __half* y, int sm_count,
                           cudaStream_t stream);

// One encode job as the kernels see it (built on the host by make_args).
struct EncArgs {
    const __half* x;
    const int8_t* signs;
    int64_t n_vec;
    int64_t T;
    int64_t pos0;
    CodecDev c;
    PlaneDev out;
    float inv_sqrt_d;
    float bins_per_rad;  // L / (2 pi)
    int64_t bh0;         // (b * H_kv + h) of vector 0; vector v is sequence bh0 + v / T
    int32_t* err_word;   // device error bits (page-table range), or NULL
    FastDiv tdiv;        // division by T
    int small;           // n_vec and T below 2^32: v / T through tdiv
};

// Codec-wide part of an encode job (x, n_vec, T, pos0 and out left empty).
EncArgs encode_args(const CodecDev& c, const int8_t* signs);

struct DecodeArgs {
    const __half* q;        // [B][H_q][d]
    CodecDev kc, vc;
    const int8_t* signs_k;
    const int8_t* signs_v;
    PlaneDev K, V;
    const int32_t* ctx_len;  // [B]
    int B, H_q, H_kv;
    int64_t max_ctx;
    float scale_log2;        // softmax_scale * log2(e)
    int num_splits;
    int64_t split_len;       // tokens per split, multiple of 16
    float* ws;               // counters [B*H_q] int32, stats [B][H_q][S][2], acc [B][H_q][S][d]
    int32_t* err_word;
    void* out;
    int out_dtype;
    // shared-memory staging layout, filled by the launcher
    int lay[6];              // byte offsets of the six arrays inside a stage
    int stage_bytes;
    int stage_offset;
    int nstages;             // ring depth
    int cluster;             // 1: the splits of a (b, KV head) form one thread-block
                             // cluster and combine through distributed shared memory
    // fused append (kvq_decode_step): the new token of every (b, KV head),
    // encoded by the CTA whose split holds position ctx_len[b] - 1
    uint32_t wait_limit;     // tries before a tile wait gives up (kvq_test_control)
    // 1: the new token's rows are being written by append_kernel, the launch
    // this one is a programmatic dependent of; that kernel starts its
    // dependents only once everything before it has completed, so this one
    // reads q and ctx_len at once and waits for the append (griddepcontrol)
    // only before copying in the tile that holds the new row
    int append_pending;
    // 1 (kvq_decode_attn_partials): stop after the per-split partials are in
    // the workspace; no combine, no output (cluster is 0)
    int partials_only;
    const __half* k_new;     // [B][H_kv][d] or NULL (no append)
    const __half* v_new;     // [B][H_kv][d]
    EncArgs enc_k, enc_v;    // codec, signs and constants of the two encodes
};

// True when the staged decode kernel is built for this (head_dim, G, L_K,
// L_V) and norm-mode combination; the generic kernel takes every other one.
bool decode_fast_supported(int d, int G, int LK, int LV, int mode_k, int mode_v);

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t stream);
// Merge of the split partials of n_parts workspaces laid out back to back
// (kvq_decode_merge_partials): out[b][h] from every part's splits.
cudaError_t launch_merge_partials(const float* parts, int n_parts, int64_t part_floats, int B,
                                  int H_q, int d, int S, const int8_t* signs_v, void* out,
                                  int out_dtype, cudaStream_t stream);
cudaError_t launch_decode_generic(const DecodeArgs& a, cudaStream_t stream);
cudaError_t launch_decode_d64_g1(const DecodeArgs& a, cudaStream_t stream);
cudaError_t launch_decode_d64_g2(const DecodeArgs& a, cudaStream_t stream);
cudaError_t launch_decode_d64_g4(const DecodeArgs& a, cudaStream_t stream);
cudaError_t launch_decode_d64_g8(const DecodeArgs& a, cudaStream_t stream);
cudaError_t launch_decode_d128_g1(const DecodeArgs& a, cudaStream_t stream);
cudaError_t launch_decode_d128_g2(const DecodeArgs& a, cudaStream_t stream);
cudaError_t launch_decode_d128_g4(const DecodeArgs& a, cudaStream_t stream);
cudaError_t launch_decode_d128_g8(const DecodeArgs& a, cudaStream_t stream);

// KVQ_DEBUG cache integrity check (kvq_debug.cu): on when the environment
// variable is set (or by kvq_test_control); launched before each decode.
bool debug_checks_on();
void set_debug_checks(int on);  // 1 on, 0 off, -1 back to the environment
cudaError_t launch_cache_check(const DecodeArgs& a, cudaStream_t stream);

// KVQ_PROFILE: an NVTX range around each call's launches when the environment
// variable is set.
struct ProfileRange {
    bool on;
    explicit ProfileRange(const char* name);
    ~ProfileRange();
};

// SM count of the current device (cached per device; 148 if unknown).
int device_sm_count();

// Default number of tries of a bounded mbarrier wait.
constexpr uint32_t kWaitLimit = 1u << 22;

// Set the calling thread's kvq_last_error() message; returns `code`.
int record_error(int code, const char* msg);

// Workspace layout helpers (host and device agree through these): completion
// counters of the fused combine (int32, zero between calls), then per split
// (m, l) pairs, then per split rotated-domain accumulators.
__host__ __device__ inline int64_t ws_counter_floats(int B, int H_q) {
    return ((int64_t)B * H_q + 3) / 4 * 4;
}
__host__ __device__ inline int64_t ws_stat_floats(int B, int H_q, int S) {
    return ((int64_t)B * H_q * S * 2 + 3) / 4 * 4;  // keeps the accumulators 16-byte aligned
}
__host__ __device__ inline int64_t ws_acc_floats(int B, int H_q, int S, int d) { return (int64_t)B * H_q * S * d; }

}  // namespace kvq
