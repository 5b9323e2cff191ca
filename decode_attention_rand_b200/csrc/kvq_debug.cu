// kvq_debug.cu - the cache integrity check of KVQ_DEBUG, and the NVTX ranges
// of KVQ_PROFILE.
//
// With checks on (environment variable KVQ_DEBUG set to anything but "0", or
// kvq_test_control(KVQ_TEST_DEBUG_CHECKS, 1)), every decode first scans the
// rows it is about to read, tokens 0 .. ctx_len[b]-1 of every (b, KV head)
// of K and V, for values the encoder never writes: an angle code >= L (a
// codebook that is not a power of two leaves 2^b - L bit patterns unused), a
// non-finite fp16 parameter (the streaming encoder marks a vector it could not
// settle with a NaN until its fixup pass rewrites it), a LOG4 vector with
// HI < LO, a LIN8 vector with a negative M.  A hit sets KVQ_DEVERR_BAD_CODE in
// the call's err_word; nothing else changes.  The check reads every byte the
// decode reads (it doubles the call's memory traffic) and is meant for
// debugging a cache, not for serving.
#include <stdlib.h>
#include <string.h>

#include <atomic>

#include <nvtx3/nvToolsExt.h>

#include "kvq_internal.h"

namespace kvq {
namespace {

std::atomic<int> g_checks{-1};  // -1: not read from the environment yet

__device__ __forceinline__ bool bad_half(uint16_t h) { return (h & 0x7C00u) == 0x7C00u; }

// One warp per (token, KV head, batch entry, K|V) row group.
__global__ void __launch_bounds__(256) check_kernel(DecodeArgs A) {
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t lim = A.max_ctx < A.K.capacity ? A.max_ctx : A.K.capacity;
    const int kvh = blockIdx.y, b = blockIdx.z;
    int64_t ctx = A.ctx_len[b];
    ctx = ctx < 0 ? 0 : (ctx > lim ? lim : ctx);
    // a decode step appends row ctx - 1 after this check: not written yet
    if (A.k_new && ctx > 0) ctx--;
    const int nwarps = gridDim.x * blockDim.x / 32;
    bool bad = false;
    for (int64_t t = warp; t < ctx; t += nwarps) {
        for (int which = 0; which < 2; which++) {
            const CodecDev& c = which == 0 ? A.kc : A.vc;
            const PlaneDev& p = which == 0 ? A.K : A.V;
            bool badrow = false;
            const int64_t row = plane_row(p, b, kvh, t, &badrow);
            if (badrow) continue;  // reported by the decode itself
            const uint32_t* aw = reinterpret_cast<const uint32_t*>(p.angles) + row * c.angle_words;
            if (c.L < (1 << c.bits)) {
                for (int i = lane; i < c.d / 2; i += 32) {
                    const int pos = i * c.bits, wi = pos >> 5, sh = pos & 31;
                    const uint32_t hi = sh + c.bits > 32 ? aw[wi + 1] : 0u;
                    const uint32_t code = __funnelshift_r(aw[wi], hi, sh) & ((1u << c.bits) - 1u);
                    bad |= code >= (uint32_t)c.L;
                }
            }
            if (lane == 0) {
                if (c.mode == KVQ_NORM_LIN8) {
                    const uint16_t m = reinterpret_cast<const uint16_t*>(p.params)[row];
                    bad |= bad_half(m) || (m & 0x8000u) != 0;
                } else {
                    const uint32_t pr = reinterpret_cast<const uint32_t*>(p.params)[row];
                    const uint16_t lo = (uint16_t)(pr & 0xFFFF), hi = (uint16_t)(pr >> 16);
                    bad |= bad_half(lo) || bad_half(hi) ||
                           half_bits_to_float(hi) < half_bits_to_float(lo);
                }
            }
        }
    }
    if (__any_sync(KVQ_FULL_MASK, bad) && lane == 0) report(A.err_word, KVQ_DEVERR_BAD_CODE);
}

bool env_on(const char* name) {
    const char* v = getenv(name);
    return v && *v && strcmp(v, "0") != 0;
}

}  // namespace

bool debug_checks_on() {
    int v = g_checks.load();
    if (v < 0) {
        v = env_on("KVQ_DEBUG") ? 1 : 0;
        int expect = -1;
        g_checks.compare_exchange_strong(expect, v);
        v = g_checks.load();
    }
    return v > 0;
}

void set_debug_checks(int on) { g_checks.store(on < 0 ? -1 : (on ? 1 : 0)); }

cudaError_t launch_cache_check(const DecodeArgs& a, cudaStream_t stream) {
    if (!a.err_word || a.B == 0 || a.H_kv == 0) return cudaSuccess;
    check_kernel<<<dim3(16, (unsigned)a.H_kv, (unsigned)a.B), 256, 0, stream>>>(a);
    return cudaGetLastError();
}

bool profile_on() {
    static const bool on = env_on("KVQ_PROFILE");
    return on;
}

ProfileRange::ProfileRange(const char* name) : on(profile_on()) {
    if (on) nvtxRangePushA(name);
}

ProfileRange::~ProfileRange() {
    if (on) nvtxRangePop();
}

}  // namespace kvq
