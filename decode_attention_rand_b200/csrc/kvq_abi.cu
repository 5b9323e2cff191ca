// kvq_abi.cu - the C ABI of include/kvq.h: argument checks, launch choice,
// error reporting.  Every compute step runs in the kernels of this library.
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <atomic>

#include "kvq_internal.h"

namespace {

thread_local char g_err[512] = "";

// kvq_test_control state: launches still to be failed, and the tile-wait
// limit of decode kernels plus one (0: the default limit).
std::atomic<int64_t> g_fail_launches{0};
std::atomic<int64_t> g_wait_limit_p1{0};

int fail(int code, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof(g_err), fmt, ap);
    va_end(ap);
    return code;
}

int ok() {
    g_err[0] = '\0';
    return KVQ_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool pow2(int v) { return v > 0 && (v & (v - 1)) == 0; }

int sm_count_current() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
        return 148;
    return n;
}

// Validate a codec and fill the device descriptor.  d_min/d_max bound head_dim.
int check_codec(const kvq_codec* c, const char* what, kvq::CodecDev* out) {
    if (!c) return fail(KVQ_EINVAL, "%s: codec is NULL", what);
    if (!pow2(c->head_dim) || c->head_dim < 4 || c->head_dim > 256)
        return fail(KVQ_EINVAL, "%s: head_dim %d is not a power of two in 4..256", what, c->head_dim);
    const int b = kvq_angle_bits(c->L);
    if (b < 0) return fail(KVQ_EINVAL, "%s: L = %d outside 2..65536", what, c->L);
    if (c->norm_mode != KVQ_NORM_LIN8 && c->norm_mode != KVQ_NORM_LOG4)
        return fail(KVQ_EINVAL, "%s: unknown norm_mode %d", what, c->norm_mode);
    out->d = c->head_dim;
    out->L = c->L;
    out->bits = b;
    out->mode = c->norm_mode;
    out->angle_words = (int)(kvq_row_bytes(c, 0) / 4);
    out->norm_bytes = (int)kvq_row_bytes(c, 1);
    out->param_bytes = (int)kvq_row_bytes(c, 2);
    return KVQ_OK;
}

int check_plane(const kvq_plane* p, const char* what, kvq::PlaneDev* out) {
    if (!p) return fail(KVQ_EINVAL, "%s: plane is NULL", what);
    if (!p->angles || !p->norms || !p->params)
        return fail(KVQ_EINVAL, "%s: NULL plane array", what);
    if (!aligned16(p->angles) || !aligned16(p->norms) || !aligned16(p->params))
        return fail(KVQ_EINVAL, "%s: plane arrays must be 16-byte aligned", what);
    if (p->capacity <= 0 || p->capacity % 16 != 0)
        return fail(KVQ_EINVAL, "%s: capacity %lld must be a positive multiple of 16", what,
                    (long long)p->capacity);
    out->angles = static_cast<uint8_t*>(p->angles);
    out->norms = static_cast<uint8_t*>(p->norms);
    out->params = static_cast<uint8_t*>(p->params);
    out->capacity = p->capacity;
    out->H_kv = 0;  // set by the call
    out->pages = nullptr;
    out->page_tokens = 0;
    out->max_pages = 0;
    out->num_pages = 0;
    return KVQ_OK;
}

// Validate a paged plane and fill the device descriptor.
int check_paged_plane(const kvq_paged_plane* p, const char* what, kvq::PlaneDev* out) {
    if (!p) return fail(KVQ_EINVAL, "%s: paged plane is NULL", what);
    if (!p->angles || !p->norms || !p->params || !p->pages)
        return fail(KVQ_EINVAL, "%s: NULL pool or page table", what);
    if (!aligned16(p->angles) || !aligned16(p->norms) || !aligned16(p->params))
        return fail(KVQ_EINVAL, "%s: pools must be 16-byte aligned", what);
    if (p->page_tokens <= 0 || p->page_tokens % 128 != 0)
        return fail(KVQ_EINVAL, "%s: page_tokens %d must be a positive multiple of 128", what,
                    p->page_tokens);
    if (p->max_pages <= 0 || p->num_pages <= 0)
        return fail(KVQ_EINVAL, "%s: max_pages and num_pages must be positive", what);
    out->angles = static_cast<uint8_t*>(p->angles);
    out->norms = static_cast<uint8_t*>(p->norms);
    out->params = static_cast<uint8_t*>(p->params);
    out->capacity = (int64_t)p->max_pages * p->page_tokens;
    out->H_kv = 0;
    out->pages = p->pages;
    out->page_tokens = p->page_tokens;
    out->max_pages = p->max_pages;
    out->num_pages = p->num_pages;
    return KVQ_OK;
}

int cuda_status(cudaError_t e, const char* what) {
    if (e != cudaSuccess)
        return fail(KVQ_ECUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
    return ok();
}

// A launch that kvq_test_control asked to fail: consumes one and reports it
// the way a failed launch is reported (nothing is queued).
bool injected_failure() {
    int64_t n = g_fail_launches.load();
    while (n > 0)
        if (g_fail_launches.compare_exchange_weak(n, n - 1)) return true;
    return false;
}

int injected(const char* what) {
    return fail(KVQ_ECUDA, "%s: cudaErrorLaunchFailure (launch failure injected by "
                "kvq_test_control)", what);
}

}  // namespace

namespace kvq {
int record_error(int code, const char* msg) { return fail(code, "%s", msg); }
}  // namespace kvq

extern "C" {

int32_t kvq_version(void) { return 1 * 10000 + 1 * 100 + 0; }

int kvq_test_control(int32_t key, int64_t value) {
    if (value < 0) return fail(KVQ_EINVAL, "kvq_test_control: negative value");
    switch (key) {
        case KVQ_TEST_RESET:
            g_fail_launches.store(0);
            g_wait_limit_p1.store(0);
            kvq::set_debug_checks(-1);
            return ok();
        case KVQ_TEST_DEBUG_CHECKS: kvq::set_debug_checks(value ? 1 : 0); return ok();
        case KVQ_TEST_FAIL_LAUNCHES: g_fail_launches.store(value); return ok();
        case KVQ_TEST_WAIT_LIMIT:
            g_wait_limit_p1.store((value < 0xFFFFFFFFll ? value : 0xFFFFFFFFll - 1) + 1);
            return ok();
        default: return fail(KVQ_EINVAL, "kvq_test_control: unknown key %d", key);
    }
}

const char* kvq_last_error(void) { return g_err; }

int32_t kvq_angle_bits(int32_t L) {
    if (L < 2 || L > 65536) return KVQ_EINVAL;
    int32_t b = 1;
    while ((1L << b) < (long)L) b++;
    return b;
}

int64_t kvq_row_bytes(const kvq_codec* c, int32_t which) {
    if (!c || !pow2(c->head_dim) || c->head_dim < 4 || c->head_dim > 256) return KVQ_EINVAL;
    const int32_t b = kvq_angle_bits(c->L);
    if (b < 0) return KVQ_EINVAL;
    const int64_t P = c->head_dim / 2;
    switch (which) {
        case 0: return 4 * ((P * b + 31) / 32);
        case 1:
            if (c->norm_mode == KVQ_NORM_LIN8) return P;
            if (c->norm_mode == KVQ_NORM_LOG4) return P / 2;
            return KVQ_EINVAL;
        case 2:
            if (c->norm_mode == KVQ_NORM_LIN8) return 2;
            if (c->norm_mode == KVQ_NORM_LOG4) return 4;
            return KVQ_EINVAL;
        default: return KVQ_EINVAL;
    }
}

}  // extern "C"

namespace {

// Argument checks of one encode job; *job->n_vec is 0 when there is nothing
// to encode.
int prep_encode(const kvq_codec* codec, const int8_t* signs, const void* x, int32_t B,
                int32_t H_kv, int32_t T, int64_t pos0, const kvq_plane* out, const char* what,
                const char* xname, kvq::EncodeJob* job, const kvq_paged_plane* paged = nullptr) {
    int rc = check_codec(codec, what, &job->c);
    if (rc) return rc;
    rc = paged ? check_paged_plane(paged, what, &job->out) : check_plane(out, what, &job->out);
    if (rc) return rc;
    job->out.H_kv = H_kv;
    job->out.hdiv = kvq::make_fast_div(H_kv > 0 ? (uint32_t)H_kv : 1u);
    job->err_word = nullptr;
    if (B < 0 || H_kv < 0 || T < 0) return fail(KVQ_EINVAL, "%s: negative size", what);
    if (paged && (int64_t)B * H_kv >= (1ll << 31))
        return fail(KVQ_EINVAL, "%s: B * H_kv must be below 2^31 for a paged plane", what);
    if (pos0 < 0 || pos0 + (int64_t)T > job->out.capacity)
        return fail(KVQ_EINVAL, "%s: tokens [%lld, %lld) exceed capacity %lld", what,
                    (long long)pos0, (long long)(pos0 + T), (long long)job->out.capacity);
    job->n_vec = (int64_t)B * H_kv * T;
    job->T = T;
    job->pos0 = pos0;
    job->signs = signs;
    job->x = static_cast<const __half*>(x);
    if (job->n_vec == 0) return KVQ_OK;
    if (!signs || !x) return fail(KVQ_EINVAL, "%s: NULL signs or %s", what, xname);
    if (!aligned16(x)) return fail(KVQ_EINVAL, "%s: %s must be 16-byte aligned", what, xname);
    return KVQ_OK;
}

}  // namespace

extern "C" {

int kvq_encode(const kvq_codec* codec, const int8_t* signs, const void* x, int32_t B, int32_t H_kv,
               int32_t T, int64_t pos0, const kvq_plane* out, void* stream) {
    kvq::EncodeJob j;
    const int rc = prep_encode(codec, signs, x, B, H_kv, T, pos0, out, "kvq_encode", "x", &j);
    if (rc) return rc;
    if (j.n_vec == 0) return ok();
    if (injected_failure()) return injected("kvq_encode");
    kvq::ProfileRange range("kvq_encode");
    return cuda_status(kvq::launch_encode_jobs(&j, 1, sm_count_current(),
                                               static_cast<cudaStream_t>(stream)),
                       "kvq_encode");
}

int kvq_encode_kv(const kvq_codec* kc, const int8_t* signs_k, const void* k, const kvq_plane* K,
                  const kvq_codec* vc, const int8_t* signs_v, const void* v, const kvq_plane* V,
                  int32_t B, int32_t H_kv, int32_t T, int64_t pos0, void* stream) {
    kvq::EncodeJob j[2];
    int rc = prep_encode(kc, signs_k, k, B, H_kv, T, pos0, K, "kvq_encode_kv", "k", &j[0]);
    if (rc) return rc;
    rc = prep_encode(vc, signs_v, v, B, H_kv, T, pos0, V, "kvq_encode_kv", "v", &j[1]);
    if (rc) return rc;
    if (j[0].c.d != j[1].c.d)
        return fail(KVQ_EINVAL, "kvq_encode_kv: K head_dim %d differs from V head_dim %d",
                    j[0].c.d, j[1].c.d);
    if (j[0].n_vec == 0) return ok();
    if (injected_failure()) return injected("kvq_encode_kv");
    kvq::ProfileRange range("kvq_encode_kv");
    return cuda_status(kvq::launch_encode_jobs(j, 2, sm_count_current(),
                                               static_cast<cudaStream_t>(stream)),
                       "kvq_encode_kv");
}

int kvq_encode_kv_paged(const kvq_codec* kc, const int8_t* signs_k, const void* k,
                        const kvq_paged_plane* K, const kvq_codec* vc, const int8_t* signs_v,
                        const void* v, const kvq_paged_plane* V, int32_t B, int32_t H_kv,
                        int32_t T, int64_t pos0, int32_t* err_word, void* stream) {
    kvq::EncodeJob j[2];
    int rc = prep_encode(kc, signs_k, k, B, H_kv, T, pos0, nullptr, "kvq_encode_kv_paged", "k",
                         &j[0], K);
    if (rc) return rc;
    rc = prep_encode(vc, signs_v, v, B, H_kv, T, pos0, nullptr, "kvq_encode_kv_paged", "v", &j[1],
                     V);
    if (rc) return rc;
    if (j[0].c.d != j[1].c.d)
        return fail(KVQ_EINVAL, "kvq_encode_kv_paged: K head_dim %d differs from V head_dim %d",
                    j[0].c.d, j[1].c.d);
    if (j[0].n_vec == 0) return ok();
    j[0].err_word = j[1].err_word = err_word;
    if (injected_failure()) return injected("kvq_encode_kv_paged");
    kvq::ProfileRange range("kvq_encode_kv_paged");
    return cuda_status(kvq::launch_encode_jobs(j, 2, sm_count_current(),
                                               static_cast<cudaStream_t>(stream)),
                       "kvq_encode_kv_paged");
}

int kvq_dequant(const kvq_codec* codec, const int8_t* signs, const kvq_plane* in, int32_t B,
                int32_t H_kv, int32_t T, int64_t pos0, void* y, void* stream) {
    kvq::CodecDev c;
    kvq::PlaneDev p;
    int rc = check_codec(codec, "kvq_dequant", &c);
    if (rc) return rc;
    rc = check_plane(in, "kvq_dequant", &p);
    if (rc) return rc;
    if (B < 0 || H_kv < 0 || T < 0) return fail(KVQ_EINVAL, "kvq_dequant: negative size");
    if (pos0 < 0 || pos0 + (int64_t)T > p.capacity)
        return fail(KVQ_EINVAL, "kvq_dequant: tokens [%lld, %lld) exceed capacity %lld",
                    (long long)pos0, (long long)(pos0 + T), (long long)p.capacity);
    const int64_t n = (int64_t)B * H_kv * T;
    if (n == 0) return ok();
    if (!signs || !y) return fail(KVQ_EINVAL, "kvq_dequant: NULL signs or y");
    if (!aligned16(y)) return fail(KVQ_EINVAL, "kvq_dequant: y must be 16-byte aligned");
    if (injected_failure()) return injected("kvq_dequant");
    kvq::ProfileRange range("kvq_dequant");
    return cuda_status(kvq::launch_dequant(c, signs, p, n, T, pos0, static_cast<__half*>(y),
                                           sm_count_current(), static_cast<cudaStream_t>(stream)),
                       "kvq_dequant");
}

int32_t kvq_decode_num_splits(int32_t B, int32_t H_kv, int64_t max_ctx, int32_t sm_count) {
    // One CTA runs per SM; a CTA's time is its tokens (the block loop skips
    // what is past its split) plus a fixed cost (prologue, the first tile's
    // copy, merge, combine) of about 512 tokens' worth.  The launch takes
    // waves x (tokens per CTA + 512); pick the split count that minimises it,
    // the fewer CTAs on ties.  Splits are at least 128 tokens long.
    if (B <= 0 || H_kv <= 0 || max_ctx <= 0 || sm_count <= 0) return 1;
    const int64_t units = (int64_t)B * H_kv;
    const int64_t tiles = (max_ctx + 127) / 128;
    int64_t max_s = tiles < 65535 ? tiles : 65535;
    // beyond eight waves the model's gains are noise
    const int64_t wave_cap = (8 * (int64_t)sm_count + units - 1) / units;
    if (max_s > wave_cap) max_s = wave_cap;
    if (max_s < 1) max_s = 1;
    int64_t best = 1, best_cost = -1;
    for (int64_t s = 1; s <= max_s; s++) {
        const int64_t waves = (units * s + sm_count - 1) / sm_count;
        const int64_t per_cta = (max_ctx + s - 1) / s;
        const int64_t cost = waves * (per_cta + 512);
        if (best_cost < 0 || cost < best_cost) {
            best_cost = cost;
            best = s;
        }
    }
    return (int32_t)best;
}

int64_t kvq_decode_workspace_bytes(int32_t B, int32_t H_q, int32_t head_dim, int32_t num_splits) {
    if (B < 0 || H_q < 0 || head_dim <= 0 || num_splits <= 0) return KVQ_EINVAL;
    return (int64_t)sizeof(float) * (kvq::ws_counter_floats(B, H_q) +
                                     kvq::ws_stat_floats(B, H_q, num_splits) +
                                     kvq::ws_acc_floats(B, H_q, num_splits, head_dim));
}

}  // extern "C"

namespace {

// Argument checks and launch of a decode, with (kvq_decode_step) or without
// (kvq_decode_attn) the fused append of the new token.
// Host buffers of kvq_decode_step_host: copied in after the argument checks
// and before the launch, copied out after it.
struct HostIO {
    const void* in_host;
    int64_t in_bytes;
    void* out_host;
    int64_t out_bytes;
};

int decode_impl(const char* what, const void* q, const void* k_new, const void* v_new,
                const kvq_codec* kc, const kvq_codec* vc, const int8_t* signs_k,
                const int8_t* signs_v, const kvq_plane* K, const kvq_plane* V,
                const int32_t* ctx_len, int32_t B, int32_t H_q, int32_t H_kv, int64_t max_ctx,
                float softmax_scale, int32_t num_splits, void* workspace, int64_t ws_bytes,
                int32_t* err_word, void* out, int32_t out_dtype, void* stream,
                const kvq_paged_plane* PK = nullptr, const kvq_paged_plane* PV = nullptr,
                const HostIO* hio = nullptr, bool partials = false) {
    char wk[64], wv[64];
    snprintf(wk, sizeof(wk), "%s (K)", what);
    snprintf(wv, sizeof(wv), "%s (V)", what);
    kvq::DecodeArgs a = {};
    int rc = check_codec(kc, wk, &a.kc);
    if (rc) return rc;
    rc = check_codec(vc, wv, &a.vc);
    if (rc) return rc;
    const bool paged = PK != nullptr;
    rc = paged ? check_paged_plane(PK, wk, &a.K) : check_plane(K, wk, &a.K);
    if (rc) return rc;
    rc = paged ? check_paged_plane(PV, wv, &a.V) : check_plane(V, wv, &a.V);
    if (rc) return rc;
    a.K.H_kv = a.V.H_kv = H_kv;
    a.K.hdiv = a.V.hdiv = kvq::make_fast_div(H_kv > 0 ? (uint32_t)H_kv : 1u);
    if (a.kc.d != a.vc.d) return fail(KVQ_EINVAL, "%s: K and V head_dim differ", what);
    if (a.K.capacity != a.V.capacity)
        return fail(KVQ_EINVAL, "%s: K and V capacity differ", what);
    if (B < 0 || H_q < 0 || H_kv < 0 || max_ctx < 0)
        return fail(KVQ_EINVAL, "%s: negative size", what);
    if (B == 0 || H_q == 0) return ok();
    if (B > 65535 || H_kv > 65535)
        return fail(KVQ_EINVAL, "%s: B and H_kv must be at most 65535", what);
    if (H_kv <= 0 || H_q % H_kv != 0)
        return fail(KVQ_EINVAL, "%s: H_q %d is not a multiple of H_kv %d", what, H_q, H_kv);
    if (num_splits < 1 || num_splits > 65535)
        return fail(KVQ_EINVAL, "%s: num_splits %d outside 1..65535", what, num_splits);
    if (out_dtype != 0 && out_dtype != 1)
        return fail(KVQ_EINVAL, "%s: out_dtype must be 0 (fp16) or 1 (fp32)", what);
    if (!(softmax_scale == softmax_scale) || softmax_scale > 3.0e38f || softmax_scale < -3.0e38f)
        return fail(KVQ_EINVAL, "%s: softmax_scale is not finite", what);
    const int64_t need = kvq_decode_workspace_bytes(B, H_q, a.kc.d, num_splits);
    if (!workspace || ws_bytes < need)
        return fail(KVQ_EINVAL, "%s: workspace of %lld bytes is below the %lld needed", what,
                    (long long)ws_bytes, (long long)need);
    if (!aligned16(workspace)) return fail(KVQ_EINVAL, "%s: workspace not 16-byte aligned", what);
    if (!q || !signs_k || !signs_v || !ctx_len || (!out && !partials))
        return fail(KVQ_EINVAL, "%s: NULL q, signs, ctx_len or out", what);
    a.q = static_cast<const __half*>(q);
    a.signs_k = signs_k;
    a.signs_v = signs_v;
    a.ctx_len = ctx_len;
    a.B = B;
    a.H_q = H_q;
    a.H_kv = H_kv;
    a.max_ctx = max_ctx;
    a.scale_log2 = softmax_scale * 1.4426950408889634f;
    a.num_splits = num_splits;
    int64_t sl = (max_ctx + num_splits - 1) / num_splits;
    // paged: splits start on whole 128-token tiles, so no staged tile crosses a page
    const int64_t gran = paged ? 128 : 16;
    sl = (sl + gran - 1) / gran * gran;
    a.split_len = sl < gran ? gran : sl;
    // the kernels count a split's tokens in 32 bits (2^30 tokens of codes are
    // already more than a GPU holds)
    if (a.split_len > (1ll << 30))
        return fail(KVQ_EINVAL, "%s: a split of %lld tokens exceeds 2^30; raise num_splits", what,
                    (long long)a.split_len);
    a.ws = static_cast<float*>(workspace);
    a.err_word = err_word;
    a.out = out;
    a.out_dtype = out_dtype;
    a.partials_only = partials ? 1 : 0;
    a.k_new = static_cast<const __half*>(k_new);
    a.v_new = static_cast<const __half*>(v_new);
    if (k_new) {
        a.enc_k = kvq::encode_args(a.kc, signs_k);
        a.enc_v = kvq::encode_args(a.vc, signs_v);
    }
    const int64_t wl = g_wait_limit_p1.load();
    a.wait_limit = wl > 0 ? (uint32_t)(wl - 1) : kvq::kWaitLimit;
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (injected_failure()) return injected(what);
    kvq::ProfileRange range(what);
    int rc2;
    if (hio && hio->in_bytes > 0) {
        rc2 = cuda_status(cudaMemcpyAsync(const_cast<void*>(q), hio->in_host, (size_t)hio->in_bytes,
                                          cudaMemcpyHostToDevice, st), what);
        if (rc2) return rc2;
    }
    if (kvq::debug_checks_on()) {
        rc2 = cuda_status(kvq::launch_cache_check(a, st), what);
        if (rc2) return rc2;
    }
    rc2 = cuda_status(kvq::launch_decode(a, st), what);
    if (rc2 || !hio || hio->out_bytes <= 0) return rc2;
    return cuda_status(
        cudaMemcpyAsync(hio->out_host, out, (size_t)hio->out_bytes, cudaMemcpyDeviceToHost, st),
        what);
}

}  // namespace

extern "C" {

int kvq_decode_attn(const void* q, const kvq_codec* kc, const kvq_codec* vc, const int8_t* signs_k,
                    const int8_t* signs_v, const kvq_plane* K, const kvq_plane* V,
                    const int32_t* ctx_len, int32_t B, int32_t H_q, int32_t H_kv, int64_t max_ctx,
                    float softmax_scale, int32_t num_splits, void* workspace, int64_t ws_bytes,
                    int32_t* err_word, void* out, int32_t out_dtype, void* stream) {
    return decode_impl("kvq_decode_attn", q, nullptr, nullptr, kc, vc, signs_k, signs_v, K, V,
                       ctx_len, B, H_q, H_kv, max_ctx, softmax_scale, num_splits, workspace,
                       ws_bytes, err_word, out, out_dtype, stream);
}

int kvq_decode_attn_partials(const void* q, const kvq_codec* kc, const kvq_codec* vc,
                             const int8_t* signs_k, const int8_t* signs_v, const kvq_plane* K,
                             const kvq_plane* V, const int32_t* ctx_len, int32_t B, int32_t H_q,
                             int32_t H_kv, int64_t max_ctx, float softmax_scale,
                             int32_t num_splits, void* workspace, int64_t ws_bytes,
                             int32_t* err_word, void* stream) {
    return decode_impl("kvq_decode_attn_partials", q, nullptr, nullptr, kc, vc, signs_k, signs_v,
                       K, V, ctx_len, B, H_q, H_kv, max_ctx, softmax_scale, num_splits,
                       workspace, ws_bytes, err_word, nullptr, 1, stream, nullptr, nullptr,
                       nullptr, true);
}

int kvq_decode_merge_partials(const void* parts, int32_t n_parts, int32_t B, int32_t H_q,
                              int32_t head_dim, int32_t num_splits, const int8_t* signs_v,
                              void* out, int32_t out_dtype, void* stream) {
    const char* what = "kvq_decode_merge_partials";
    if (n_parts < 1 || n_parts > 4096)
        return fail(KVQ_EINVAL, "%s: n_parts %d outside 1..4096", what, n_parts);
    if (B < 0 || H_q < 0) return fail(KVQ_EINVAL, "%s: negative size", what);
    if (head_dim < 4 || head_dim > 256 || (head_dim & (head_dim - 1)))
        return fail(KVQ_EINVAL, "%s: head_dim %d is not a power of two in 4..256", what,
                    head_dim);
    if (num_splits < 1 || num_splits > 65535)
        return fail(KVQ_EINVAL, "%s: num_splits %d outside 1..65535", what, num_splits);
    if ((int64_t)n_parts * num_splits > 16384)
        return fail(KVQ_EINVAL, "%s: n_parts x num_splits above 16384", what);
    if (out_dtype != 0 && out_dtype != 1)
        return fail(KVQ_EINVAL, "%s: out_dtype must be 0 (fp16) or 1 (fp32)", what);
    if (B == 0 || H_q == 0) return ok();
    if (!parts || !signs_v || !out) return fail(KVQ_EINVAL, "%s: NULL parts, signs or out", what);
    if (!aligned16(parts)) return fail(KVQ_EINVAL, "%s: parts not 16-byte aligned", what);
    const int64_t part_floats = kvq_decode_workspace_bytes(B, H_q, head_dim, num_splits) / 4;
    if (injected_failure()) return injected(what);
    kvq::ProfileRange range(what);
    return cuda_status(kvq::launch_merge_partials(static_cast<const float*>(parts), n_parts,
                                                  part_floats, B, H_q, head_dim, num_splits,
                                                  signs_v, out, out_dtype,
                                                  static_cast<cudaStream_t>(stream)),
                       what);
}

int kvq_decode_step(const void* q, const void* k_new, const void* v_new, const kvq_codec* kc,
                    const kvq_codec* vc, const int8_t* signs_k, const int8_t* signs_v,
                    const kvq_plane* K, const kvq_plane* V, const int32_t* ctx_len, int32_t B,
                    int32_t H_q, int32_t H_kv, int64_t max_ctx, float softmax_scale,
                    int32_t num_splits, void* workspace, int64_t ws_bytes, int32_t* err_word,
                    void* out, int32_t out_dtype, void* stream) {
    if (!k_new || !v_new) return fail(KVQ_EINVAL, "kvq_decode_step: NULL k_new or v_new");
    if (!aligned16(k_new) || !aligned16(v_new))
        return fail(KVQ_EINVAL, "kvq_decode_step: k_new and v_new must be 16-byte aligned");
    return decode_impl("kvq_decode_step", q, k_new, v_new, kc, vc, signs_k, signs_v, K, V,
                       ctx_len, B, H_q, H_kv, max_ctx, softmax_scale, num_splits, workspace,
                       ws_bytes, err_word, out, out_dtype, stream);
}

int kvq_decode_step_host(const void* in_host, void* in_dev, void* out_host, void* out_dev,
                         const kvq_codec* kc, const kvq_codec* vc, const int8_t* signs_k,
                         const int8_t* signs_v, const kvq_plane* K, const kvq_plane* V,
                         const int32_t* ctx_len, int32_t B, int32_t H_q, int32_t H_kv,
                         int64_t max_ctx, float softmax_scale, int32_t num_splits,
                         void* workspace, int64_t ws_bytes, int32_t* err_word, int32_t out_dtype,
                         void* stream) {
    const char* what = "kvq_decode_step_host";
    if (!in_host || !out_host) return fail(KVQ_EINVAL, "%s: NULL host buffer", what);
    const bool mapped = !in_dev && !out_dev;
    if (!mapped && (!in_dev || !out_dev))
        return fail(KVQ_EINVAL, "%s: give both device buffers or neither", what);
    if (!kc) return fail(KVQ_EINVAL, "%s (K): codec is NULL", what);
    if (B < 0 || H_q < 0 || H_kv < 0) return fail(KVQ_EINVAL, "%s: negative size", what);
    const int64_t d = kc->head_dim;
    const int64_t nq = (int64_t)B * H_q * d, nkv = (int64_t)B * H_kv * d;
    if ((nq * 2) % 16 != 0 || (nkv * 2) % 16 != 0)
        return fail(KVQ_EINVAL, "%s: q and k_new sizes must be multiples of 16 bytes", what);
    if (mapped) {
        // the kernel reads the inputs from, and writes the output to, host
        // memory that the device can address: page-locked memory only
        void* dev_ptr[2] = {nullptr, nullptr};
        const void* host[2] = {in_host, out_host};
        for (int i = 0; i < 2; i++) {
            cudaPointerAttributes at;
            if (cudaPointerGetAttributes(&at, host[i]) != cudaSuccess ||
                at.type != cudaMemoryTypeHost || !at.devicePointer) {
                (void)cudaGetLastError();
                return fail(KVQ_EINVAL, "%s: host buffers must be page-locked to pass no device "
                            "buffers", what);
            }
            dev_ptr[i] = at.devicePointer;
        }
        if (!aligned16(dev_ptr[0]) || !aligned16(dev_ptr[1]))
            return fail(KVQ_EINVAL, "%s: host buffers must be 16-byte aligned", what);
        const uint16_t* dq = static_cast<const uint16_t*>(dev_ptr[0]);
        return decode_impl(what, dq, dq + nq, dq + nq + nkv, kc, vc, signs_k, signs_v, K, V,
                           ctx_len, B, H_q, H_kv, max_ctx, softmax_scale, num_splits, workspace,
                           ws_bytes, err_word, dev_ptr[1], out_dtype, stream);
    }
    if (!aligned16(in_dev) || !aligned16(out_dev))
        return fail(KVQ_EINVAL, "%s: device buffers must be 16-byte aligned", what);
    const HostIO hio{in_host, (nq + 2 * nkv) * 2, out_host, nq * (out_dtype == 1 ? 4 : 2)};
    const uint16_t* dq = static_cast<const uint16_t*>(in_dev);
    return decode_impl(what, dq, dq + nq, dq + nq + nkv, kc, vc, signs_k, signs_v, K, V, ctx_len,
                       B, H_q, H_kv, max_ctx, softmax_scale, num_splits, workspace, ws_bytes,
                       err_word, out_dev, out_dtype, stream, nullptr, nullptr, &hio);
}

int kvq_decode_attn_paged(const void* q, const kvq_codec* kc, const kvq_codec* vc,
                          const int8_t* signs_k, const int8_t* signs_v, const kvq_paged_plane* K,
                          const kvq_paged_plane* V, const int32_t* ctx_len, int32_t B,
                          int32_t H_q, int32_t H_kv, int64_t max_ctx, float softmax_scale,
                          int32_t num_splits, void* workspace, int64_t ws_bytes,
                          int32_t* err_word, void* out, int32_t out_dtype, void* stream) {
    if (!K || !V) return fail(KVQ_EINVAL, "kvq_decode_attn_paged: paged plane is NULL");
    return decode_impl("kvq_decode_attn_paged", q, nullptr, nullptr, kc, vc, signs_k, signs_v,
                       nullptr, nullptr, ctx_len, B, H_q, H_kv, max_ctx, softmax_scale,
                       num_splits, workspace, ws_bytes, err_word, out, out_dtype, stream, K, V);
}

int kvq_decode_step_paged(const void* q, const void* k_new, const void* v_new,
                          const kvq_codec* kc, const kvq_codec* vc, const int8_t* signs_k,
                          const int8_t* signs_v, const kvq_paged_plane* K,
                          const kvq_paged_plane* V, const int32_t* ctx_len, int32_t B,
                          int32_t H_q, int32_t H_kv, int64_t max_ctx, float softmax_scale,
                          int32_t num_splits, void* workspace, int64_t ws_bytes,
                          int32_t* err_word, void* out, int32_t out_dtype, void* stream) {
    if (!K || !V) return fail(KVQ_EINVAL, "kvq_decode_step_paged: paged plane is NULL");
    if (!k_new || !v_new) return fail(KVQ_EINVAL, "kvq_decode_step_paged: NULL k_new or v_new");
    if (!aligned16(k_new) || !aligned16(v_new))
        return fail(KVQ_EINVAL, "kvq_decode_step_paged: k_new and v_new must be 16-byte aligned");
    return decode_impl("kvq_decode_step_paged", q, k_new, v_new, kc, vc, signs_k, signs_v,
                       nullptr, nullptr, ctx_len, B, H_q, H_kv, max_ctx, softmax_scale,
                       num_splits, workspace, ws_bytes, err_word, out, out_dtype, stream, K, V);
}

}  // extern "C"
