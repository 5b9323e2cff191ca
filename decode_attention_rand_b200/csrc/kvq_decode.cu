// kvq_decode.cu - split-K decode attention straight from packed codes, and
// the combine pass.
//
// The cache is never dequantized ("OCTOPUS: Joint Triplet Quantization for KV
// Cache via Octahedral Parametrization", "Why it matters": keys are rebuilt on
// the fly inside attention).  With the rotation R = H D / sqrt(d) orthogonal,
// q . k^ = (R q) . z^_K, so each query head is rotated once and every cached
// token is scored in the rotated domain from its codes:
//     s_t = tau * sum_i r^_i (q'[2i] cos theta^_i + q'[2i+1] sin theta^_i),
// the softmax runs online, the values are accumulated in the rotated domain
// (acc = sum_t p_t z^_V,t) and one inverse rotation D_V H / sqrt(d) per head
// finishes the output.  Codec: "TurboAngle: Near-Lossless KV Cache
// Compression via Uniform Angle Quantization", Abstract.
//
// Pass 1 (split-K): one CTA per (split, KV head, batch).  Each group of NL
// lanes owns one token at a time; each lane owns PP = 4 pairs of it and the
// matching pairs of the G query heads that share the KV head (GQA), so every
// unpacked code serves all G heads.  Per-group online-softmax states are
// merged in shared memory and written as (m, l, acc[d]) partials.
// Pass 2 (combine): per query head, log-sum-exp merge of the splits, divide
// by l, inverse FWHT, D_V / sqrt(d), store fp16 or fp32.
#include "kvq_internal.h"

namespace kvq {

constexpr int kDecWarps = 4;
constexpr int kPP = 4;  // pairs per lane

template <int D>
struct DecCfg {
    static constexpr int P = D / 2;
    static constexpr int NL = P / kPP;     // lanes per token
    static constexpr int TPW = 32 / NL;    // tokens per warp step
    static constexpr int NG = kDecWarps * TPW;  // token groups per CTA
};

struct CodeView {
    const uint32_t* angles;  // row words of token 0 of this (b, h)
    const uint8_t* norms;
    const uint8_t* params;
};

// r^ for the kPP pairs of this lane of one token; returns the angle codes.
__device__ __forceinline__ void token_pairs(const CodeView& cv, const CodecDev& c, int64_t t,
                                            int lg, int (&a)[kPP], float (&r)[kPP]) {
    const int bits = c.bits;
    const int cb = lg * kPP * bits;
    const int w0 = cb >> 5, sh = cb & 31;
    const uint32_t* row = cv.angles + t * c.angle_words;
    const uint32_t lo = row[w0];
    const uint32_t hi = (w0 + 1 < c.angle_words) ? row[w0 + 1] : 0u;
    const uint32_t chunk = __funnelshift_r(lo, hi, sh);
    const uint32_t mask = (1u << bits) - 1u;
#pragma unroll
    for (int k = 0; k < kPP; k++) a[k] = (int)((chunk >> (k * bits)) & mask);
    if (c.mode == KVQ_NORM_LIN8) {
        const uint32_t nb = *reinterpret_cast<const uint32_t*>(cv.norms + t * c.norm_bytes + lg * kPP);
        const float s = half_bits_to_float(reinterpret_cast<const uint16_t*>(cv.params)[t]) *
                        (1.f / 255.f);
#pragma unroll
        for (int k = 0; k < kPP; k++) r[k] = (float)((nb >> (8 * k)) & 0xFFu) * s;
    } else {
        const uint32_t nb =
            *reinterpret_cast<const uint16_t*>(cv.norms + t * c.norm_bytes + lg * (kPP / 2));
        const uint32_t pr = reinterpret_cast<const uint32_t*>(cv.params)[t];
        const float LO = half_bits_to_float((uint16_t)(pr & 0xFFFF));
        const float HI = half_bits_to_float((uint16_t)(pr >> 16));
        const float step = (HI - LO) * (1.f / 15.f);
#pragma unroll
        for (int k = 0; k < kPP; k++) r[k] = exp2f(fmaf((float)((nb >> (4 * k)) & 0xFu), step, LO));
    }
}

template <int D, int G>
__global__ void __launch_bounds__(kDecWarps * 32)
decode_split_kernel(DecodeArgs A) {
    using Cfg = DecCfg<D>;
    constexpr int NL = Cfg::NL, TPW = Cfg::TPW, NG = Cfg::NG;
    constexpr int EPQ = D / 32;  // q elements per lane in the rotation prologue

    extern __shared__ float4 smem_f4[];
    float* smem = reinterpret_cast<float*>(smem_f4);
    float2* tabK = reinterpret_cast<float2*>(smem);          // [256]
    float2* tabV = tabK + 256;                                // [256]
    float* qs = reinterpret_cast<float*>(tabV + 256);         // [G][D]
    float* gm = qs + G * D;                                   // [NG][G]
    float* gl = gm + NG * G;                                  // [NG][G]
    float* gacc = gl + NG * G;                                // [NG][G][D]

    const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int grp = lane / NL, lg = lane % NL;
    const int gidx = warp * TPW + grp;

    // ---- tables of bin-centre cos/sin -------------------------------------
    for (int j = tid; j < A.kc.L; j += blockDim.x) {
        float s, c;
        sincospif((float)(2 * j + 1) / (float)A.kc.L - 1.f, &s, &c);
        tabK[j] = make_float2(c, s);
    }
    for (int j = tid; j < A.vc.L; j += blockDim.x) {
        float s, c;
        sincospif((float)(2 * j + 1) / (float)A.vc.L - 1.f, &s, &c);
        tabV[j] = make_float2(c, s);
    }
    // ---- rotate the G query heads once: q' = H D_K q / sqrt(d) ------------
    for (int h = warp; h < G; h += kDecWarps) {
        const __half* qh = A.q + ((int64_t)b * A.H_q + (int64_t)kvh * G + h) * D;
        float v[EPQ];
#pragma unroll
        for (int e = 0; e < EPQ; e++) {
            const int j = lane * EPQ + e;
            const float f = __half2float(qh[j]);
            v[e] = A.signs_k[j] < 0 ? -f : f;
        }
        fwht_local<EPQ>(v);
        fwht_cross<EPQ, 32>(v, lane);
        const float isd = rsqrtf((float)D);
#pragma unroll
        for (int e = 0; e < EPQ; e++) qs[h * D + lane * EPQ + e] = v[e] * isd;
    }
    __syncthreads();

    float q0[G][kPP], q1[G][kPP];
#pragma unroll
    for (int h = 0; h < G; h++)
#pragma unroll
        for (int k = 0; k < kPP; k++) {
            const int i = lg * kPP + k;
            q0[h][k] = qs[h * D + 2 * i];
            q1[h][k] = qs[h * D + 2 * i + 1];
        }

    // ---- token range of this split -----------------------------------------
    int64_t ctx = A.ctx_len[b];
    const int64_t lim = A.max_ctx < A.K.capacity ? A.max_ctx : A.K.capacity;
    if (ctx < 0 || ctx > lim) {
        if (split == 0 && kvh == 0 && tid == 0) report(A.err_word, KVQ_DEVERR_CTX_RANGE);
        ctx = ctx < 0 ? 0 : lim;
    }
    const int64_t t0 = (int64_t)split * A.split_len;
    const int64_t t1 = (t0 + A.split_len < ctx) ? t0 + A.split_len : ctx;

    const int64_t plane = (int64_t)b * A.H_kv + kvh;
    CodeView kv_k, kv_v;
    kv_k.angles = reinterpret_cast<const uint32_t*>(A.K.angles) + plane * A.K.capacity * A.kc.angle_words;
    kv_k.norms = A.K.norms + plane * A.K.capacity * A.kc.norm_bytes;
    kv_k.params = A.K.params + plane * A.K.capacity * A.kc.param_bytes;
    kv_v.angles = reinterpret_cast<const uint32_t*>(A.V.angles) + plane * A.V.capacity * A.vc.angle_words;
    kv_v.norms = A.V.norms + plane * A.V.capacity * A.vc.norm_bytes;
    kv_v.params = A.V.params + plane * A.V.capacity * A.vc.param_bytes;

    float m[G], l[G], acc0[G][kPP], acc1[G][kPP];
#pragma unroll
    for (int h = 0; h < G; h++) {
        m[h] = -INFINITY;
        l[h] = 0.f;
#pragma unroll
        for (int k = 0; k < kPP; k++) acc0[h][k] = acc1[h][k] = 0.f;
    }

    for (int64_t base = t0 + warp * TPW; base < t1; base += NG) {
        const int64_t t = base + grp;
        const bool valid = t < t1;
        float s[G];
#pragma unroll
        for (int h = 0; h < G; h++) s[h] = 0.f;
        if (valid) {
            int a[kPP];
            float r[kPP];
            token_pairs(kv_k, A.kc, t, lg, a, r);
#pragma unroll
            for (int k = 0; k < kPP; k++) {
                const float2 cs = tabK[a[k]];
                const float x = r[k] * cs.x, y = r[k] * cs.y;
#pragma unroll
                for (int h = 0; h < G; h++) s[h] = fmaf(q0[h][k], x, fmaf(q1[h][k], y, s[h]));
            }
        }
#pragma unroll
        for (int h = 0; h < G; h++) s[h] = group_sum<NL>(s[h]);
        if (valid) {
            float p[G];
#pragma unroll
            for (int h = 0; h < G; h++) {
                const float sv = s[h] * A.scale_log2;
                const float mn = fmaxf(m[h], sv);
                const float al = exp2f(m[h] - mn);
                p[h] = exp2f(sv - mn);
                l[h] = l[h] * al + p[h];
                m[h] = mn;
#pragma unroll
                for (int k = 0; k < kPP; k++) {
                    acc0[h][k] *= al;
                    acc1[h][k] *= al;
                }
            }
            int a[kPP];
            float r[kPP];
            token_pairs(kv_v, A.vc, t, lg, a, r);
#pragma unroll
            for (int k = 0; k < kPP; k++) {
                const float2 cs = tabV[a[k]];
                const float x = r[k] * cs.x, y = r[k] * cs.y;
#pragma unroll
                for (int h = 0; h < G; h++) {
                    acc0[h][k] = fmaf(p[h], x, acc0[h][k]);
                    acc1[h][k] = fmaf(p[h], y, acc1[h][k]);
                }
            }
        }
    }

    // ---- merge the NG group states of this CTA -----------------------------
    if (lg == 0) {
#pragma unroll
        for (int h = 0; h < G; h++) {
            gm[gidx * G + h] = m[h];
            gl[gidx * G + h] = l[h];
        }
    }
#pragma unroll
    for (int h = 0; h < G; h++)
#pragma unroll
        for (int k = 0; k < kPP; k++) {
            const int i = lg * kPP + k;
            gacc[(gidx * G + h) * D + 2 * i] = acc0[h][k];
            gacc[(gidx * G + h) * D + 2 * i + 1] = acc1[h][k];
        }
    __syncthreads();

    const int S = A.num_splits;
    for (int idx = tid; idx < G * D; idx += blockDim.x) {
        const int h = idx / D, j = idx % D;
        float mx = -INFINITY;
        for (int g = 0; g < NG; g++) mx = fmaxf(mx, gm[g * G + h]);
        float sum_l = 0.f, sum_a = 0.f;
        if (mx != -INFINITY) {
            for (int g = 0; g < NG; g++) {
                const float w = exp2f(gm[g * G + h] - mx);
                sum_l += w * gl[g * G + h];
                sum_a += w * gacc[(g * G + h) * D + j];
            }
        }
        const int64_t hq = (int64_t)b * A.H_q + (int64_t)kvh * G + h;
        const int64_t slot = hq * S + split;
        A.ws[ws_stat_floats(A.B, A.H_q, S) + slot * D + j] = sum_a;
        if (j == 0) {
            A.ws[slot * 2] = mx;
            A.ws[slot * 2 + 1] = sum_l;
        }
    }
}

// Pass 2: one warp per query head.
template <int D>
__global__ void __launch_bounds__(128)
decode_combine_kernel(DecodeArgs A) {
    constexpr int EPL = D / 32;
    const int lane = threadIdx.x & 31;
    const int64_t hq = (int64_t)blockIdx.x * 4 + (threadIdx.x >> 5);
    if (hq >= (int64_t)A.B * A.H_q) return;
    const int S = A.num_splits;
    const float* stats = A.ws + hq * S * 2;
    const float* accs = A.ws + ws_stat_floats(A.B, A.H_q, S) + hq * S * D;

    float mx = -INFINITY;
    for (int s = lane; s < S; s += 32) mx = fmaxf(mx, stats[2 * s]);
    mx = group_max<32>(mx);
    float v[EPL];
#pragma unroll
    for (int e = 0; e < EPL; e++) v[e] = 0.f;
    float sum_l = 0.f;
    if (mx != -INFINITY) {
        for (int s = 0; s < S; s++) {
            const float w = exp2f(stats[2 * s] - mx);
            sum_l += w * stats[2 * s + 1];
#pragma unroll
            for (int e = 0; e < EPL; e++) v[e] = fmaf(w, accs[(int64_t)s * D + lane * EPL + e], v[e]);
        }
    }
    const float inv = sum_l > 0.f ? 1.f / sum_l : 0.f;
#pragma unroll
    for (int e = 0; e < EPL; e++) v[e] *= inv;
    fwht_local<EPL>(v);
    fwht_cross<EPL, 32>(v, lane);
    const float isd = rsqrtf((float)D);
#pragma unroll
    for (int e = 0; e < EPL; e++) {
        const int j = lane * EPL + e;
        float o = v[e] * isd;
        o = A.signs_v[j] < 0 ? -o : o;
        if (A.out_dtype == 0)
            reinterpret_cast<__half*>(A.out)[hq * D + j] = __float2half_rn(o);
        else
            reinterpret_cast<float*>(A.out)[hq * D + j] = o;
    }
}

template <int D, int G>
static size_t split_smem_bytes() {
    using Cfg = DecCfg<D>;
    return sizeof(float2) * 512 + sizeof(float) * ((size_t)G * D + 2 * Cfg::NG * G +
                                                   (size_t)Cfg::NG * G * D);
}

template <int D, int G>
static cudaError_t launch_decode_dg(const DecodeArgs& a, cudaStream_t stream) {
    const size_t smem = split_smem_bytes<D, G>();
    // the dynamic shared-memory limit is set once per device and instantiation
    static bool attr_done[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64 || !attr_done[dev]) {
        e = cudaFuncSetAttribute(decode_split_kernel<D, G>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) attr_done[dev] = true;
    }
    dim3 grid((unsigned)a.num_splits, (unsigned)a.H_kv, (unsigned)a.B);
    decode_split_kernel<D, G><<<grid, kDecWarps * 32, smem, stream>>>(a);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int64_t heads = (int64_t)a.B * a.H_q;
    decode_combine_kernel<D><<<(unsigned)((heads + 3) / 4), 128, 0, stream>>>(a);
    return cudaGetLastError();
}

bool decode_supported(int d, int G, int LK, int LV, int mode_k, int mode_v) {
    (void)mode_k;
    (void)mode_v;
    if (d != 64 && d != 128) return false;
    if (G != 1 && G != 2 && G != 4 && G != 8) return false;
    return LK >= 2 && LK <= 256 && LV >= 2 && LV <= 256;
}

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t stream) {
    const int G = a.H_q / a.H_kv;
    const int d = a.kc.d;
#define KVQ_DEC_CASE(DD, GG) \
    if (d == DD && G == GG) return launch_decode_dg<DD, GG>(a, stream);
    KVQ_DEC_CASE(64, 1) KVQ_DEC_CASE(64, 2) KVQ_DEC_CASE(64, 4) KVQ_DEC_CASE(64, 8)
    KVQ_DEC_CASE(128, 1) KVQ_DEC_CASE(128, 2) KVQ_DEC_CASE(128, 4) KVQ_DEC_CASE(128, 8)
#undef KVQ_DEC_CASE
    return cudaErrorInvalidValue;
}

}  // namespace kvq
