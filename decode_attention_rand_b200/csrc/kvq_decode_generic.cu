// kvq_decode_generic.cu - decode attention for every codec the library
// encodes: head_dim 4..256, any number G of query heads per KV head, codebook
// sizes 2..65536, either norm mode for K and for V.  The shapes of the
// benchmarked models (head_dim 64 or 128, G a power of two up to 8, L up to
// 256, 8-bit linear K norms with 4-bit log V norms) run in the staged kernel
// of kvq_decode_impl.cuh; everything else runs here.
//
// Same method and result as that kernel ("TurboAngle: Near-Lossless KV Cache
// Compression via Uniform Angle Quantization", Abstract; scores from the codes
// in the rotated domain, the on-the-fly reconstruction of "OCTOPUS: Joint
// Triplet Quantization for KV Cache via Octahedral Parametrization", "Why it
// matters"), written for generality instead of speed:
//   - one CTA of four warps per (split, KV head, batch entry, chunk of up to
//     eight query heads); codes are read straight from global memory (each
//     group of lanes reads one token's rows, coalesced), no staging ring;
//   - a group of NLT = min(32, d/2) lanes owns one token at a time, each lane
//     PPL = d/2 / NLT pairs and the matching pairs of the chunk's heads;
//     partial scores are summed over the group with shuffles;
//   - bin centres come from a shared-memory cos/sin table for codebooks up to
//     4096 entries and from sincospif beyond;
//   - every group keeps an exact online softmax (rescaled whenever its
//     maximum grows); groups, then splits, are merged as in the staged kernel,
//     through the same workspace layout (completion counters, per-split max
//     and denominator, per-split accumulators) and a last-CTA combine.
// kvq_decode_step on these codecs runs append_kernel first (the new token's
// K and V rows, exactly as kvq_encode_kv writes them), then this kernel, as a
// programmatic dependent of it.
#include "kvq_encode_impl.cuh"
#include "kvq_internal.h"

namespace kvq {
namespace {

constexpr int kGenWarps = 4;
constexpr int kGenThreads = kGenWarps * 32;
constexpr int kGenHeads = 8;      // query heads per CTA (a chunk of the G heads)
constexpr int kGenTabMax = 4096;  // largest codebook with a shared-memory table

template <int D>
struct GenCfg {
    static constexpr int P = D / 2;
    static constexpr int NLT = P < 32 ? P : 32;  // lanes per token
    static constexpr int PPL = P / NLT;          // pairs per lane
    static constexpr int TPW = 32 / NLT;         // tokens per warp step
    static constexpr int NG = kGenWarps * TPW;   // groups per CTA
};

__device__ __forceinline__ void gen_griddep_wait() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

// Angle code of pair i of a row (bits [i b, i b + b) of its LSB-first stream).
__device__ __forceinline__ uint32_t gen_code(const uint32_t* row, int i, int bits) {
    const int pos = i * bits;
    const int wi = pos >> 5, sh = pos & 31;
    const uint32_t lo = row[wi];
    const uint32_t hi = sh + bits > 32 ? row[wi + 1] : 0u;
    return __funnelshift_r(lo, hi, sh) & ((1u << bits) - 1u);
}

// Per-token norm parameters: LIN8 (M / 255, 0), LOG4 (LO, (HI - LO) / 15).
__device__ __forceinline__ float2 gen_params(const CodecDev& c, const uint8_t* params,
                                             int64_t row) {
    if (c.mode == KVQ_NORM_LIN8) {
        const uint16_t m = reinterpret_cast<const uint16_t*>(params)[row];
        return make_float2(half_bits_to_float(m) * (1.f / 255.f), 0.f);
    }
    const uint32_t pr = reinterpret_cast<const uint32_t*>(params)[row];
    const float lo = half_bits_to_float((uint16_t)(pr & 0xFFFF));
    const float hi = half_bits_to_float((uint16_t)(pr >> 16));
    return make_float2(lo, (hi - lo) * (1.f / 15.f));
}

// Reconstructed norm r^ of pair i of a row.
__device__ __forceinline__ float gen_norm(const CodecDev& c, const uint8_t* norms, int64_t row,
                                          int i, float2 prm) {
    if (c.mode == KVQ_NORM_LIN8) return (float)norms[row * c.norm_bytes + i] * prm.x;
    const uint32_t byte = norms[row * c.norm_bytes + i / 2];
    const float code = (float)((byte >> (4 * (i & 1))) & 0xFu);
    return exp2f(fmaf(code, prm.y, prm.x));
}

// Bin centre of code a: (cos, sin) of -pi + (a + 1/2) 2 pi / L.  A code of
// L or more (never written by the encoder; KVQ_DEBUG reports it) reads entry
// 0 rather than past the table.
__device__ __forceinline__ float2 gen_centre(const float2* tab, uint32_t a, int L) {
    if (L <= kGenTabMax) return tab[a < (uint32_t)L ? a : 0u];
    float s, c;
    sincospif((float)(2 * (int)a + 1) / (float)L - 1.f, &s, &c);
    return make_float2(c, s);
}

// In-place Walsh-Hadamard transform (Sylvester order, unscaled) of `n` rows
// of D floats in shared memory, by the whole CTA.
template <int D>
__device__ void gen_fwht_rows(float* rows, int n) {
    for (int h = 1; h < D; h <<= 1) {
        __syncthreads();
        for (int idx = threadIdx.x; idx < n * (D / 2); idx += blockDim.x) {
            const int r = idx / (D / 2), k = idx % (D / 2);
            const int i = (k / h) * (2 * h) + (k % h);
            float* v = rows + r * D;
            const float a = v[i], bb = v[i + h];
            v[i] = a + bb;
            v[i + h] = a - bb;
        }
    }
    __syncthreads();
}

template <int D>
__global__ void __launch_bounds__(kGenThreads)
decode_generic_kernel(DecodeArgs A, int chunks) {
    // the next launch on the stream may start its setup now (see gen_griddep_wait)
    asm volatile("griddepcontrol.launch_dependents;");
    using Cfg = GenCfg<D>;
    constexpr int NLT = Cfg::NLT, PPL = Cfg::PPL, TPW = Cfg::TPW, NG = Cfg::NG;
    const int G = A.H_q / A.H_kv;
    const int split = blockIdx.x, kvh = blockIdx.y / chunks, chunk = blockIdx.y % chunks;
    const int b = blockIdx.z;
    const int h0 = chunk * kGenHeads;
    const int nh = G - h0 < kGenHeads ? G - h0 : kGenHeads;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int grp = lane / NLT, lg = lane % NLT;
    const int gidx = warp * TPW + grp;

    extern __shared__ __align__(16) unsigned char smem[];
    const int nTK = A.kc.L <= kGenTabMax ? A.kc.L : 0;
    const int nTV = A.vc.L <= kGenTabMax ? A.vc.L : 0;
    float2* tabK = reinterpret_cast<float2*>(smem);  // [nTK]
    float2* tabV = tabK + nTK;                       // [nTV]
    float* qs = reinterpret_cast<float*>(tabV + nTV);  // [kGenHeads][D] rotated queries
    float* gm = qs + kGenHeads * D;                   // [NG][kGenHeads] group maxima
    float* gl = gm + NG * kGenHeads;                  // [NG][kGenHeads] denominators
    float* gacc = gl + NG * kGenHeads;                // [NG][kGenHeads][D] accumulators
    int* sflag = reinterpret_cast<int*>(gacc + NG * kGenHeads * D);

    for (int a = tid; a < nTK + nTV; a += kGenThreads) {
        const bool isK = a < nTK;
        const int code = isK ? a : a - nTK;
        float s, c;
        sincospif((float)(2 * code + 1) / (float)(isK ? A.kc.L : A.vc.L) - 1.f, &s, &c);
        tabK[a] = make_float2(c, s);
    }
    // nothing global is read before the previous launch on the stream (for
    // kvq_decode_step: the append) has completed
    gen_griddep_wait();

    // ---- q' = H D_K q / sqrt(d) for the chunk's heads ------------------------
    for (int idx = tid; idx < kGenHeads * D; idx += kGenThreads) {
        const int h = idx / D, j = idx % D;
        float v = 0.f;
        if (h < nh) {
            const __half* qh = A.q + ((int64_t)b * A.H_q + (int64_t)kvh * G + h0 + h) * D;
            v = __half2float(qh[j]);
            v = A.signs_k[j] < 0 ? -v : v;
        }
        qs[idx] = v;
    }
    gen_fwht_rows<D>(qs, kGenHeads);
    const float isd = rsqrtf((float)D);
    float2 q2[kGenHeads][PPL];
#pragma unroll
    for (int h = 0; h < kGenHeads; h++)
#pragma unroll
        for (int k = 0; k < PPL; k++) {
            const int i = lg + NLT * k;
            q2[h][k] = make_float2(qs[h * D + 2 * i] * isd, qs[h * D + 2 * i + 1] * isd);
        }

    // ---- token range of this split, clipped to the context -------------------
    const int64_t lim = A.max_ctx < A.K.capacity ? A.max_ctx : A.K.capacity;
    int64_t ctx = A.ctx_len[b];
    if (ctx < 0 || ctx > lim) {
        if (split == 0 && blockIdx.y == 0 && tid == 0) report(A.err_word, KVQ_DEVERR_CTX_RANGE);
        ctx = ctx < 0 ? 0 : lim;
    }
    const int64_t t0 = (int64_t)split * A.split_len;
    int64_t t1 = t0 + A.split_len < ctx ? t0 + A.split_len : ctx;

    float m[kGenHeads], l[kGenHeads];
    float2 acc[kGenHeads][PPL];
#pragma unroll
    for (int h = 0; h < kGenHeads; h++) {
        m[h] = -INFINITY;
        l[h] = 0.f;
#pragma unroll
        for (int k = 0; k < PPL; k++) acc[h][k] = make_float2(0.f, 0.f);
    }
    const uint32_t* ka = reinterpret_cast<const uint32_t*>(A.K.angles);
    const uint32_t* va = reinterpret_cast<const uint32_t*>(A.V.angles);
    for (int64_t tb = t0 + (int64_t)warp * TPW; tb < t1; tb += (int64_t)kGenWarps * TPW) {
        const int64_t t = tb + grp;
        const bool valid = t < t1;
        bool bad = false;
        const int64_t rk = valid ? plane_row(A.K, b, kvh, t, &bad) : 0;
        const int64_t rv = valid ? plane_row(A.V, b, kvh, t, &bad) : 0;
        if (bad) report(A.err_word, KVQ_DEVERR_PAGE_RANGE);
        // scores: this lane's pairs, then the group sum
        float part[kGenHeads];
#pragma unroll
        for (int h = 0; h < kGenHeads; h++) part[h] = 0.f;
        if (valid) {
            const float2 pk = gen_params(A.kc, A.K.params, rk);
#pragma unroll
            for (int k = 0; k < PPL; k++) {
                const int i = lg + NLT * k;
                const float2 cs = gen_centre(tabK, gen_code(ka + rk * A.kc.angle_words, i,
                                                            A.kc.bits), A.kc.L);
                const float r = gen_norm(A.kc, A.K.norms, rk, i, pk);
                const float kx = r * cs.x, ky = r * cs.y;
#pragma unroll
                for (int h = 0; h < kGenHeads; h++)
                    part[h] = fmaf(q2[h][k].x, kx, fmaf(q2[h][k].y, ky, part[h]));
            }
        }
#pragma unroll
        for (int h = 0; h < kGenHeads; h++) part[h] = group_sum<NLT>(part[h]);
        // values in the rotated domain
        float2 vz[PPL];
#pragma unroll
        for (int k = 0; k < PPL; k++) vz[k] = make_float2(0.f, 0.f);
        if (valid) {
            const float2 pv = gen_params(A.vc, A.V.params, rv);
#pragma unroll
            for (int k = 0; k < PPL; k++) {
                const int i = lg + NLT * k;
                const float2 cs = gen_centre(tabV, gen_code(va + rv * A.vc.angle_words, i,
                                                            A.vc.bits), A.vc.L);
                const float r = gen_norm(A.vc, A.V.norms, rv, i, pv);
                vz[k] = make_float2(r * cs.x, r * cs.y);
            }
        }
        // exact online softmax of this group's token stream
#pragma unroll
        for (int h = 0; h < kGenHeads; h++) {
            if (!valid || h >= nh) continue;
            const float s = part[h] * A.scale_log2;
            if (s > m[h]) {
                const float al = m[h] == -INFINITY ? 0.f : exp2f(m[h] - s);
                l[h] *= al;
#pragma unroll
                for (int k = 0; k < PPL; k++) {
                    acc[h][k].x *= al;
                    acc[h][k].y *= al;
                }
                m[h] = s;
            }
            const float p = exp2f(s - m[h]);
            l[h] += p;
#pragma unroll
            for (int k = 0; k < PPL; k++) {
                acc[h][k].x = fmaf(p, vz[k].x, acc[h][k].x);
                acc[h][k].y = fmaf(p, vz[k].y, acc[h][k].y);
            }
        }
    }

    // ---- merge the groups of this CTA --------------------------------------
#pragma unroll
    for (int h = 0; h < kGenHeads; h++) {
        if (lg == 0) {
            gm[gidx * kGenHeads + h] = m[h];
            gl[gidx * kGenHeads + h] = l[h];
        }
#pragma unroll
        for (int k = 0; k < PPL; k++) {
            const int i = lg + NLT * k;
            float* row = gacc + ((size_t)gidx * kGenHeads + h) * D;
            row[2 * i] = acc[h][k].x;
            row[2 * i + 1] = acc[h][k].y;
        }
    }
    __syncthreads();
    const int S = A.num_splits;
    float* stats = A.ws + ws_counter_floats(A.B, A.H_q);
    float* accs = stats + ws_stat_floats(A.B, A.H_q, S);
    for (int idx = tid; idx < nh * D; idx += kGenThreads) {
        const int h = idx / D, j = idx % D;
        float mx = -INFINITY;
        for (int g = 0; g < NG; g++) mx = fmaxf(mx, gm[g * kGenHeads + h]);
        float sl = 0.f, sa = 0.f;
        if (mx != -INFINITY)
            for (int g = 0; g < NG; g++) {
                const float w = exp2f(gm[g * kGenHeads + h] - mx);
                sl = fmaf(w, gl[g * kGenHeads + h], sl);
                sa = fmaf(w, gacc[((size_t)g * kGenHeads + h) * D + j], sa);
            }
        const int64_t slot = ((int64_t)b * A.H_q + (int64_t)kvh * G + h0 + h) * S + split;
        accs[slot * D + j] = sa;
        if (j == 0) {
            stats[slot * 2] = mx;
            stats[slot * 2 + 1] = sl;
        }
    }

    // partials only (kvq_decode_attn_partials): the caller merges them
    if (A.partials_only) return;

    // ---- the last CTA of this (b, KV head, chunk) merges the splits ----------
    __threadfence();
    __syncthreads();
    int* counters = reinterpret_cast<int*>(A.ws);
    const int64_t cidx = (int64_t)b * A.H_q + (int64_t)kvh * G + h0;
    if (tid == 0) {
        const int prev = atomicAdd(&counters[cidx], 1);
        sflag[0] = prev == S - 1;
    }
    __syncthreads();
    if (!sflag[0]) return;
    __threadfence();
    for (int idx = tid; idx < kGenHeads * D; idx += kGenThreads) {
        const int h = idx / D, j = idx % D;
        float v = 0.f;
        if (h < nh) {
            const int64_t hq = (int64_t)b * A.H_q + (int64_t)kvh * G + h0 + h;
            const float* stp = stats + hq * S * 2;
            float mx = -INFINITY;
            for (int s = 0; s < S; s++) mx = fmaxf(mx, __ldcg(stp + 2 * s));
            float sl = 0.f, sa = 0.f;
            if (mx != -INFINITY)
                for (int s = 0; s < S; s++) {
                    const float w = exp2f(__ldcg(stp + 2 * s) - mx);
                    sl = fmaf(w, __ldcg(stp + 2 * s + 1), sl);
                    sa = fmaf(w, __ldcg(accs + (hq * S + s) * D + j), sa);
                }
            v = sl > 0.f ? sa / sl : 0.f;
        }
        qs[idx] = v;
    }
    gen_fwht_rows<D>(qs, kGenHeads);
    for (int idx = tid; idx < nh * D; idx += kGenThreads) {
        const int h = idx / D, j = idx % D;
        const int64_t hq = (int64_t)b * A.H_q + (int64_t)kvh * G + h0 + h;
        float o = qs[idx] * isd;
        o = A.signs_v[j] < 0 ? -o : o;
        if (A.out_dtype == 0)
            reinterpret_cast<__half*>(A.out)[hq * D + j] = __float2half_rn(o);
        else
            reinterpret_cast<float*>(A.out)[hq * D + j] = o;
    }
    if (tid == 0) atomicExch(&counters[cidx], 0);
}

// The new token of every (b, KV head) at position ctx_len[b] - 1, written
// exactly as kvq_encode_kv writes it (the same encode_tile): warp 0 encodes
// the K vector, warp 1 the V vector.
//
// Its dependent (the decode) may start once every CTA here has passed the
// wait for the kernels before it: by then everything those kernels wrote (q,
// ctx_len, the cache) is complete and visible, and the decode needs to wait
// for this kernel only before it copies in the tile holding the new rows.
template <int D>
__global__ void __launch_bounds__(64) append_kernel(DecodeArgs A) {
    __shared__ uint32_t est[2][kEncStageWords];
    const int kvh = blockIdx.x, b = blockIdx.y;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    gen_griddep_wait();
    asm volatile("griddepcontrol.launch_dependents;");
    const int64_t lim = A.max_ctx < A.K.capacity ? A.max_ctx : A.K.capacity;
    const int64_t ctx = A.ctx_len[b];
    if (ctx < 1 || ctx > lim) return;  // nothing to append (the decode reports the clip)
    using ECfg = EncCfg<D>;
    EncArgs E = warp == 0 ? A.enc_k : A.enc_v;
    const int64_t bh = (int64_t)b * A.H_kv + kvh;
    E.x = (warp == 0 ? A.k_new : A.v_new) + bh * D;
    E.n_vec = 1;
    E.T = 1;
    E.pos0 = ctx - 1;
    E.bh0 = bh;
    E.out = warp == 0 ? A.K : A.V;
    E.err_word = A.err_word;
    for (int i = lane; i < kEncStageWords; i += 32) est[warp][i] = 0u;
    __syncwarp();
    const int elg = lane % ECfg::NL, egrp = lane / ECfg::NL;
    uint32_t smask[ECfg::PPL];
    lane_sign_masks<D>(E.signs, elg, smask);
    (void)encode_tile<D, true>(E, 0, smask, est[warp], angle_margin(E), lane, egrp, elg);
}

template <int D>
cudaError_t launch_append_d(const DecodeArgs& a, cudaStream_t stream) {
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cfg.gridDim = dim3((unsigned)a.H_kv, (unsigned)a.B, 1);
    cfg.blockDim = dim3(64);
    return cudaLaunchKernelEx(&cfg, append_kernel<D>, a);
}

template <int D>
cudaError_t launch_generic_d(const DecodeArgs& a, cudaStream_t stream) {
    using Cfg = GenCfg<D>;
    const int G = a.H_q / a.H_kv;
    const int chunks = (G + kGenHeads - 1) / kGenHeads;
    const int nTK = a.kc.L <= kGenTabMax ? a.kc.L : 0;
    const int nTV = a.vc.L <= kGenTabMax ? a.vc.L : 0;
    const size_t smem = sizeof(float2) * (size_t)(nTK + nTV) +
                        sizeof(float) * ((size_t)kGenHeads * D + 2 * Cfg::NG * kGenHeads +
                                         (size_t)Cfg::NG * kGenHeads * D) +
                        16;
    auto kernel = decode_generic_kernel<D>;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (a.k_new) {
        e = launch_append_d<D>(a, stream);
        if (e != cudaSuccess) return e;
    }
    cfg.gridDim = dim3((unsigned)a.num_splits, (unsigned)(a.H_kv * chunks), (unsigned)a.B);
    cfg.blockDim = dim3(kGenThreads);
    cfg.dynamicSmemBytes = smem;
    e = cudaLaunchKernelEx(&cfg, kernel, a, chunks);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_append(const DecodeArgs& a, cudaStream_t stream) {
    switch (a.kc.d) {
        case 4: return launch_append_d<4>(a, stream);
        case 8: return launch_append_d<8>(a, stream);
        case 16: return launch_append_d<16>(a, stream);
        case 32: return launch_append_d<32>(a, stream);
        case 64: return launch_append_d<64>(a, stream);
        case 128: return launch_append_d<128>(a, stream);
        case 256: return launch_append_d<256>(a, stream);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_decode_generic(const DecodeArgs& a, cudaStream_t stream) {
    switch (a.kc.d) {
        case 4: return launch_generic_d<4>(a, stream);
        case 8: return launch_generic_d<8>(a, stream);
        case 16: return launch_generic_d<16>(a, stream);
        case 32: return launch_generic_d<32>(a, stream);
        case 64: return launch_generic_d<64>(a, stream);
        case 128: return launch_generic_d<128>(a, stream);
        case 256: return launch_generic_d<256>(a, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace kvq
