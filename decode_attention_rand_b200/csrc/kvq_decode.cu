// kvq_decode.cu - split-K decode attention straight from packed codes, with
// the split combine fused into the same kernel.
//
// The cache is never dequantized ("OCTOPUS: Joint Triplet Quantization for KV
// Cache via Octahedral Parametrization", "Why it matters": keys are rebuilt on
// the fly inside attention).  With the rotation R = H D / sqrt(d) orthogonal,
// q . k^ = (R q) . z^_K, so each query head is rotated once and every cached
// token is scored in the rotated domain from its codes:
//     s_t = tau * sum_i r^_i (q'[2i] cos theta^_i + q'[2i+1] sin theta^_i),
// the softmax runs online, values are accumulated in the rotated domain
// (acc = sum_t p_t z^_V,t) and one inverse rotation D_V H / sqrt(d) per head
// finishes the output.  Codec: "TurboAngle: Near-Lossless KV Cache
// Compression via Uniform Angle Quantization", Abstract (8-bit linear K
// norms, 4-bit log-space V norms).
//
// One CTA per (split, KV head, batch entry):
//   - tiles of kTT tokens of the six code arrays (K/V angles, norms, params)
//     stream into shared memory through 1-D bulk asynchronous copies (TMA,
//     no multicast) on a kStages-deep ring of mbarrier-tracked stages; every
//     wait is bounded and a timeout is reported, never trapped;
//   - a group of NL lanes owns four tokens at a time, each lane PP pairs of
//     them and the matching pairs of all G query heads of the KV head (GQA),
//     so every unpacked code serves G heads; partial scores are reduced with a
//     transpose-reduce over the group, softmax weights gathered back the same
//     way;
//   - bin-centre cos/sin come from tables replicated 16 times so a half-warp's
//     64-bit lookups never collide on a bank;
//   - the online softmax rescales lazily, only when a score exceeds the
//     running reference max by more than 2^8;
//   - per-split partials (m, l, acc[d]) go to the workspace; the last CTA of a
//     (batch, KV head) to finish (atomic counter, no waiting) merges the
//     splits, divides by l, applies the inverse FWHT and D_V / sqrt(d).
#include "kvq_internal.h"

namespace kvq {

constexpr int kTT = 128;          // tokens per staged tile
constexpr int kStages = 3;        // ring depth
constexpr int kTPG = 4;           // tokens per group chunk
constexpr float kLazyThr = 8.f;   // log2 units
constexpr uint32_t kWaitLimit = 1u << 22;
constexpr int kTabRep = 16;       // table replicas (one per half-warp lane)

template <int D, int G>
struct DecCfg {
    static constexpr int P = D / 2;
    static constexpr int PP = (32 / G) > 16 ? 16 : (32 / G);  // pairs per lane
    static constexpr int NL = P / PP;                          // lanes per token group
    static constexpr int GPW = 32 / NL;                        // groups per warp
    // enough warps that every group owns one chunk per tile (at most 8)
    static constexpr int WARPS = (kTT / kTPG) / GPW > 8 ? 8
                                 : ((kTT / kTPG) / GPW < 2 ? 2 : (kTT / kTPG) / GPW);
    static constexpr int THREADS = WARPS * 32;
    static constexpr int NG = WARPS * GPW;                     // groups per CTA
    static constexpr int V = kTPG * G;                         // partial sums per lane
    static constexpr int VF = V / NL;                          // final sums per lane
    static_assert(VF >= 1, "group too wide");
    static_assert(PP % 4 == 0, "codes are unpacked four at a time");
};

// --------------------------------------------------------------- PTX ----

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void mbar_fence_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; "
        "selp.u32 %0, 1, 0, p; }"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0u;
}

// Bounded wait: false when the limit ran out.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity) {
    for (uint32_t it = 0; it < kWaitLimit; ++it)
        if (mbar_try_wait(bar, parity)) return true;
    return false;
}

__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void fence_proxy_async() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

typedef unsigned long long f32x2;  // two packed fp32 lanes

__device__ __forceinline__ f32x2 pack2(float lo, float hi) {
    return (f32x2)__float_as_uint(lo) | ((f32x2)__float_as_uint(hi) << 32);
}
__device__ __forceinline__ float lo2(f32x2 v) { return __uint_as_float((uint32_t)v); }
__device__ __forceinline__ float hi2(f32x2 v) { return __uint_as_float((uint32_t)(v >> 32)); }

__device__ __forceinline__ f32x2 fma2(f32x2 a, f32x2 b, f32x2 c) {
    f32x2 d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ f32x2 mul2(f32x2 a, f32x2 b) {
    f32x2 d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

// ------------------------------------------------------- group exchange --

// Transpose-reduce over the NL lanes of a group: on return v[0..VF) holds the
// group sums of entries lg*VF + e.
template <int V, int NL>
__device__ __forceinline__ void transpose_reduce(float (&v)[V], int lg) {
#pragma unroll
    for (int r = 0; (NL >> (r + 1)) >= 1; r++) {
        const int o = NL >> (r + 1);
        const int half = V >> (r + 1);
        const bool upper = (lg & o) != 0;
#pragma unroll
        for (int i = 0; i < half; i++) {
            const float send = upper ? v[i] : v[i + half];
            const float keep = upper ? v[i + half] : v[i];
            v[i] = keep + __shfl_xor_sync(KVQ_FULL_MASK, send, o);
        }
    }
}

// Inverse of transpose_reduce: from v[0..VF) (entries lg*VF + e) rebuild all
// V entries in every lane of the group.
template <int V, int NL>
__device__ __forceinline__ void transpose_gather(float (&v)[V], int lg) {
    constexpr int VF = V / NL;
#pragma unroll
    for (int r = 0; (1 << r) < NL; r++) {
        const int o = 1 << r;
        const int cur = VF << r;
        const bool upper = (lg & o) != 0;
#pragma unroll
        for (int i = 0; i < cur; i++) {
            const float mine = v[i];
            const float other = __shfl_xor_sync(KVQ_FULL_MASK, mine, o);
            v[i] = upper ? other : mine;
            v[i + cur] = upper ? mine : other;
        }
    }
}

// PP angle codes of this lane (bits [cb, cb + PP*bits) of a row), four at a
// time from 32-bit windows.  The second word of a window may lie past the
// row; it is in the staged shared memory and its bits are masked off.
template <int PP>
__device__ __forceinline__ void unpack_angles(const uint32_t* row, int cb, int bits,
                                              uint32_t (&a)[PP]) {
    const uint32_t mask = (1u << bits) - 1u;
#pragma unroll
    for (int q = 0; q < PP / 4; q++) {
        const int pos = cb + q * 4 * bits;
        const uint32_t win = __funnelshift_r(row[pos >> 5], row[(pos >> 5) + 1], pos & 31);
#pragma unroll
        for (int k = 0; k < 4; k++) a[4 * q + k] = (win >> (k * bits)) & mask;
    }
}

template <int NBYTES>
__device__ __forceinline__ void load_bytes(const uint8_t* p, uint32_t (&w)[(NBYTES + 3) / 4]) {
    if constexpr (NBYTES == 16) {
        const uint4 q = *reinterpret_cast<const uint4*>(p);
        w[0] = q.x; w[1] = q.y; w[2] = q.z; w[3] = q.w;
    } else if constexpr (NBYTES == 8) {
        const uint2 q = *reinterpret_cast<const uint2*>(p);
        w[0] = q.x; w[1] = q.y;
    } else if constexpr (NBYTES == 4) {
        w[0] = *reinterpret_cast<const uint32_t*>(p);
    } else {
        w[0] = *reinterpret_cast<const uint16_t*>(p);
    }
}

// ------------------------------------------------------------- kernel ---

template <int D, int G>
__global__ void __launch_bounds__(DecCfg<D, G>::THREADS, 1)
decode_kernel(DecodeArgs A) {
    using Cfg = DecCfg<D, G>;
    constexpr int P = Cfg::P, PP = Cfg::PP, NL = Cfg::NL, GPW = Cfg::GPW, NG = Cfg::NG;
    constexpr int WARPS = Cfg::WARPS, THREADS = Cfg::THREADS;
    constexpr int V = Cfg::V, VF = Cfg::VF;
    constexpr int EPQ = D / 32;

    extern __shared__ __align__(16) unsigned char smem[];
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem);             // [kStages]
    int* sflag = reinterpret_cast<int*>(smem + 32);                 // timeout, last
    // tables hold 2^bits entries so that any bit pattern indexes inside them
    const int nK = 1 << A.kc.bits, nV = 1 << A.vc.bits;
    float2* tabK = reinterpret_cast<float2*>(smem + 64);            // [2^bK][16]
    float2* tabV = tabK + nK * kTabRep;                             // [2^bV][16]
    float* qs = reinterpret_cast<float*>(tabV + nV * kTabRep);      // [G][D]
    unsigned char* stages = smem + A.stage_offset;                  // [kStages][stage]

    const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int grp = lane / NL, lg = lane % NL;
    const int gidx = warp * GPW + grp;
    const int l16 = lane & 15;

    // ---- token range of this split -----------------------------------------
    int64_t ctx = A.ctx_len[b];
    const int64_t lim = A.max_ctx < A.K.capacity ? A.max_ctx : A.K.capacity;
    if (ctx < 0 || ctx > lim) {
        if (split == 0 && kvh == 0 && tid == 0) report(A.err_word, KVQ_DEVERR_CTX_RANGE);
        ctx = ctx < 0 ? 0 : lim;
    }
    const int64_t t0 = (int64_t)split * A.split_len;
    const int64_t t1 = (t0 + A.split_len < ctx) ? t0 + A.split_len : ctx;
    const int ntiles = t1 > t0 ? (int)((t1 - t0 + kTT - 1) / kTT) : 0;

    const int64_t row0 = ((int64_t)b * A.H_kv + kvh) * A.K.capacity;
    const int rbK = A.kc.angle_words * 4, rbV = A.vc.angle_words * 4;
    const uint8_t* srcs[6] = {A.K.angles + row0 * rbK, A.K.norms + row0 * A.kc.norm_bytes,
                              A.K.params + row0 * A.kc.param_bytes, A.V.angles + row0 * rbV,
                              A.V.norms + row0 * A.vc.norm_bytes, A.V.params + row0 * A.vc.param_bytes};
    const int rbs[6] = {rbK, A.kc.norm_bytes, A.kc.param_bytes, rbV, A.vc.norm_bytes,
                        A.vc.param_bytes};

    auto issue_tile = [&](int tile) {  // thread 0 only
        const int s = tile % kStages;
        const int64_t tt0 = t0 + (int64_t)tile * kTT;
        const int64_t left = t1 - tt0;
        const int n16 = (int)(((left < kTT ? left : kTT) + 15) / 16 * 16);
        uint32_t bytes = 0;
#pragma unroll
        for (int k = 0; k < 6; k++) bytes += (uint32_t)(n16 * rbs[k]);
        fence_proxy_async();
        mbar_expect_tx(&bars[s], bytes);
        unsigned char* dst = stages + (size_t)s * A.stage_bytes;
#pragma unroll
        for (int k = 0; k < 6; k++)
            bulk_g2s(dst + A.lay[k], srcs[k] + tt0 * rbs[k], (uint32_t)(n16 * rbs[k]), &bars[s]);
    };

    if (tid == 0) {
        for (int s = 0; s < kStages; s++) mbar_init(&bars[s], 1);
        mbar_fence_init();
        sflag[0] = 0;
        sflag[1] = 0;
    }
    __syncthreads();
    int issued = 0;  // tiles issued so far (meaningful in thread 0)
    if (tid == 0)
        for (; issued < kStages && issued < ntiles; issued++) issue_tile(issued);

    // ---- cos/sin tables of the bin centres, 16 replicas -------------------
    for (int j = tid; j < nK; j += THREADS) {
        float s, c;
        sincospif((float)(2 * j + 1) / (float)A.kc.L - 1.f, &s, &c);
#pragma unroll
        for (int r = 0; r < kTabRep; r++) tabK[j * kTabRep + r] = make_float2(c, s);
    }
    for (int j = tid; j < nV; j += THREADS) {
        float s, c;
        sincospif((float)(2 * j + 1) / (float)A.vc.L - 1.f, &s, &c);
#pragma unroll
        for (int r = 0; r < kTabRep; r++) tabV[j * kTabRep + r] = make_float2(c, s);
    }
    // ---- q' = H D_K q / sqrt(d) for the G heads, one warp per head ---------
    for (int h = warp; h < G; h += WARPS) {
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

    f32x2 q2[G][PP];
#pragma unroll
    for (int h = 0; h < G; h++)
#pragma unroll
        for (int k = 0; k < PP; k++) {
            const float2 qq = reinterpret_cast<const float2*>(qs + h * D)[lg * PP + k];
            q2[h][k] = pack2(qq.x, qq.y);
        }

    f32x2 acc[G][PP];
#pragma unroll
    for (int h = 0; h < G; h++)
#pragma unroll
        for (int k = 0; k < PP; k++) acc[h][k] = 0ull;
    float mref[G];
#pragma unroll
    for (int h = 0; h < G; h++) mref[h] = -INFINITY;
    float lpart[VF];
#pragma unroll
    for (int e = 0; e < VF; e++) lpart[e] = 0.f;

    const int bitsK = A.kc.bits, bitsV = A.vc.bits;
    const int cbK = lg * PP * bitsK, cbV = lg * PP * bitsV;
    const float2* tK = tabK + l16;
    const float2* tV = tabV + l16;

    // ---- main loop over staged tiles ---------------------------------------
    int broken = ntiles;  // first tile not consumed after a timeout
    for (int tile = 0; tile < ntiles; tile++) {
        const int s = tile % kStages;
        if (!mbar_wait_bounded(&bars[s], (uint32_t)(tile / kStages) & 1u)) atomicOr(&sflag[0], 1);
        __syncthreads();
        if (sflag[0]) {
            broken = tile;
            break;
        }
        const unsigned char* st = stages + (size_t)s * A.stage_bytes;
        const uint32_t* sKa = reinterpret_cast<const uint32_t*>(st + A.lay[0]);
        const uint8_t* sKn = st + A.lay[1];
        const uint16_t* sKp = reinterpret_cast<const uint16_t*>(st + A.lay[2]);
        const uint32_t* sVa = reinterpret_cast<const uint32_t*>(st + A.lay[3]);
        const uint8_t* sVn = st + A.lay[4];
        const uint32_t* sVp = reinterpret_cast<const uint32_t*>(st + A.lay[5]);
        const int64_t tt0 = t0 + (int64_t)tile * kTT;
        const int ntok = (int)((t1 - tt0) < kTT ? (t1 - tt0) : kTT);

        for (int c = gidx; c < kTT / kTPG; c += NG) {
            // -- scores: partial dot products of this lane's pairs --------------
            float part[V];
#pragma unroll
            for (int j = 0; j < kTPG; j++) {
                const int t = c * kTPG + j;
                uint32_t a[PP];
                unpack_angles<PP>(sKa + t * A.kc.angle_words, cbK, bitsK, a);
                uint32_t nw[(PP + 3) / 4];
                load_bytes<PP>(sKn + t * P + lg * PP, nw);
                f32x2 dot[G];
#pragma unroll
                for (int h = 0; h < G; h++) dot[h] = 0ull;
#pragma unroll
                for (int k = 0; k < PP; k++) {
                    const float cf = (float)((nw[k / 4] >> (8 * (k % 4))) & 0xFFu);
                    const float2 cs = tK[a[k] * kTabRep];
                    const f32x2 xy = mul2(pack2(cf, cf), pack2(cs.x, cs.y));
#pragma unroll
                    for (int h = 0; h < G; h++) dot[h] = fma2(q2[h][k], xy, dot[h]);
                }
#pragma unroll
                for (int h = 0; h < G; h++) part[j * G + h] = lo2(dot[h]) + hi2(dot[h]);
            }
            transpose_reduce<V, NL>(part, lg);
            // -- scale by M/255 * tau * log2(e), mask, lazy softmax reference ---
            bool need = false;
#pragma unroll
            for (int e = 0; e < VF; e++) {
                const int idx = lg * VF + e;
                const int j = idx / G, h = idx % G;
                const int t = c * kTPG + j;
                const float M = half_bits_to_float(sKp[t]);
                float sv = part[e] * (M * (1.f / 255.f)) * A.scale_log2;
                sv = t < ntok ? sv : -INFINITY;
                part[e] = sv;
                float mh = mref[0];
#pragma unroll
                for (int hh = 1; hh < G; hh++) mh = (hh == h) ? mref[hh] : mh;
                need |= sv > mh + kLazyThr;
            }
            if (__any_sync(KVQ_FULL_MASK, need)) {
                float mx[G];
#pragma unroll
                for (int h = 0; h < G; h++) mx[h] = -INFINITY;
#pragma unroll
                for (int e = 0; e < VF; e++) {
                    const int h = (lg * VF + e) % G;
#pragma unroll
                    for (int hh = 0; hh < G; hh++)
                        if (hh == h) mx[hh] = fmaxf(mx[hh], part[e]);
                }
#pragma unroll
                for (int h = 0; h < G; h++) {
                    mx[h] = group_max<NL>(mx[h]);
                    const float mn = fmaxf(mref[h], mx[h]);
                    const float al = (mn == -INFINITY) ? 0.f : exp2f(mref[h] - mn);
                    const f32x2 al2 = pack2(al, al);
#pragma unroll
                    for (int k = 0; k < PP; k++) acc[h][k] = mul2(acc[h][k], al2);
#pragma unroll
                    for (int e = 0; e < VF; e++)
                        if ((lg * VF + e) % G == h) lpart[e] *= al;
                    mref[h] = mn;
                }
            }
#pragma unroll
            for (int e = 0; e < VF; e++) {
                const int h = (lg * VF + e) % G;
                float mh = mref[0];
#pragma unroll
                for (int hh = 1; hh < G; hh++) mh = (hh == h) ? mref[hh] : mh;
                const float p = part[e] == -INFINITY ? 0.f : exp2f(part[e] - mh);
                part[e] = p;
                lpart[e] += p;
            }
            transpose_gather<V, NL>(part, lg);
            // -- values: acc[h] += p[t][h] * r^ (cos, sin), rotated domain ------
#pragma unroll
            for (int j = 0; j < kTPG; j++) {
                const int t = c * kTPG + j;
                const bool valid = t < ntok;
                uint32_t a[PP];
                unpack_angles<PP>(sVa + t * A.vc.angle_words, cbV, bitsV, a);
                uint32_t nw[(PP / 2 + 3) / 4];
                load_bytes<PP / 2>(sVn + t * (P / 2) + lg * (PP / 2), nw);
                const uint32_t pr = sVp[t];
                const float LO = half_bits_to_float((uint16_t)(pr & 0xFFFF));
                const float HI = half_bits_to_float((uint16_t)(pr >> 16));
                const float step = (HI - LO) * (1.f / 15.f);
                f32x2 pw[G];
#pragma unroll
                for (int h = 0; h < G; h++) pw[h] = pack2(part[j * G + h], part[j * G + h]);
#pragma unroll
                for (int k = 0; k < PP; k++) {
                    const float cf = (float)((nw[k / 8] >> (4 * (k % 8))) & 0xFu);
                    float r = exp2f(fmaf(cf, step, LO));
                    r = valid ? r : 0.f;
                    const float2 cs = tV[a[k] * kTabRep];
                    const f32x2 xy = mul2(pack2(r, r), pack2(cs.x, cs.y));
#pragma unroll
                    for (int h = 0; h < G; h++) acc[h][k] = fma2(pw[h], xy, acc[h][k]);
                }
            }
        }
        __syncthreads();
        if (tid == 0 && tile + kStages < ntiles) {
            issue_tile(tile + kStages);
            issued = tile + kStages + 1;
        }
    }

    if (sflag[0]) {
        // a stage never arrived: report, then wait (bounded) for the copies
        // still in flight before the shared memory is released
        if (tid == 0) {
            report(A.err_word, KVQ_DEVERR_TIMEOUT);
            for (int t = broken; t < issued; t++)
                (void)mbar_wait_bounded(&bars[t % kStages], (uint32_t)(t / kStages) & 1u);
        }
        __syncthreads();
#pragma unroll
        for (int h = 0; h < G; h++) {
            mref[h] = -INFINITY;
#pragma unroll
            for (int k = 0; k < PP; k++) acc[h][k] = 0ull;
        }
#pragma unroll
        for (int e = 0; e < VF; e++) lpart[e] = 0.f;
    }

    // ---- merge the NG group states of this CTA (reuses the stage memory) --
    float* gm = reinterpret_cast<float*>(stages);  // [NG][G]
    float* gl = gm + NG * G;                      // [NG][G]
    float* gacc = gl + NG * G;                    // [NG][G][D]
    __syncthreads();
    float lh[G];
#pragma unroll
    for (int h = 0; h < G; h++) lh[h] = 0.f;
#pragma unroll
    for (int e = 0; e < VF; e++) {
        const int h = (lg * VF + e) % G;
#pragma unroll
        for (int hh = 0; hh < G; hh++)
            if (hh == h) lh[hh] += lpart[e];
    }
#pragma unroll
    for (int h = 0; h < G; h++) lh[h] = group_sum<NL>(lh[h]);
    if (lg == 0) {
#pragma unroll
        for (int h = 0; h < G; h++) {
            gm[gidx * G + h] = mref[h];
            gl[gidx * G + h] = lh[h];
        }
    }
#pragma unroll
    for (int h = 0; h < G; h++)
#pragma unroll
        for (int k = 0; k < PP; k++) {
            const int i = lg * PP + k;
            reinterpret_cast<float2*>(gacc + (gidx * G + h) * D)[i] =
                make_float2(lo2(acc[h][k]), hi2(acc[h][k]));
        }
    __syncthreads();

    const int S = A.num_splits;
    float* stats = A.ws + ws_counter_floats(A.B, A.H_q);
    float* accs = stats + ws_stat_floats(A.B, A.H_q, S);
    for (int idx = tid; idx < G * D; idx += THREADS) {
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
        const int64_t slot = ((int64_t)b * A.H_q + (int64_t)kvh * G + h) * S + split;
        accs[slot * D + j] = sum_a;
        if (j == 0) {
            stats[slot * 2] = mx;
            stats[slot * 2 + 1] = sum_l;
        }
    }

    // ---- the last CTA of this (b, KV head) merges the splits ----------------
    __threadfence();
    __syncthreads();
    int* counters = reinterpret_cast<int*>(A.ws);
    if (tid == 0) {
        const int prev = atomicAdd(&counters[b * A.H_kv + kvh], 1);
        sflag[1] = (prev == S - 1);
    }
    __syncthreads();
    if (!sflag[1]) return;
    __threadfence();
    for (int h = warp; h < G; h += WARPS) {
        const int64_t hq = (int64_t)b * A.H_q + (int64_t)kvh * G + h;
        const float* st = stats + hq * S * 2;
        const float* ac = accs + hq * S * D;
        float mx = -INFINITY;
        for (int s = lane; s < S; s += 32) mx = fmaxf(mx, __ldcg(st + 2 * s));
        mx = group_max<32>(mx);
        float v[EPQ];
#pragma unroll
        for (int e = 0; e < EPQ; e++) v[e] = 0.f;
        float sum_l = 0.f;
        if (mx != -INFINITY) {
            for (int s = 0; s < S; s++) {
                const float w = exp2f(__ldcg(st + 2 * s) - mx);
                sum_l += w * __ldcg(st + 2 * s + 1);
#pragma unroll
                for (int e = 0; e < EPQ; e++)
                    v[e] = fmaf(w, __ldcg(ac + (int64_t)s * D + lane * EPQ + e), v[e]);
            }
        }
        const float inv = sum_l > 0.f ? 1.f / sum_l : 0.f;
#pragma unroll
        for (int e = 0; e < EPQ; e++) v[e] *= inv;
        fwht_local<EPQ>(v);
        fwht_cross<EPQ, 32>(v, lane);
        const float isd = rsqrtf((float)D);
#pragma unroll
        for (int e = 0; e < EPQ; e++) {
            const int j = lane * EPQ + e;
            float o = v[e] * isd;
            o = A.signs_v[j] < 0 ? -o : o;
            if (A.out_dtype == 0)
                reinterpret_cast<__half*>(A.out)[hq * D + j] = __float2half_rn(o);
            else
                reinterpret_cast<float*>(A.out)[hq * D + j] = o;
        }
    }
    if (tid == 0) atomicExch(&counters[b * A.H_kv + kvh], 0);
}

// ------------------------------------------------------------------ host --

template <int D, int G>
static cudaError_t launch_decode_dg(DecodeArgs a, cudaStream_t stream) {
    using Cfg = DecCfg<D, G>;
    // shared memory: barriers/flags, two replicated tables, q', stages
    size_t off = 64 + sizeof(float2) * kTabRep * (size_t)((1 << a.kc.bits) + (1 << a.vc.bits)) +
                 sizeof(float) * G * D;
    off = (off + 15) / 16 * 16;
    a.stage_offset = (int)off;
    const int rb[6] = {a.kc.angle_words * 4, a.kc.norm_bytes, a.kc.param_bytes,
                       a.vc.angle_words * 4, a.vc.norm_bytes, a.vc.param_bytes};
    int sb = 0;
    for (int k = 0; k < 6; k++) {
        a.lay[k] = sb;
        sb += (kTT * rb[k] + 15) / 16 * 16;
    }
    a.stage_bytes = sb;
    size_t ring = (size_t)kStages * sb;
    const size_t merge = sizeof(float) * ((size_t)2 * Cfg::NG * G + (size_t)Cfg::NG * G * D);
    if (ring < merge) ring = merge;
    const size_t smem = off + ring;
    if (smem > 227 * 1024) return cudaErrorInvalidConfiguration;
    static bool attr_done[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64 || !attr_done[dev]) {
        e = cudaFuncSetAttribute(decode_kernel<D, G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 227 * 1024);
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) attr_done[dev] = true;
    }
    dim3 grid((unsigned)a.num_splits, (unsigned)a.H_kv, (unsigned)a.B);
    decode_kernel<D, G><<<grid, Cfg::THREADS, smem, stream>>>(a);
    return cudaGetLastError();
}

bool decode_supported(int d, int G, int LK, int LV, int mode_k, int mode_v) {
    if (d != 64 && d != 128) return false;
    if (G != 1 && G != 2 && G != 4 && G != 8) return false;
    if (mode_k != KVQ_NORM_LIN8 || mode_v != KVQ_NORM_LOG4) return false;
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
