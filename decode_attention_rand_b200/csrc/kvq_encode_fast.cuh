// kvq_encode_fast.cuh - the streaming encode for head_dim 64, 128 and 256 and
// codebooks with L % 8 == 0, 16 <= L <= 256 (angle codes of 4 to 8 bits);
// codec of "TurboAngle: Near-Lossless KV Cache Compression via Uniform Angle
// Quantization", Abstract.  Produces the same codes as encode_tile, byte for
// byte, with a third of its instructions.
//
// Layout: 32 elements per lane, NL = d / 32 lanes per vector, 32 / NL vectors
// per warp tile; 128-bit streaming loads.
//
// The Walsh-Hadamard transform runs in fp32 on packed two-lane adds, and its
// butterfly between elements 2i and 2i+1 is never applied: with w the
// transform over the other index bits, the rotated pair is
//     (z[2i], z[2i+1]) = (w[2i] + w[2i+1], w[2i] - w[2i+1]),
// a reflection of (w[2i], w[2i+1]) scaled by sqrt 2, so |z| = sqrt(2) |w| and
// angle(z) = pi/4 - angle(w); the bin (angle(z) + pi) L / 2pi is then
// 5L/8 - angle(w) L / 2pi (mod L).
//
// Exactness.  Each input is split as x = hi + lo, hi being x rounded to a
// multiple of 2^(E+S-24) where |x| < 2^(E+1) over the vector (S = log2 d):
// a sum of 2^(S-1) such values is an integer multiple below 2^24, so the
// transform of hi is exact in fp32.  lo is a multiple of 2^-24 (as every fp16
// value is) below 2^(E+S-25), and its transform is exact too when
// E <= 26 - 2S.  Then w = hi_w + lo_w exactly, the decisions see w rounded
// once to fp32 (the slacks of encode_tile cover that), and a decision in doubt
// is re-taken from the exact pair, formed in fp64, by exact_fast.  Vectors
// with a larger E (|x| >= 2^(27-2S)) go through the general fp64 path.
#pragma once

#include "kvq_encode_impl.cuh"

namespace kvq {

template <int D>
struct FastCfg {
    static_assert(D == 64 || D == 128 || D == 256, "fast encode covers d = 64, 128, 256");
    static constexpr int EPL = 32;        // elements per lane
    static constexpr int NL = D / 32;     // lanes per vector
    static constexpr int PPL = 16;        // pairs per lane
    static constexpr int VPW = 32 / NL;   // vectors per warp tile
    static constexpr int S = D == 64 ? 6 : D == 128 ? 7 : 8;  // log2 d
};

constexpr int kFastWarps = 8;
constexpr int kFastBlocksPerSM = 2;

// Clamped shifts (a shift by 32 gives 0): one funnel-shift instruction each.
__device__ __forceinline__ uint32_t shl_c(uint32_t x, uint32_t n) {
    return __funnelshift_lc(0u, x, n);
}
__device__ __forceinline__ uint32_t shr_c(uint32_t x, uint32_t n) {
    return __funnelshift_rc(x, 0u, n);
}

// fp16 sign-bit masks of D for the 16 element pairs of lane lg: bit 15 for
// the even element, bit 31 for the odd one.
__device__ __forceinline__ void fast_sign_masks(const int8_t* signs, int lg, uint32_t* smask) {
#pragma unroll
    for (int w = 0; w < 16; w++) {
        const int e = lg * 32 + 2 * w;
        smask[w] = (signs[e] < 0 ? 0x8000u : 0u) | (signs[e + 1] < 0 ? 0x80000000u : 0u);
    }
}

// The 32 inputs of this lane with the signs of D applied (fp16 pairs);
// smask points at the lane's 16 masks in shared memory.
template <int D>
__device__ __forceinline__ void fast_load(const EncArgs& A, uint32_t v, int lg,
                                          const uint32_t* smask, uint32_t (&raw)[16]) {
    const uint4* src = reinterpret_cast<const uint4*>(A.x + (size_t)v * D + lg * 32);
    const uint4* msk = reinterpret_cast<const uint4*>(smask);
#pragma unroll
    for (int q = 0; q < 4; q++) {
        const uint4 t = __ldcs(src + q);
        const uint4 m = msk[q];
        raw[4 * q + 0] = t.x ^ m.x;
        raw[4 * q + 1] = t.y ^ m.y;
        raw[4 * q + 2] = t.z ^ m.z;
        raw[4 * q + 3] = t.w ^ m.w;
    }
}


// Transform over index bits 1 .. S-1 of 16 packed pairs: local butterflies on
// pair strides 1, 2, 4, 8, then the lanes of the group.
template <int NL>
__device__ __forceinline__ void fwht_pairs(f32x2 (&P)[16], int lg) {
#pragma unroll
    for (int s = 1; s < 16; s <<= 1) {
#pragma unroll
        for (int k = 0; k < 16; k++) {
            if ((k & s) == 0) {
                const f32x2 a = P[k], b = P[k + s];
                P[k] = add2(a, b);
                P[k + s] = sub2(a, b);
            }
        }
    }
#pragma unroll
    for (int m = 1; m < NL; m <<= 1) {
        // lower lane: own + other; upper lane: other - own
        const float sg = (lg & m) ? -1.f : 1.f;
        const f32x2 sg2 = pack2(sg, sg);
#pragma unroll
        for (int k = 0; k < 16; k++) {
            const uint32_t lo = __shfl_xor_sync(KVQ_FULL_MASK, (uint32_t)P[k], m);
            const uint32_t hi = __shfl_xor_sync(KVQ_FULL_MASK, (uint32_t)(P[k] >> 32), m);
            P[k] = fma2(sg2, P[k], ((f32x2)hi << 32) | lo);
        }
    }
}

// The split transform of the header: HI and LO hold the transforms of hi and
// lo (pairs (w[2k], w[2k+1]) of this lane); E as defined there and whether
// the vector is all zero (both uniform over the group).
template <int D>
__device__ __forceinline__ void split_fwht(const uint32_t (&raw)[16], int lg, f32x2 (&HI)[16],
                                           f32x2 (&LO)[16], int& E, bool& zero) {
    constexpr int NL = FastCfg<D>::NL, S = FastCfg<D>::S;
    // largest |x|: non-negative fp16 values order like their bit patterns
    __half2 mh = __float2half2_rn(0.f);
#pragma unroll
    for (int k = 0; k < 16; k++) {
        const uint32_t a = raw[k] & 0x7FFF7FFFu;
        mh = __hmax2(mh, *reinterpret_cast<const __half2*>(&a));
    }
    const uint32_t mb = *reinterpret_cast<const uint32_t*>(&mh);
    uint32_t m = max(mb & 0xFFFFu, mb >> 16);
#pragma unroll
    for (int o = 1; o < NL; o <<= 1) m = max(m, __shfl_xor_sync(KVQ_FULL_MASK, m, o));
    zero = m == 0u;
    E = (int)max(m >> 10, 1u) - 15;  // |x| < 2^(E+1)
    // adding and removing 1.5 * 2^(E+S-1) rounds x to a multiple of 2^(E+S-24)
    const float C = __uint_as_float(((uint32_t)(E + S - 1 + 127) << 23) | 0x400000u);
    const f32x2 C2 = pack2(C, C);
#pragma unroll
    for (int k = 0; k < 16; k++) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&raw[k]));
        const f32x2 X = pack2(f.x, f.y);
        HI[k] = sub2(add2(X, C2), C2);
        LO[k] = sub2(X, HI[k]);
    }
    fwht_pairs<NL>(HI, lg);
    fwht_pairs<NL>(LO, lg);
}

// r (LIN8) or log2 max(r, 2^-24) (LOG4) of an exact rotated pair, in fp64
// (the formulas of exact_path); inv_d = 1/d.
static __device__ __noinline__ double exact_norm_value(double z0, double z1, bool lin8,
                                                       double inv_d) {
    const double r2 = fma(z0, z0, z1 * z1) * inv_d;
    return lin8 ? sqrt(r2) : 0.5 * exact_log2_sq(r2);
}

// Per-lane state handed to exact_fast through shared memory: word i of lane
// l at st[i * 32 + l] (the lane's column; no bank conflicts).
constexpr int kFsNv = 0;      // 16 words: LIN8 |w pair|, LOG4 fp32 log2 r
constexpr int kFsQ4 = 16;     // 4 words: angle codes, four per word
constexpr int kFsNc = 20;     // 4 words: norm codes (bytes or nibbles)
constexpr int kFsNeedA = 24, kFsNeedN = 25, kFsPrm = 26, kFsPmin = 27, kFsPmax = 28,
              kFsPband = 29, kFsFlags = 30;
constexpr uint32_t kFsValid = 1u, kFsNeedP = 2u, kFsUnsure = 4u, kFsInexact = 8u;
constexpr int kFsWords = 32;

// Parameter of a vector left for the fixup pass: an fp16 NaN (LIN8 M) or two
// (LOG4 LO, HI), values the codec never stores (its parameters saturate to
// finite fp16).
constexpr uint32_t kFixupMark16 = 0xFFFFu;
constexpr uint32_t kFixupMark32 = 0xFFFFFFFFu;

// The decisions in doubt of one warp tile.  From the split transform, the
// exact pair (w0, w1) is hi_w + lo_w in fp64, and z = (w0 + w1, w0 - w1) is
// exact as well; each lane re-takes its own flagged decisions with the
// definition's formulas (encode_tile's exact_path rules: a parameter in doubt
// is settled by the pairs that can hold the extreme, and if it moves every
// norm code of the vector is re-decided).  A warp holding a vector outside
// the exact range of the split takes the general fp64 path (exact_fixup).
// Out of line, fed through shared memory, so the streaming loop keeps its
// registers; called by every lane of the warp.
template <int D>
__device__ __noinline__ void exact_fast(const __half* x, const uint32_t* smask, uint32_t v, int lg,
                                        uint32_t* st, int L, int mode, int bits, float bpr) {
    using Cfg = FastCfg<D>;
    constexpr int NL = Cfg::NL;
    const float sc = (float)(Cfg::S == 6 ? 0.17677669529663687
                                         : Cfg::S == 7 ? 0.125 : 0.08838834764831845);
    uint32_t raw[16];
    {
        const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)v * D + lg * 32);
        const uint4* msk = reinterpret_cast<const uint4*>(smask);
#pragma unroll
        for (int q = 0; q < 4; q++) {
            const uint4 t = src[q];
            const uint4 m = msk[q];
            raw[4 * q + 0] = t.x ^ m.x;
            raw[4 * q + 1] = t.y ^ m.y;
            raw[4 * q + 2] = t.z ^ m.z;
            raw[4 * q + 3] = t.w ^ m.w;
        }
    }
    const bool lin8 = mode == KVQ_NORM_LIN8;
    const uint32_t am = (1u << bits) - 1u;
    int acode[16], ncode[16];
#pragma unroll
    for (int k = 0; k < 16; k++) {
        acode[k] = (int)((st[(kFsQ4 + (k >> 2)) * 32] >> ((uint32_t)bits * (uint32_t)(k & 3))) & am);
        ncode[k] = lin8 ? (int)((st[(kFsNc + (k >> 2)) * 32] >> (8 * (k & 3))) & 255u)
                        : (int)((st[(kFsNc + (k >> 3)) * 32] >> (4 * (k & 7))) & 15u);
    }
    const uint32_t need_a = st[kFsNeedA * 32], need_n = st[kFsNeedN * 32];
    uint32_t prm = st[kFsPrm * 32];
    const float pmin = __uint_as_float(st[kFsPmin * 32]), pmax = __uint_as_float(st[kFsPmax * 32]),
                pband = __uint_as_float(st[kFsPband * 32]);
    const uint32_t fl = st[kFsFlags * 32];
    const bool valid = fl & kFsValid, need_p = fl & kFsNeedP, unsure = fl & kFsUnsure;
    // fp32 value of pair k the parameter decision was based on
    auto v32 = [&](int k) -> float {
        const float nv = __uint_as_float(st[(kFsNv + k) * 32]);
        return lin8 ? nv * sc : nv;
    };
    if (__any_sync(KVQ_FULL_MASK, (fl & kFsInexact) != 0u)) {
        ExactIn<16> in;
#pragma unroll
        for (int k = 0; k < 16; k++) {
            in.raw[k] = raw[k];
            in.rr[k] = lin8 ? v32(k) : 0.f;
            in.ll[k] = lin8 ? 0.f : v32(k);
            in.acode[k] = acode[k];
            in.ncode[k] = ncode[k];
        }
        in.need_a = need_a;
        in.need_n = need_n;
        in.prm = prm;
        in.pmin = pmin;
        in.pmax = pmax;
        in.pband = pband;
        in.valid = valid;
        in.need_p = need_p;
        in.unsure = unsure;
        const ExactOut<16> o = exact_fixup<D, Cfg>(in, lg, L, mode);
#pragma unroll
        for (int k = 0; k < 16; k++) {
            acode[k] = o.acode[k];
            ncode[k] = o.ncode[k];
        }
        prm = o.prm;
    } else {
        // the exact rotated pairs (rolled loops below index them at run time,
        // from local memory: this path is rare, its code is kept small)
        double z0[16], z1[16];
        {
            f32x2 HI[16], LO[16];
            int E;
            bool zero;
            split_fwht<D>(raw, lg, HI, LO, E, zero);
            (void)E;
            (void)zero;
#pragma unroll
            for (int k = 0; k < 16; k++) {
                const double w0 = (double)lo2(HI[k]) + (double)lo2(LO[k]);
                const double w1 = (double)hi2(HI[k]) + (double)hi2(LO[k]);
                z0[k] = w0 + w1;
                z1[k] = w0 - w1;
            }
        }
#pragma unroll 1
        for (uint32_t t = valid ? need_a : 0u; t; t &= t - 1u) {
            const int k = __ffs(t) - 1;
            acode[k] = angle_code_from_exact(z0[k], z1[k], L, bpr);
        }
        const bool gp = valid && need_p;  // uniform within the group
        bool redo = false;
        if (__any_sync(KVQ_FULL_MASK, gp)) {
            double ext_hi = lin8 ? 0.0 : -1e300, ext_lo = 1e300;
            uint32_t ch = 0, cl = 0;  // candidates for the largest / smallest value
            if (gp) {
#pragma unroll
                for (int k = 0; k < 16; k++) {
                    const float f = v32(k);
                    if (unsure || f >= pmax - pband) ch |= 1u << k;
                    if (!lin8 && (unsure || f <= pmin + pband)) cl |= 1u << k;
                }
            }
#pragma unroll 1
            for (uint32_t t = ch | cl; t; t &= t - 1u) {
                const int k = __ffs(t) - 1;
                const double xk = exact_norm_value(z0[k], z1[k], lin8, 1.0 / D);
                if ((ch >> k) & 1u) ext_hi = fmax(ext_hi, xk);
                if ((cl >> k) & 1u) ext_lo = fmin(ext_lo, xk);
            }
            ext_hi = group_max_d<NL>(ext_hi);
            ext_lo = group_min_d<NL>(ext_lo);
            if (gp) {
                const uint32_t px = lin8 ? (uint32_t)f64_to_f16_sat(ext_hi)
                                         : ((uint32_t)f64_to_f16_sat(ext_lo) |
                                            ((uint32_t)f64_to_f16_sat(ext_hi) << 16));
                redo = unsure || px != prm;
                prm = px;
            }
        }
        const double M = (double)half_bits_to_float((uint16_t)(prm & 0xFFFF));
        const double HIp = (double)half_bits_to_float((uint16_t)(prm >> 16));
#pragma unroll 1
        for (uint32_t t = redo ? 0xFFFFu : (valid ? need_n : 0u); t; t &= t - 1u) {
            const int k = __ffs(t) - 1;
            const double xk = exact_norm_value(z0[k], z1[k], lin8, 1.0 / D);
            ncode[k] = lin8 ? lin8_code_exact(xk, M) : log4_code_exact(xk, M, HIp);
        }
    }
    uint32_t q4[4] = {0u, 0u, 0u, 0u}, nc[4] = {0u, 0u, 0u, 0u};
#pragma unroll
    for (int k = 0; k < 16; k++) {
        q4[k >> 2] |= (uint32_t)acode[k] << ((uint32_t)bits * (uint32_t)(k & 3));
        if (lin8)
            nc[k >> 2] |= (uint32_t)ncode[k] << (8 * (k & 3));
        else
            nc[k >> 3] |= (uint32_t)ncode[k] << (4 * (k & 7));
    }
#pragma unroll
    for (int j = 0; j < 4; j++) {
        st[(kFsQ4 + j) * 32] = q4[j];
        st[(kFsNc + j) * 32] = nc[j];
    }
    st[kFsPrm * 32] = prm;
}

// One warp tile: vector v per group of NL lanes (lanes past n_vec compute on
// vector 0 and store nothing).  pwk = {1, 2^b, 2^2b, 2^3b} places four b-bit
// angle codes in one word; st is this lane's column of the warp's state.
template <int D, bool EXACT>
__device__ __forceinline__ void encode_tile_fast(const EncArgs& A, uint32_t v,
                                                 const uint32_t* smask, int lg,
                                                 const uint32_t (&pwk)[4], uint32_t* st) {
    using Cfg = FastCfg<D>;
    constexpr int NL = Cfg::NL, S = Cfg::S;
    const bool valid = (int64_t)v < A.n_vec;
    const int L = A.c.L;
    const bool lin8 = A.c.mode == KVQ_NORM_LIN8;

    // ---- load, D, split transform: P[k] = (w[2k], w[2k+1]) rounded once ---
    f32x2 P[16];
    int E;
    bool zero;
    {
        uint32_t raw[16];
        fast_load<D>(A, valid ? v : 0u, lg, smask, raw);
        f32x2 HI[16], LO[16];
        split_fwht<D>(raw, lg, HI, LO, E, zero);
#pragma unroll
        for (int k = 0; k < 16; k++) P[k] = add2(HI[k], LO[k]);
    }
    const bool inexact = E > 26 - 2 * S;  // lo's transform may have rounded
    // sqrt(2/d): scaled norm r = |z| / sqrt(d) = sqrt(2/d) |w pair|
    const float sc = (float)(S == 6 ? 0.17677669529663687 : S == 7 ? 0.125 : 0.08838834764831845);

    // ---- angles ------------------------------------------------------------
    const float bpr = A.bins_per_rad;
    const float u0 = 0.625f * (float)L;  // 5L/8
    const float du = angle_margin(A);
    uint32_t q4[4] = {0u, 0u, 0u, 0u};  // angle codes, four per word
    uint32_t need_a = 0;
    float rw2[16];
#pragma unroll
    for (int k = 0; k < 16; k++) {
        const float a = lo2(P[k]), b = hi2(P[k]);
        rw2[k] = fmaf(a, a, b * b);
        const float th = atan2_poly(b, a);
        const float u = fmaf(th, -bpr, u0);
        const float fl = floorf(u);
        const float fr = u - fl;
        int c = (int)fl;
        c = c >= L ? c - L : c;
        // an exactly zero pair has code 0 (its fr is NaN: never flagged)
        c = rw2[k] > 0.f ? c : 0;
        q4[k >> 2] += (uint32_t)c * pwk[k & 3];
        need_a |= (0.5f - fabsf(fr - 0.5f) < du) ? (1u << k) : 0u;
    }

    // ---- norms and parameters (the formulas and slacks of encode_tile) ----
    uint32_t nc[4] = {0u, 0u, 0u, 0u};  // norm codes: 4 bytes (LIN8) / 8 nibbles (LOG4) a word
    float nv[16];  // LIN8: |w pair|; LOG4: fp32 log2 r
    uint32_t prm = 0, need_n = 0;
    bool need_p = false, unsure = false;
    float pmax = 0.f, pmin = 0.f, pband = 0.f;
    if (lin8) {
        float m = 0.f;
#pragma unroll
        for (int k = 0; k < 16; k++) {
            nv[k] = sqrt_approx(rw2[k]);
            m = fmaxf(m, nv[k]);
        }
        m = group_max<NL>(m) * sc;  // max r
        const float eM = m * 1e-6f;
        need_p = near_f16_midpoint(m, eM);
        pmax = m;
        pband = 2.f * eM;
        const uint16_t Mh = f32_to_f16_sat(m);
        const float Mf = half_bits_to_float(Mh);
        prm = Mh;
        const float inv = Mf > 0.f ? 255.f * rcp_approx(Mf) : 0.f;
        const float invw = inv * sc;
#pragma unroll
        for (int k = 0; k < 16; k++) {
            const float vq = nv[k] * invw;
            const float t = vq + 0.5f;
            const float fl = floorf(t);
            const float fr = t - fl;
            const float dv = fmaf(vq, 1.2e-6f, 2e-6f);
            if (Mf > 0.f && (fr < dv || fr > 1.f - dv)) need_n |= 1u << k;
            const uint32_t c = Mf > 0.f ? (uint32_t)min(255, (int)fl) : 0u;
            nc[k >> 2] |= c << (8 * (k & 3));
        }
    } else {
        // l = log2 max(r, 2^-24) with r^2 = (2/d) rw2:
        // l = (log2 max(rw2, 2^(S-49)) + 1 - S) / 2
        const float lfloor = __uint_as_float((uint32_t)(S - 49 + 127) << 23);
        const float tiny = __uint_as_float((uint32_t)(S - 45 + 127) << 23);  // r < 2^-22
        float lmin = 1e30f, lmax = -1e30f;
#pragma unroll
        for (int k = 0; k < 16; k++) {
            nv[k] = fmaf(0.5f, lg2_approx(fmaxf(rw2[k], lfloor)), 0.5f * (float)(1 - S));
            unsure |= rw2[k] < tiny;
            lmin = fminf(lmin, nv[k]);
            lmax = fmaxf(lmax, nv[k]);
        }
        unsure &= !zero;  // a zero vector is exact: every l is -24
        lmin = group_min<NL>(lmin);
        lmax = group_max<NL>(lmax);
        unsure = group_any<NL>(unsure);
        // log2 error of a pair norm (relative 1e-6 of r, lg2 approximation),
        // as in encode_tile, plus 2^-23 of |l|
        const float elmax = fmaf(fmaxf(fabsf(lmin), fabsf(lmax)), 1.2e-7f, 2.6717e-6f);
        need_p = unsure || near_f16_midpoint(lmin, elmax) || near_f16_midpoint(lmax, elmax);
        pmin = lmin;
        pmax = lmax;
        pband = 2.f * elmax;
        const uint16_t LOh = f32_to_f16_sat(lmin), HIh = f32_to_f16_sat(lmax);
        const float LOf = half_bits_to_float(LOh), HIf = half_bits_to_float(HIh);
        prm = (uint32_t)LOh | ((uint32_t)HIh << 16);
        const float inv = HIf != LOf ? 15.f * rcp_approx(HIf - LOf) : 0.f;
#pragma unroll
        for (int k = 0; k < 16; k++) {
            const float vq = (nv[k] - LOf) * inv;
            const float t = vq + 0.5f;
            const float fl = floorf(t);
            const float fr = t - fl;
            const float dv = (2.6717e-6f + (fabsf(nv[k]) + fabsf(LOf)) * 1.2e-7f) * inv * 1.02f +
                             fabsf(vq) * 1e-6f + 2e-6f;
            if (HIf != LOf && (fr < dv || fr > 1.f - dv)) need_n |= 1u << k;
            const uint32_t c = HIf != LOf ? (uint32_t)min(15, max(0, (int)fl)) : 0u;
            nc[k >> 3] |= c << (4 * (k & 7));
        }
    }
    if (inexact) {
        need_a = need_n = 0xFFFFu;
        need_p = unsure = true;
    }

    // ---- decisions in doubt ----------------------------------------------------
    // streaming pass: the vector keeps its fp32 codes and gets the marker
    // parameter (fixup pass); fixup pass: exact_fast re-takes them
    const uint32_t bits = (uint32_t)A.c.bits;
    const bool lane_need = valid && ((need_a | need_n) != 0u || need_p);
    if constexpr (!EXACT) {
        if (group_any<NL>(lane_need)) prm = lin8 ? kFixupMark16 : kFixupMark32;
    } else if (__any_sync(KVQ_FULL_MASK, lane_need)) {
#pragma unroll
        for (int k = 0; k < 16; k++) st[(kFsNv + k) * 32] = __float_as_uint(nv[k]);
#pragma unroll
        for (int j = 0; j < 4; j++) {
            st[(kFsQ4 + j) * 32] = q4[j];
            st[(kFsNc + j) * 32] = nc[j];
        }
        st[kFsNeedA * 32] = need_a;
        st[kFsNeedN * 32] = need_n;
        st[kFsPrm * 32] = prm;
        st[kFsPmin * 32] = __float_as_uint(pmin);
        st[kFsPmax * 32] = __float_as_uint(pmax);
        st[kFsPband * 32] = __float_as_uint(pband);
        st[kFsFlags * 32] = (valid ? kFsValid : 0u) | (need_p ? kFsNeedP : 0u) |
                            (unsure ? kFsUnsure : 0u) | (inexact ? kFsInexact : 0u);
        exact_fast<D>(A.x, smask, valid ? v : 0u, lg, st, L, A.c.mode, (int)bits, bpr);
#pragma unroll
        for (int j = 0; j < 4; j++) {
            q4[j] = st[(kFsQ4 + j) * 32];
            nc[j] = st[(kFsNc + j) * 32];
        }
        prm = st[kFsPrm * 32];
    }

    // ---- pack and store ------------------------------------------------------
    // angle stream of this lane: 16 codes of b bits at bit 16 b lg of the row
    const uint32_t s4 = 4u * bits;  // 16 .. 32
    const uint32_t a0 = q4[0] | shl_c(q4[1], s4), a1 = shr_c(q4[1], 32u - s4);
    const uint32_t b0 = q4[2] | shl_c(q4[3], s4), b1 = shr_c(q4[3], 32u - s4);
    const uint32_t r8 = 8u * bits - 32u;  // 0 .. 32: offset of codes 8..15 past word 1
    uint32_t o[4];
    o[0] = a0;
    o[1] = a1 | shl_c(b0, r8);
    o[2] = shr_c(b0, 32u - r8) | shl_c(b1, r8);
    o[3] = shr_c(b1, 32u - r8);
    if (bits & 1u) {
        // odd b: odd lanes start half way into a word; they hand their first
        // 16 bits to the lane below, which completes its last word with them
        const uint32_t up = __shfl_down_sync(KVQ_FULL_MASK, o[0], 1);
        const uint32_t last = (bits - 1u) >> 1;  // half-filled word of an even lane
        if (lg & 1) {
            o[0] = __funnelshift_r(o[0], o[1], 16);
            o[1] = __funnelshift_r(o[1], o[2], 16);
            o[2] = __funnelshift_r(o[2], o[3], 16);
            o[3] >>= 16;
        } else {
#pragma unroll
            for (int j = 0; j < 4; j++)
                if ((uint32_t)j == last) o[j] |= up << 16;
        }
    }
    if (valid) {
        const uint32_t vt = fast_div(v, A.tdiv);
        bool bad = false;
        const int64_t row =
            plane_row_bh(A.out, A.bh0 + vt, A.pos0 + (int64_t)(v - vt * (uint32_t)A.T), &bad);
        if (bad && lg == 0) report(A.err_word, KVQ_DEVERR_PAGE_RANGE);
        // this lane's words: [ceil(lg b / 2), ceil((lg + 1) b / 2))
        const uint32_t w0 = ((uint32_t)lg * bits + 1u) >> 1;
        const uint32_t nw = (((uint32_t)lg + 1u) * bits + 1u) / 2u - w0;
        uint32_t* dst = reinterpret_cast<uint32_t*>(A.out.angles) + row * A.c.angle_words + w0;
#pragma unroll
        for (int j = 0; j < 4; j++)
            if ((uint32_t)j < nw) dst[j] = o[j];
        if (lin8) {
            *reinterpret_cast<uint4*>(A.out.norms + row * (D / 2) + lg * 16) =
                make_uint4(nc[0], nc[1], nc[2], nc[3]);
            if (lg == 0) reinterpret_cast<uint16_t*>(A.out.params)[row] = (uint16_t)prm;
        } else {
            *reinterpret_cast<uint2*>(A.out.norms + row * (D / 4) + lg * 8) = make_uint2(nc[0], nc[1]);
            if (lg == 0) reinterpret_cast<uint32_t*>(A.out.params)[row] = prm;
        }
    }
}

// Streaming pass: grid-stride over warp tiles; blockIdx.y selects the tensor
// (K, V).  Vectors with a decision in doubt are left marked for
// encode_fixup_kernel, launched right after on the same stream.
template <int D>
__global__ void __launch_bounds__(kFastWarps * 32, kFastBlocksPerSM)
encode_fast_kernel(EncPair PA) {
    // the kernel launched after this one may start its own setup now; it
    // reads nothing this grid writes before this grid completes
    asm volatile("griddepcontrol.launch_dependents;");
    const EncArgs A = blockIdx.y ? PA.a[1] : PA.a[0];
    using Cfg = FastCfg<D>;
    __shared__ __align__(16) uint32_t masks[Cfg::NL][16];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int grp = lane / Cfg::NL, lg = lane % Cfg::NL;
    if (threadIdx.x < Cfg::NL) fast_sign_masks(A.signs, threadIdx.x, masks[threadIdx.x]);
    __syncthreads();
    const uint32_t b = (uint32_t)A.c.bits;
    const uint32_t pwk[4] = {1u, 1u << b, 1u << (2 * b), 1u << (3 * b)};
    const uint32_t n_tiles = (uint32_t)((A.n_vec + Cfg::VPW - 1) / Cfg::VPW);
    const uint32_t stride = gridDim.x * kFastWarps;
    for (uint32_t wt = blockIdx.x * kFastWarps + warp; wt < n_tiles; wt += stride)
        encode_tile_fast<D, false>(A, wt * Cfg::VPW + grp, masks[lg], lg, pwk, nullptr);
}

// Fixup pass: every lane reads the parameter of one vector; the marked ones
// are gathered, VPW at a time (one per group), and encoded again with their
// decisions in doubt re-taken exactly.
template <int D>
__global__ void __launch_bounds__(kFastWarps * 32, kFastBlocksPerSM)
encode_fixup_kernel(EncPair PA) {
    asm volatile("griddepcontrol.launch_dependents;");
    const EncArgs A = blockIdx.y ? PA.a[1] : PA.a[0];
    using Cfg = FastCfg<D>;
    __shared__ __align__(16) uint32_t masks[Cfg::NL][16];
    __shared__ uint32_t state[kFastWarps][kFsWords * 32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int grp = lane / Cfg::NL, lg = lane % Cfg::NL;
    if (threadIdx.x < Cfg::NL) fast_sign_masks(A.signs, threadIdx.x, masks[threadIdx.x]);
    __syncthreads();
    const uint32_t b = (uint32_t)A.c.bits;
    const uint32_t pwk[4] = {1u, 1u << b, 1u << (2 * b), 1u << (3 * b)};
    const bool lin8 = A.c.mode == KVQ_NORM_LIN8;
    const uint32_t n = (uint32_t)A.n_vec;
    const uint32_t n_chunks = (n + 31u) / 32u;
    const uint32_t stride = gridDim.x * kFastWarps;
    for (uint32_t ch = blockIdx.x * kFastWarps + warp; ch < n_chunks; ch += stride) {
        const uint32_t v = ch * 32u + (uint32_t)lane;
        bool marked = false;
        if (v < n) {
            const uint32_t vt = fast_div(v, A.tdiv);
            bool bad = false;
            const int64_t row =
                plane_row_bh(A.out, A.bh0 + vt, A.pos0 + (int64_t)(v - vt * (uint32_t)A.T), &bad);
            marked = lin8 ? reinterpret_cast<const uint16_t*>(A.out.params)[row] == kFixupMark16
                          : reinterpret_cast<const uint32_t*>(A.out.params)[row] == kFixupMark32;
        }
        uint32_t bal = __ballot_sync(KVQ_FULL_MASK, marked);
        while (bal) {
            // group g takes the (g+1)-th marked vector, if there is one
            const uint32_t pos = __fns(bal, 0, grp + 1);
            const uint32_t vg = pos < 32u ? ch * 32u + pos : n;  // n: no vector
            encode_tile_fast<D, true>(A, vg, masks[lg], lg, pwk, state[warp] + lane);
            for (int g = 0; g < Cfg::VPW && bal; g++) bal &= bal - 1u;
        }
    }
}

}  // namespace kvq
