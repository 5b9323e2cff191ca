// kvq_encode_impl.cuh - encoding of head vectors into packed angle and norm
// codes, one warp tile at a time; used by the encode kernel (kvq_encode.cu)
// and by the decode kernel when it appends the new token itself ("TurboAngle: Near-Lossless KV Cache Compression via Uniform
// Angle Quantization", Abstract: random diagonal, FWHT domain, consecutive
// pairs, uniform angles, 8-bit linear K norms / 4-bit log-space V norms).
//
// Layout of the work: one head vector per group of NL = d/EPL lanes, each
// lane holding EPL (<= 16) consecutive elements, loaded with 128-bit loads.
// The Walsh-Hadamard transform runs in registers (log2 EPL stages) and
// across the group with shuffles (log2 NL stages).
//
// Exactness.  Codes must equal the definition's exactly except within a hair
// of a decision edge.
//   - The transform runs in fp64, where it is exact: fp16 inputs are integer
//     multiples of 2^-24 below 2^16, so all partial sums over d <= 256 terms
//     fit in 53 bits.  The decisions then see z rounded once to fp32.
//   - The angle comes from an octant reduction and an odd polynomial for
//     atan on [0, 1] (kvq_atan_poly.h, fitted to 3.7e-8 rad); with the
//     approximate reciprocal, fp32 coefficients, Horner rounding and the
//     rounding of z its error stays far below the 1.5e-6 rad margin.
//   - sqrt, reciprocal and log2 use the hardware approximations
//     (sqrt/rcp/lg2.approx, documented to about 2^-22 relative or absolute),
//     budgeted at several times that.
// Any decision (angle bin, norm code, fp16 parameter) whose fp32 value lies
// within its error bound of the edge is re-taken out of line (exact_path):
// the exact rotated pair is summed in fp64 straight from the inputs and the
// decision follows the definition's own formulas in fp64.  What remains
// open is a value within an fp64 rounding of an edge.
#pragma once

#include "kvq_atan_poly.h"
#include "kvq_internal.h"

namespace kvq {

template <int D>
struct EncCfg {
    static constexpr int EPL = D < 16 ? D : 16;  // elements per lane
    static constexpr int NL = D / EPL;           // lanes per vector
    static constexpr int PPL = EPL / 2;          // pairs per lane
    static constexpr int VPW = 32 / NL;          // vectors per warp
    static constexpr int S = D == 4 ? 2 : D == 8 ? 3 : D == 16 ? 4 : D == 32 ? 5 : D == 64 ? 6
                           : D == 128 ? 7 : 8;   // log2 D
};

constexpr int kEncWarps = 8;
constexpr int kEncBlocksPerSM = 3;  // register budget: 24 resident warps per SM
constexpr int kEncStageWords = 128;  // max VPW * angle_words over all D, b <= 16
constexpr float kAngleSlack = 1.5e-6f;  // rad: polynomial, reciprocal, constants, rounding


// ------------------------------------------------------------ fp32 math --

__device__ __forceinline__ float rcp_approx(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float sqrt_approx(float x) {
    float y;
    asm("sqrt.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float lg2_approx(float x) {
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// atan2(y, x) for (x, y) != (0, 0): octant reduction to t in [0, 1] and the
// fitted odd polynomial.  Same conventions as atan2 on the axes.
__device__ __forceinline__ float atan2_poly(float y, float x) {
    const float ax = fabsf(x), ay = fabsf(y);
    const float mx = fmaxf(ax, ay), mn = fminf(ax, ay);
    const float t = mn * rcp_approx(mx);
    const float t2 = t * t;
    static_assert(KVQ_ATAN_NCOEF == 8, "Horner chain below has eight terms");
    float p = fmaf(KVQ_ATAN_C7, t2, KVQ_ATAN_C6);
    p = fmaf(p, t2, KVQ_ATAN_C5);
    p = fmaf(p, t2, KVQ_ATAN_C4);
    p = fmaf(p, t2, KVQ_ATAN_C3);
    p = fmaf(p, t2, KVQ_ATAN_C2);
    p = fmaf(p, t2, KVQ_ATAN_C1);
    p = fmaf(p, t2, KVQ_ATAN_C0);
    float th = p * t;
    th = ay > ax ? 1.5707963267948966f - th : th;
    th = x < 0.f ? kPiF - th : th;
    return y < 0.f ? -th : th;
}

// ------------------------------------------------ exact (fp64) decisions --

static __device__ __noinline__ int exact_angle_code(double u, double v, int L) {
    if (u == 0.0 && v == 0.0) return 0;
    const double theta = atan2(v, u);
    const double t = (theta + kPi) * (double)L / (2.0 * kPi);
    return (int)floor(t) % L;
}

static __device__ __noinline__ double exact_norm(double u, double v, double sqrt_d) {
    return hypot(u / sqrt_d, v / sqrt_d);
}

static __device__ __noinline__ double exact_log2(double r) { return log2(fmax(r, 5.9604644775390625e-8)); }

// log2 of r^2 with r floored at 2^-24 (so half of it is the definition's
// log2 max(r, 2^-24)).
static __device__ __noinline__ double exact_log2_sq(double r2) {
    return log2(fmax(r2, 3.552713678800501e-15));
}

__device__ __forceinline__ int lin8_code_exact(double r, double M) {
    if (M == 0.0) return 0;
    const double q = floor(255.0 * r / M + 0.5);
    return q > 255.0 ? 255 : (int)q;
}

__device__ __forceinline__ int log4_code_exact(double l, double LO, double HI) {
    if (HI == LO) return 0;
    const double q = floor(15.0 * (l - LO) / (HI - LO) + 0.5);
    return q < 0.0 ? 0 : (q > 15.0 ? 15 : (int)q);
}

// Exact rotated values (z[2p], z[2p+1]) of pair p of a group's vector, in
// fp64, straight from the lane's fp16 inputs: z_j = sum_k H[j][k] y_k with
// H[j][k] = (-1)^popcount(j & k).  Every input is a multiple of 2^-24 below
// 2^16, so every partial sum is exact in fp64.  j = 2p is even, so inputs
// 2w and 2w+1 of a lane share their sign, and z[2p+1] = E - O where E and O
// are the signed sums over even and odd inputs.  Every lane of the warp
// calls this (it sums across its group of NL lanes); each group passes its
// own p.
template <int EPL, int NL>
__device__ __forceinline__ void exact_pair_z(const uint32_t (&raw)[EPL / 2], int p, int lg,
                                             double& z0, double& z1) {
    constexpr int LOGE = EPL == 2 ? 1 : EPL == 4 ? 2 : EPL == 8 ? 3 : EPL == 16 ? 4 : 5;
    static_assert(EPL <= 32, "word signs below assume at most 16 words per lane");
    const unsigned j0 = 2u * (unsigned)p;
    const unsigned m = (j0 & (unsigned)(EPL - 1)) >> 1;
    // bit w of `row` = parity(m & w): the Sylvester row m over the lane's words
    const unsigned row = ((m & 1u) ? 0xAAAAu : 0u) ^ ((m & 2u) ? 0xCCCCu : 0u) ^
                         ((m & 4u) ? 0xF0F0u : 0u) ^ ((m & 8u) ? 0xFF00u : 0u);
    double E = 0.0, O = 0.0;
#pragma unroll
    for (int w = 0; w < EPL / 2; w++) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&raw[w]));
        const bool neg = (row >> w) & 1u;
        E += neg ? -(double)f.x : (double)f.x;
        O += neg ? -(double)f.y : (double)f.y;
    }
    if (__popc((j0 >> LOGE) & (unsigned)lg) & 1) {
        E = -E;
        O = -O;
    }
#pragma unroll
    for (int o = 1; o < NL; o <<= 1) {
        E += __shfl_xor_sync(KVQ_FULL_MASK, E, o);
        O += __shfl_xor_sync(KVQ_FULL_MASK, O, o);
    }
    z0 = E + O;
    z1 = E - O;
}

// Angle bin of an exactly known pair: the fp32 polynomial on the rounded
// values errs by far less than kAngleSlack, so outside that distance from an
// edge its bin is the definition's; inside it, libm atan2 in fp64.
__device__ __forceinline__ int angle_code_from_exact(double u, double v, int L,
                                                     float bins_per_rad) {
    if (u == 0.0 && v == 0.0) return 0;
    const float th = atan2_poly((float)v, (float)u);
    const float uu = fmaf(th, bins_per_rad, kPiF * bins_per_rad);
    const float fl = floorf(uu);
    const float fr = uu - fl;
    const float du = bins_per_rad * kAngleSlack + (float)L * 2.4e-7f;
    if (fr < du || fr > 1.f - du) return exact_angle_code(u, v, L);
    const int a = (int)fl;
    return a >= L ? a - L : (a < 0 ? a + L : a);
}

template <int N, typename T>
__device__ __forceinline__ T pick(const T (&a)[N], int i) {
    T v = a[0];
#pragma unroll
    for (int k = 1; k < N; k++) v = (k == i) ? a[k] : v;
    return v;
}

template <int N, typename T>
__device__ __forceinline__ void put(T (&a)[N], int i, T v) {
#pragma unroll
    for (int k = 0; k < N; k++)
        if (k == i) a[k] = v;
}

// ------------------------------------------------------ exact path ----

// State of one lane handed to the exact path.  The path is rare, so it lives
// out of line: its fp64 registers and code stay out of the streaming loop,
// and the arguments travel through the stack only when it runs.
template <int PPL>
struct ExactIn {
    uint32_t raw[PPL];  // the lane's fp16 elements, two per word, signs applied
    float rr[PPL];      // fp32 pair norms
    float ll[PPL];      // fp32 log2 of the pair norms (LOG4)
    int acode[PPL], ncode[PPL];
    uint32_t need_a, need_n, prm;
    float pmin, pmax, pband;
    int valid, need_p, unsure;
};

template <int PPL>
struct ExactOut {
    int acode[PPL], ncode[PPL];
    uint32_t prm;
};

// The transform recomputed in fp64 (exact for fp16 inputs) and the flagged
// decisions re-taken with the definition's own formulas.  Called by every
// lane of the warp (it shuffles across the group).
template <int D, class Cfg = EncCfg<D>>
__device__ __noinline__ ExactOut<Cfg::PPL> exact_fixup(ExactIn<Cfg::PPL> in, int lg, int L,
                                                      int mode) {
    constexpr int EPL = Cfg::EPL, NL = Cfg::NL, PPL = Cfg::PPL;
    ExactOut<PPL> o;
#pragma unroll
    for (int i = 0; i < PPL; i++) {
        o.acode[i] = in.acode[i];
        o.ncode[i] = in.ncode[i];
    }
    o.prm = in.prm;
    const double sqrt_d = sqrt((double)D);
    double zd[EPL];
#pragma unroll
    for (int w = 0; w < PPL; w++) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&in.raw[w]));
        zd[2 * w] = (double)f.x;
        zd[2 * w + 1] = (double)f.y;
    }
    fwht_local<EPL>(zd);
    fwht_cross<EPL, NL>(zd, lg);
    const bool gp = in.valid && in.need_p;  // uniform within the group
    uint32_t need_n = in.need_n;
#pragma unroll
    for (int i = 0; i < PPL; i++)
        if ((in.need_a >> i) & 1u) o.acode[i] = exact_angle_code(zd[2 * i], zd[2 * i + 1], L);
    // A parameter in doubt is decided by the pairs that can hold the exact
    // extreme: pair i can only if its fp32 value lies within the two error
    // bounds (its own and the fp32 extreme's) of the fp32 extreme.  Only
    // those pairs get exact norms here; when the exact parameter equals the
    // fp32 one, the fp32 codes stand except those already flagged, otherwise
    // (or when the bounds themselves are in doubt) every code of the group is
    // re-decided.
    double x64[PPL];  // exact r (LIN8) or log2 r (LOG4) where computed
    uint32_t have = 0;
    const bool lin8 = mode == KVQ_NORM_LIN8;
    if (__any_sync(KVQ_FULL_MASK, gp)) {
        double ext_hi = lin8 ? 0.0 : -1e300, ext_lo = 1e300;
#pragma unroll
        for (int i = 0; i < PPL; i++) {
            const float v32 = lin8 ? in.rr[i] : in.ll[i];
            const bool cand_hi = v32 >= in.pmax - in.pband;
            const bool cand_lo = !lin8 && v32 <= in.pmin + in.pband;
            if (gp && (in.unsure || cand_hi || cand_lo)) {
                const double r = exact_norm(zd[2 * i], zd[2 * i + 1], sqrt_d);
                x64[i] = lin8 ? r : exact_log2(r);
                have |= 1u << i;
                if (in.unsure || cand_hi) ext_hi = fmax(ext_hi, x64[i]);
                if (in.unsure || cand_lo) ext_lo = fmin(ext_lo, x64[i]);
            }
        }
        ext_hi = group_max_d<NL>(ext_hi);
        ext_lo = group_min_d<NL>(ext_lo);
        const uint32_t prm_x = lin8 ? (uint32_t)f64_to_f16_sat(ext_hi)
                                    : ((uint32_t)f64_to_f16_sat(ext_lo) |
                                       ((uint32_t)f64_to_f16_sat(ext_hi) << 16));
        const bool redo_all = gp && (in.unsure || prm_x != in.prm);
        if (gp) o.prm = prm_x;
        if (redo_all) need_n = (1u << PPL) - 1u;
    }
    if (need_n) {
#pragma unroll
        for (int i = 0; i < PPL; i++) {
            if (!((need_n >> i) & 1u)) continue;
            if (!((have >> i) & 1u)) {
                const double r = exact_norm(zd[2 * i], zd[2 * i + 1], sqrt_d);
                x64[i] = lin8 ? r : exact_log2(r);
            }
            if (lin8) {
                o.ncode[i] = lin8_code_exact(x64[i], (double)half_bits_to_float((uint16_t)o.prm));
            } else {
                o.ncode[i] = log4_code_exact(x64[i],
                                             (double)half_bits_to_float((uint16_t)(o.prm & 0xFFFF)),
                                             (double)half_bits_to_float((uint16_t)(o.prm >> 16)));
            }
        }
    }
    return o;
}

// Re-decide what the fp32 pass left in doubt.  Only the pairs in doubt get
// exact values (exact_pair_z), one pair per group per round: the group's
// lowest lane with work names its pair and the whole group sums it.  A
// parameter in doubt is decided by the pairs that can hold the exact extreme
// (fp32 value within the two error bounds of the fp32 extreme); flagged codes
// are re-decided against the fp32 parameter, which stands unless the exact
// extreme moves it.  When it moves (or the bounds themselves are in doubt)
// every code of the group changes, and exact_fixup redoes the whole vector.
// Out of line, so none of this costs the streaming pass registers; called by
// every lane of the warp.
// Cfg gives the lane layout (EPL elements per lane, NL lanes per vector).
template <int D, class Cfg = EncCfg<D>>
__device__ __noinline__ ExactOut<Cfg::PPL> exact_path(ExactIn<Cfg::PPL> in, int lg, int grp,
                                                     int L, int mode, float bins_per_rad) {
    constexpr int EPL = Cfg::EPL, NL = Cfg::NL, PPL = Cfg::PPL;
    ExactOut<PPL> o;
#pragma unroll
    for (int i = 0; i < PPL; i++) {
        o.acode[i] = in.acode[i];
        o.ncode[i] = in.ncode[i];
    }
    o.prm = in.prm;
    const bool lin8 = mode == KVQ_NORM_LIN8;
    const bool gp = in.valid && in.need_p;  // uniform within the group
    const int gshift = grp * NL;
    const unsigned gbits = NL >= 32 ? 0xffffffffu : ((1u << NL) - 1u);
    uint32_t cand = 0;
    if (gp) {
#pragma unroll
        for (int i = 0; i < PPL; i++) {
            const float v32 = lin8 ? in.rr[i] : in.ll[i];
            if (in.unsure || v32 >= in.pmax - in.pband || (!lin8 && v32 <= in.pmin + in.pband))
                cand |= 1u << i;
        }
    }
    const double M = (double)half_bits_to_float((uint16_t)(in.prm & 0xFFFF));
    const double HI = (double)half_bits_to_float((uint16_t)(in.prm >> 16));
    double ext_hi = lin8 ? 0.0 : -1e300, ext_lo = 1e300;
    uint32_t todo = in.valid ? (cand | in.need_a | in.need_n) : 0u;
    while (__any_sync(KVQ_FULL_MASK, todo != 0u)) {
        const unsigned gb = (__ballot_sync(KVQ_FULL_MASK, todo != 0u) >> gshift) & gbits;
        const int leader = gb ? __ffs(gb) - 1 : 0;
        const int i = __shfl_sync(KVQ_FULL_MASK, todo ? __ffs(todo) - 1 : 0, gshift + leader);
        double z0, z1;
        exact_pair_z<EPL, NL>(in.raw, leader * PPL + i, lg, z0, z1);
        if (gb && lg == leader) {
            const uint32_t bit = 1u << i;
            if (in.need_a & bit) put(o.acode, i, angle_code_from_exact(z0, z1, L, bins_per_rad));
            if ((cand | in.need_n) & bit) {
                // r^2 d = z0^2 + z1^2 (unscaled transform); r or log2 r from it
                const double r2 = fma(z0, z0, z1 * z1) * (1.0 / D);
                const double x = lin8 ? sqrt(r2) : 0.5 * exact_log2_sq(r2);
                if (cand & bit) {
                    const float v32 = lin8 ? pick(in.rr, i) : pick(in.ll, i);
                    if (in.unsure || v32 >= in.pmax - in.pband) ext_hi = fmax(ext_hi, x);
                    if (!lin8 && (in.unsure || v32 <= in.pmin + in.pband)) ext_lo = fmin(ext_lo, x);
                }
                if (in.need_n & bit)
                    put(o.ncode, i, lin8 ? lin8_code_exact(x, M) : log4_code_exact(x, M, HI));
            }
            todo &= ~bit;
        }
    }
    bool redo = false;
    if (__any_sync(KVQ_FULL_MASK, cand != 0u)) {
        ext_hi = group_max_d<NL>(ext_hi);
        ext_lo = group_min_d<NL>(ext_lo);
        if (gp) {
            o.prm = lin8 ? (uint32_t)f64_to_f16_sat(ext_hi)
                         : ((uint32_t)f64_to_f16_sat(ext_lo) | ((uint32_t)f64_to_f16_sat(ext_hi) << 16));
            redo = in.unsure || o.prm != in.prm;
        }
    }
    if (__any_sync(KVQ_FULL_MASK, redo)) return exact_fixup<D, Cfg>(in, lg, L, mode);
    return o;
}

// One launch encodes one tensor (blockIdx.y = 0) or K and V together
// (blockIdx.y selects the tensor).
struct EncPair {
    EncArgs a[2];
};

// One warp tile (VPW head vectors, NL lanes each): load, apply D, FWHT,
// decisions, pack, store.  Decisions in doubt are re-taken by exact_path
// (EXACT = true); with EXACT = false the tile is left untouched and reported
// instead (returns true).
template <int D, bool EXACT>
__device__ __forceinline__ bool encode_tile(const EncArgs& A, int64_t wt,
                                            const uint32_t (&smask)[EncCfg<D>::PPL], uint32_t* st,
                                            float du, int lane, int grp, int lg) {
    using Cfg = EncCfg<D>;
    constexpr int EPL = Cfg::EPL, NL = Cfg::NL, PPL = Cfg::PPL, VPW = Cfg::VPW;
    constexpr int NW = EPL / 2;  // packed pairs per lane (= PPL)
    const int L = A.c.L;
    const int bits = A.c.bits;
    const int AW = A.c.angle_words;
    const int64_t v = wt * VPW + grp;
    const bool valid = v < A.n_vec;

    // ---- load EPL fp16 values (128-bit loads), apply D -------------
    uint32_t raw[NW];
    {
        const __half* src = A.x + (valid ? v : 0) * D + lg * EPL;
        if constexpr (EPL == 16) {
            const uint4 q0 = reinterpret_cast<const uint4*>(src)[0];
            const uint4 q1 = reinterpret_cast<const uint4*>(src)[1];
            raw[0] = q0.x; raw[1] = q0.y; raw[2] = q0.z; raw[3] = q0.w;
            raw[4] = q1.x; raw[5] = q1.y; raw[6] = q1.z; raw[7] = q1.w;
        } else if constexpr (EPL == 8) {
            const uint4 q0 = reinterpret_cast<const uint4*>(src)[0];
            raw[0] = q0.x; raw[1] = q0.y; raw[2] = q0.z; raw[3] = q0.w;
        } else {
            const uint2 q0 = reinterpret_cast<const uint2*>(src)[0];
            raw[0] = q0.x; raw[1] = q0.y;
        }
#pragma unroll
        for (int w = 0; w < NW; w++) raw[w] = valid ? (raw[w] ^ smask[w]) : 0u;
    }

    // ---- fp32 (exact), L1 norm, FWHT ----------------------------------
    // ---- FWHT in fp64: exact for fp16 inputs ------------------------------
    // (every input is a multiple of 2^-24 below 2^16, so all partial sums
    // over d <= 256 terms fit in 53 bits); the decisions below then see z
    // with one fp32 rounding per component and nothing else
    double zd[EPL];
#pragma unroll
    for (int w = 0; w < NW; w++) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&raw[w]));
        zd[2 * w] = (double)f.x + (double)f.y;  // first stage inside the pair
        zd[2 * w + 1] = (double)f.x - (double)f.y;
    }
#pragma unroll
    for (int h = 2; h < EPL; h <<= 1) {
#pragma unroll
        for (int e = 0; e < EPL; e++) {
            if ((e & h) == 0) {
                const double a = zd[e], b = zd[e + h];
                zd[e] = a + b;
                zd[e + h] = a - b;
            }
        }
    }
#pragma unroll
    for (int m = 1; m < NL; m <<= 1) {  // cross-lane stages: v' = s * v + o
        const double sg = (lg & m) ? -1.0 : 1.0;
#pragma unroll
        for (int e = 0; e < EPL; e++) zd[e] = fma(sg, zd[e], __shfl_xor_sync(KVQ_FULL_MASK, zd[e], m));
    }
    f32x2 W[NW];  // W[k] = (z[2k], z[2k+1]), rounded once to fp32
#pragma unroll
    for (int k = 0; k < NW; k++) W[k] = pack2((float)zd[2 * k], (float)zd[2 * k + 1]);
    constexpr float ezr = 0.f;  // no transform error: z is exact before the rounding

    // ---- per pair: angle code and norm, with margins -------------------
    int acode[PPL];
    float rr[PPL];
    uint32_t need_a = 0, need_n = 0;
#pragma unroll
    for (int i = 0; i < PPL; i++) {
        const float x = lo2(W[i]), y = hi2(W[i]);
        const float rho = sqrt_approx(fmaf(x, x, y * y));
        // a nonzero exact z is at least 2^-24 in magnitude, so rho == 0
        // exactly when the pair is zero: code 0 by definition
        int a = 0;
        if (rho > 0.f) {
            const float th = atan2_poly(y, x);
            const float u = fmaf(th, A.bins_per_rad, kPiF * A.bins_per_rad);
            const float fl = floorf(u);
            const float fr = u - fl;
            if (fr < du || fr > 1.f - du) need_a |= 1u << i;
            a = (int)fl;
            a = a >= L ? a - L : (a < 0 ? a + L : a);
        }
        acode[i] = a;
        rr[i] = rho * A.inv_sqrt_d;
    }

    int ncode[PPL];
    uint32_t prm = 0;     // packed fp16 parameter(s)
    bool need_p = false;  // group-uniform
    // group-wide values the exact path reuses to find the pairs that can
    // decide a parameter
    float pmax = 0.f, pmin = 0.f, pband = 0.f;
    bool unsure = false;  // LOG4: some norm too small to trust its fp32 log2
    float ll[PPL];        // LOG4: fp32 log2 of each pair norm
    if (A.c.mode == KVQ_NORM_LIN8) {
#pragma unroll
        for (int i = 0; i < PPL; i++) ll[i] = 0.f;
        float m = 0.f;
#pragma unroll
        for (int i = 0; i < PPL; i++) m = fmaxf(m, rr[i]);
        m = group_max<NL>(m);
        const float eM = ezr + m * 1e-6f;
        need_p = near_f16_midpoint(m, eM);
        pmax = m;
        pband = 2.f * eM;
        const uint16_t Mh = f32_to_f16_sat(m);
        const float Mf = half_bits_to_float(Mh);
        prm = Mh;
        const float inv = Mf > 0.f ? 255.f * rcp_approx(Mf) : 0.f;
        const float dvc = ezr * inv * 1.01f + 2e-6f;
#pragma unroll
        for (int i = 0; i < PPL; i++) {
            const float vq = rr[i] * inv;
            const float t = vq + 0.5f;
            const float fl = floorf(t);
            const float fr = t - fl;
            const float dv = fmaf(vq, 1.2e-6f, dvc);
            if (Mf > 0.f && (fr < dv || fr > 1.f - dv)) need_n |= 1u << i;
            ncode[i] = Mf > 0.f ? min(255, (int)fl) : 0;
        }
    } else {
        float lmin = 1e30f, lmax = -1e30f, elmax = 0.f;
        float el[PPL];
#pragma unroll
        for (int i = 0; i < PPL; i++) {
            const float r = rr[i];
            const float er = fmaf(r, 1e-6f, ezr);
            unsure |= r < 2.3841858e-7f;  // r < 2^-22: leave tiny norms to fp64
            const float l = lg2_approx(fmaxf(r, 5.9604645e-8f));
            ll[i] = l;
            el[i] = er * rcp_approx(fmaxf(r, 1e-30f)) * 1.4717f + 1.2e-6f;
            lmin = fminf(lmin, l);
            lmax = fmaxf(lmax, l);
            elmax = fmaxf(elmax, el[i]);
        }
        lmin = group_min<NL>(lmin);
        lmax = group_max<NL>(lmax);
        elmax = group_max<NL>(elmax);
        unsure = group_any<NL>(unsure);
        need_p = unsure || near_f16_midpoint(lmin, elmax) || near_f16_midpoint(lmax, elmax);
        pmin = lmin;
        pmax = lmax;
        pband = 2.f * elmax;
        const uint16_t LOh = f32_to_f16_sat(lmin), HIh = f32_to_f16_sat(lmax);
        const float LOf = half_bits_to_float(LOh), HIf = half_bits_to_float(HIh);
        prm = (uint32_t)LOh | ((uint32_t)HIh << 16);
        const float inv = HIf != LOf ? 15.f * rcp_approx(HIf - LOf) : 0.f;
#pragma unroll
        for (int i = 0; i < PPL; i++) {
            const float vq = (ll[i] - LOf) * inv;
            const float t = vq + 0.5f;
            const float fl = floorf(t);
            const float fr = t - fl;
            const float dv = (el[i] + (fabsf(ll[i]) + fabsf(LOf)) * 1.2e-7f) * inv * 1.02f +
                             fabsf(vq) * 1e-6f + 2e-6f;
            if (HIf != LOf && (fr < dv || fr > 1.f - dv)) need_n |= 1u << i;
            ncode[i] = HIf != LOf ? min(15, max(0, (int)fl)) : 0;
        }
    }

    // ---- exact path: re-decide what was near an edge -------------------
    // Only the pairs in doubt get exact values (exact_pair_z), one pair per
    // group per round: the group's lowest lane with work names its pair and
    // the whole group sums it.  A parameter in doubt is decided by the pairs
    // that can hold the exact extreme (fp32 value within the two error
    // bounds of the fp32 extreme); when the exact parameter equals the fp32
    // one, the fp32 codes stand except those flagged.  When it does not (or
    // the bounds themselves are in doubt) the group's codes all change: the
    // whole transform is redone in fp64 out of line (rare).
    const bool lane_need = valid && ((need_a | need_n) != 0u || need_p);
    if constexpr (!EXACT) {
        // the streaming pass leaves the tile to encode_tile_exact
        if (__any_sync(KVQ_FULL_MASK, lane_need)) return true;
    } else {
        if (__any_sync(KVQ_FULL_MASK, lane_need)) {
            ExactIn<PPL> in;
    #pragma unroll
            for (int i = 0; i < PPL; i++) {
                in.raw[i] = raw[i];
                in.rr[i] = rr[i];
                in.ll[i] = ll[i];
                in.acode[i] = acode[i];
                in.ncode[i] = ncode[i];
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
            const ExactOut<PPL> o = exact_path<D>(in, lg, grp, L, A.c.mode, A.bins_per_rad);
    #pragma unroll
            for (int i = 0; i < PPL; i++) {
                acode[i] = o.acode[i];
                ncode[i] = o.ncode[i];
            }
            prm = o.prm;
        }
    }

    // ---- pack and store ------------------------------------------------
    int64_t row = 0;
    if (valid) {
        const int64_t vt = A.small ? (int64_t)fast_div((uint32_t)v, A.tdiv) : v / A.T;
        bool bad = false;
        row = plane_row_bh(A.out, A.bh0 + vt, A.pos0 + (v - vt * A.T), &bad);
        if (bad && lg == 0) report(A.err_word, KVQ_DEVERR_PAGE_RANGE);
    }
    // angle bit stream: this lane's PPL codes occupy bits [cb, cb + PPL*bits)
    {
        uint64_t lo = 0, hi = 0;
#pragma unroll
        for (int k = 0; k < PPL; k++) {
            const int pos = k * bits;
            const uint64_t a = (uint64_t)(uint32_t)acode[k];
            if (pos < 64) {
                lo |= a << pos;
                if (pos + bits > 64) hi |= a >> (64 - pos);
            } else {
                hi |= a << (pos - 64);
            }
        }
        const int cb = lg * PPL * bits;
        const int w0 = cb >> 5, sh = cb & 31;
        uint32_t w[5];
        {
            const uint64_t l2 = sh ? (lo << sh) : lo;
            const uint64_t h2 = sh ? ((hi << sh) | (lo >> (64 - sh))) : hi;
            const uint32_t top = sh ? (uint32_t)(hi >> (64 - sh)) : 0u;
            w[0] = (uint32_t)l2;
            w[1] = (uint32_t)(l2 >> 32);
            w[2] = (uint32_t)h2;
            w[3] = (uint32_t)(h2 >> 32);
            w[4] = top;
        }
        if (valid) {
#pragma unroll
            for (int j = 0; j < 5; j++)
                if (w[j] != 0u && w0 + j < AW) atomicOr(&st[grp * AW + w0 + j], w[j]);
        }
        __syncwarp();
        if (valid) {
            uint32_t* dst = reinterpret_cast<uint32_t*>(A.out.angles) + row * AW;
            for (int j = lg; j < AW; j += NL) {
                dst[j] = st[grp * AW + j];
                st[grp * AW + j] = 0u;
            }
        }
        __syncwarp();
    }
    if (valid) {
        if (A.c.mode == KVQ_NORM_LIN8) {
            uint8_t* dst = A.out.norms + row * (D / 2) + lg * PPL;
            if constexpr (PPL == 8) {
                uint2 q;
                q.x = (uint32_t)ncode[0] | (uint32_t)ncode[1] << 8 | (uint32_t)ncode[2] << 16 |
                      (uint32_t)ncode[3] << 24;
                q.y = (uint32_t)ncode[4] | (uint32_t)ncode[5] << 8 | (uint32_t)ncode[6] << 16 |
                      (uint32_t)ncode[7] << 24;
                *reinterpret_cast<uint2*>(dst) = q;
            } else if constexpr (PPL == 4) {
                *reinterpret_cast<uint32_t*>(dst) = (uint32_t)ncode[0] | (uint32_t)ncode[1] << 8 |
                                                    (uint32_t)ncode[2] << 16 |
                                                    (uint32_t)ncode[3] << 24;
            } else {
                *reinterpret_cast<uint16_t*>(dst) = (uint16_t)(ncode[0] | ncode[1] << 8);
            }
            if (lg == 0) reinterpret_cast<uint16_t*>(A.out.params)[row] = (uint16_t)prm;
        } else {
            uint8_t* dst = A.out.norms + row * (D / 4) + lg * (PPL / 2);
            uint32_t packed = 0;
#pragma unroll
            for (int i = 0; i < PPL; i++) packed |= (uint32_t)ncode[i] << (4 * i);
            if constexpr (PPL == 8) {
                *reinterpret_cast<uint32_t*>(dst) = packed;
            } else if constexpr (PPL == 4) {
                *reinterpret_cast<uint16_t*>(dst) = (uint16_t)packed;
            } else {
                *dst = (uint8_t)packed;
            }
            if (lg == 0) reinterpret_cast<uint32_t*>(A.out.params)[row] = prm;
        }
    }
    return false;
}

template <int D>
__device__ __forceinline__ void lane_sign_masks(const int8_t* signs, int lg,
                                                uint32_t (&smask)[EncCfg<D>::PPL]) {
    // fp16 sign-bit masks of this lane's elements (element pairs per word)
#pragma unroll
    for (int w = 0; w < EncCfg<D>::PPL; w++) {
        const int e = lg * EncCfg<D>::EPL + 2 * w;
        smask[w] = (signs[e] < 0 ? 0x8000u : 0u) | (signs[e + 1] < 0 ? 0x80000000u : 0u);
    }
}

// angle margin in bin units: polynomial, reciprocal, constants and the fp32
// rounding of z (kAngleSlack), plus the rounding of u near L
__device__ __forceinline__ float angle_margin(const EncArgs& A) {
    return A.bins_per_rad * kAngleSlack + (float)A.c.L * 2.4e-7f;
}

}  // namespace kvq
