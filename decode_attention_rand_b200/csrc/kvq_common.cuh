// kvq_common.cuh - device helpers shared by the kvq kernels (sm_100a).
//
// Codec of "TurboAngle: Near-Lossless KV Cache Compression via Uniform Angle
// Quantization" (Abstract): +-1 diagonal, Walsh-Hadamard transform scaled by
// 1/sqrt(d), consecutive pairs as (norm, uniformly quantized angle).  The
// exact formulas and the byte layout are the ones stated in include/kvq.h.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "kvq.h"  // include/ is on the include path

#define KVQ_FULL_MASK 0xffffffffu

namespace kvq {

constexpr float kPiF = 3.14159265358979323846f;
constexpr double kPi = 3.14159265358979323846264338327950288;

// ---------------------------------------------------------------- codec --

struct CodecDev {
    int d;          // head dim
    int L;          // codebook size
    int bits;       // bits per angle code
    int mode;       // KVQ_NORM_LIN8 / KVQ_NORM_LOG4
    int angle_words;  // 32-bit words per token row
    int norm_bytes;   // bytes per token row
    int param_bytes;  // 2 (LIN8) or 4 (LOG4)
};

// Division of a 32-bit unsigned dividend by a divisor fixed per launch:
// multiply-high and shifts (Granlund and Montgomery, "Division by Invariant
// Integers using Multiplication", PLDI 1994, section 4), exact for every
// dividend below 2^32 and divisor 1 <= d < 2^32.
struct FastDiv {
    uint32_t m;   // 2^32 (2^l - d) / d + 1, l = ceil(log2 d)
    uint32_t s1;  // min(l, 1)
    uint32_t s2;  // max(l - 1, 0)
};

inline FastDiv make_fast_div(uint32_t d) {
    if (d == 0) d = 1;
    uint32_t l = 0;
    while (l < 32 && (1ull << l) < (unsigned long long)d) l++;
    FastDiv f;
    f.m = (uint32_t)((((1ull << l) - d) << 32) / d + 1);
    f.s1 = l < 1 ? l : 1;
    f.s2 = l > 1 ? l - 1 : 0;
    return f;
}

__device__ __forceinline__ uint32_t fast_div(uint32_t n, const FastDiv& f) {
    const uint32_t t = __umulhi(f.m, n);
    return (t + ((n - t) >> f.s1)) >> f.s2;
}

struct PlaneDev {
    uint8_t* angles;
    uint8_t* norms;
    uint8_t* params;
    int64_t capacity;      // tokens per sequence (max_pages * page_tokens when paged)
    int H_kv;              // KV heads of the call
    const int32_t* pages;  // NULL: contiguous [B][H_kv][capacity]; else [B][max_pages]
    int page_tokens;
    int max_pages;
    int64_t num_pages;
    FastDiv hdiv;          // division by H_kv (paged row lookup by sequence index)
};

// Row of token t of sequence (b, h) in each array of a plane.  A page-table
// entry outside the pool is replaced by page 0 and flagged in *bad.
__device__ __forceinline__ int64_t plane_row(const PlaneDev& p, int64_t b, int h, int64_t t,
                                             bool* bad) {
    if (!p.pages) return (b * p.H_kv + h) * p.capacity + t;
    int64_t pg = p.pages[b * p.max_pages + t / p.page_tokens];
    if (pg < 0 || pg >= p.num_pages) {
        *bad = true;
        pg = 0;
    }
    return (pg * p.H_kv + h) * p.page_tokens + t % p.page_tokens;
}

// Row of token t of sequence bh = b * H_kv + h (B * H_kv < 2^32 when paged).
__device__ __forceinline__ int64_t plane_row_bh(const PlaneDev& p, int64_t bh, int64_t t,
                                                bool* bad) {
    if (!p.pages) return bh * p.capacity + t;
    const uint32_t b = fast_div((uint32_t)bh, p.hdiv);
    return plane_row(p, b, (int)((uint32_t)bh - b * (uint32_t)p.H_kv), t, bad);
}

// --------------------------------------------------------------- warps --

template <int WIDTH>
__device__ __forceinline__ float group_sum(float v) {
#pragma unroll
    for (int o = WIDTH / 2; o > 0; o >>= 1) v += __shfl_xor_sync(KVQ_FULL_MASK, v, o);
    return v;
}

template <int WIDTH>
__device__ __forceinline__ float group_max(float v) {
#pragma unroll
    for (int o = WIDTH / 2; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(KVQ_FULL_MASK, v, o));
    return v;
}

template <int WIDTH>
__device__ __forceinline__ float group_min(float v) {
#pragma unroll
    for (int o = WIDTH / 2; o > 0; o >>= 1) v = fminf(v, __shfl_xor_sync(KVQ_FULL_MASK, v, o));
    return v;
}

template <int WIDTH>
__device__ __forceinline__ double group_max_d(double v) {
#pragma unroll
    for (int o = WIDTH / 2; o > 0; o >>= 1) v = fmax(v, __shfl_xor_sync(KVQ_FULL_MASK, v, o));
    return v;
}

template <int WIDTH>
__device__ __forceinline__ double group_min_d(double v) {
#pragma unroll
    for (int o = WIDTH / 2; o > 0; o >>= 1) v = fmin(v, __shfl_xor_sync(KVQ_FULL_MASK, v, o));
    return v;
}

template <int WIDTH>
__device__ __forceinline__ bool group_any(bool p) {
    unsigned b = __ballot_sync(KVQ_FULL_MASK, p);
    if (WIDTH == 32) return b != 0u;
    const int lane = threadIdx.x & 31;
    const unsigned gmask = ((1u << WIDTH) - 1u) << (lane & ~(WIDTH - 1));
    return (b & gmask) != 0u;
}

// ------------------------------------------------------------ FWHT -------
// In-register Sylvester-ordered Walsh-Hadamard butterflies over the EPL
// elements a lane holds, followed by the cross-lane stages over NL lanes.
// Element g of the vector lives in lane g / EPL (within its group), slot
// g % EPL, so stage p pairs g with g ^ (1 << p): out[g] = v[g] + v[g'] for the
// lower index and v[g] - v[g'] for the upper one (natural-order transform).

template <int EPL, typename T>
__device__ __forceinline__ void fwht_local(T (&v)[EPL]) {
#pragma unroll
    for (int h = 1; h < EPL; h <<= 1) {
#pragma unroll
        for (int e = 0; e < EPL; e++) {
            if ((e & h) == 0) {
                T a = v[e], b = v[e + h];
                v[e] = a + b;
                v[e + h] = a - b;
            }
        }
    }
}

template <int EPL, int NL, typename T>
__device__ __forceinline__ void fwht_cross(T (&v)[EPL], int lane_g) {
#pragma unroll
    for (int m = 1; m < NL; m <<= 1) {
        const bool upper = (lane_g & m) != 0;
#pragma unroll
        for (int e = 0; e < EPL; e++) {
            T o = __shfl_xor_sync(KVQ_FULL_MASK, v[e], m);
            v[e] = upper ? (o - v[e]) : (v[e] + o);
        }
    }
}

// -------------------------------------------------------------- fp16 ----

__device__ __forceinline__ float half_bits_to_float(uint16_t h) {
    return __half2float(__ushort_as_half(h));
}

// The codec's fp16 parameter rule: round to nearest even, saturate to the
// largest finite fp16, store a zero as +0.
__device__ __forceinline__ uint16_t f16_param_bits(uint16_t h) {
    if ((h & 0x7FFF) >= 0x7C00) h = (uint16_t)((h & 0x8000) | 0x7BFF);
    return h == 0x8000 ? (uint16_t)0 : h;
}

__device__ __forceinline__ uint16_t f32_to_f16_sat(float x) {
    return f16_param_bits(__half_as_ushort(__float2half_rn(x)));
}

__device__ __forceinline__ uint16_t f64_to_f16_sat(double x) {
    return f16_param_bits(__half_as_ushort(__double2half(x)));
}

// True when |x| lies within tol of a midpoint between two adjacent finite
// fp16 values, i.e. where the fp16 rounding of the exact value could differ
// from the rounding of x.  Midpoints of fp16 values are exact in fp32.
__device__ __forceinline__ bool near_f16_midpoint(float x, float tol) {
    const float a = fabsf(x);
    uint16_t h = __half_as_ushort(__float2half_rn(a));
    if (h >= 0x7C00) h = 0x7BFF;
    const float hv = half_bits_to_float(h);
    bool near = false;
    if (h < 0x7BFF) near |= fabsf(a - 0.5f * (hv + half_bits_to_float((uint16_t)(h + 1)))) <= tol;
    if (h > 0) near |= fabsf(a - 0.5f * (hv + half_bits_to_float((uint16_t)(h - 1)))) <= tol;
    return near;
}

// ------------------------------------------------------ packed fp32 ----
// Two fp32 lanes in a 64-bit register pair for the f32x2 instructions.
typedef unsigned long long f32x2;  // two packed fp32 lanes

__device__ __forceinline__ f32x2 pack2(float lo, float hi) {
    f32x2 v;
    asm("mov.b64 %0, {%1, %2};" : "=l"(v) : "f"(lo), "f"(hi));
    return v;
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

__device__ __forceinline__ f32x2 add2(f32x2 a, f32x2 b) {
    f32x2 d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ f32x2 sub2(f32x2 a, f32x2 b) {
    f32x2 d;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

// Walsh-Hadamard butterflies over every index bit but bit 0, for 32 elements
// per lane held as 16 packed pairs (w[2k], w[2k+1]) in P[k]: local stages on
// pair strides 1, 2, 4, 8, then the NL lanes of the group.
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

// ------------------------------------------- lane slices <-> runs ----
// A vector of d = 32 NL elements held 32 per lane (lane l of its group: the
// slice l 32 .. l 32 + 31, as 16 packed pairs) is transposed through shared
// memory so that lane l holds, for every slice Lh, the run of RL = 32 / NL
// elements starting at Lh 32 + l RL (P[Lh RL/2 .. Lh RL/2 + RL/2 - 1]).  The
// butterfly stages over the slice index then run in registers (fwht_runs)
// instead of through shuffles.  Lane (g, l) writes its 16-byte chunk q to
// slot q ^ f(g, l) of its 8-chunk block, f(g, l) = l K + (g mod K) with
// K = 8 / NL; a quarter warp (K vectors of NL lanes) then covers all eight
// bank groups on the writes and on the reads (chunk l K + h of the block of
// lane Lh sits in slot (l ^ Lh) K + (h ^ (g mod K))), and on a 128-byte
// aligned block both addresses are a per-lane base XOR a constant.  Chunks
// move as single 128-bit accesses: two 64-bit ones would each be served per
// half warp, where the slot pattern does not keep the banks apart.  The
// "memory" clobbers keep them on their side of the __syncwarp()s.
__device__ __forceinline__ void xch_store(uint32_t addr, f32x2 a, f32x2 b) {
    asm volatile("st.shared.v2.b64 [%0], {%1, %2};" ::"r"(addr), "l"(a), "l"(b) : "memory");
}
__device__ __forceinline__ void xch_load(uint32_t addr, f32x2& a, f32x2& b) {
    asm volatile("ld.shared.v2.b64 {%0, %1}, [%2];" : "=l"(a), "=l"(b) : "r"(addr) : "memory");
}

template <int NL>
struct LaneRuns {
    static constexpr int RL = 32 / NL;              // elements per run
    static constexpr int K = 8 / NL;                // chunks a lane reads from each block
    static constexpr int WARP_BYTES = 32 * 8 * 16;  // exchange bytes of one warp
    uint32_t xw, xr;  // chunk q: xw ^ (q << 4); run Lh, chunk h: (xr ^ ((Lh K + h) << 4)) + Lh 128
    // warp_base: shared-window address of the warp's WARP_BYTES, 128-byte aligned
    __device__ __forceinline__ LaneRuns(uint32_t warp_base, int grp, int lg) {
        const uint32_t row = warp_base + (uint32_t)grp * (NL * 128);
        const uint32_t sw = (uint32_t)(lg * K + grp % K) << 4;
        xw = row + (uint32_t)lg * 128 + sw;
        xr = row | sw;
    }
    // slices -> runs (the whole warp takes part)
    __device__ __forceinline__ void to_runs(f32x2 (&P)[16]) const {
        __syncwarp();  // earlier readers of the buffer are done
#pragma unroll
        for (int q = 0; q < 8; q++) xch_store(xw ^ (q << 4), P[2 * q], P[2 * q + 1]);
        __syncwarp();
#pragma unroll
        for (int Lh = 0; Lh < NL; Lh++)
#pragma unroll
            for (int h = 0; h < K; h++)
                xch_load((xr ^ ((Lh * K + h) << 4)) + Lh * 128, P[Lh * (RL / 2) + 2 * h],
                         P[Lh * (RL / 2) + 2 * h + 1]);
    }
    // runs -> slices
    __device__ __forceinline__ void from_runs(f32x2 (&P)[16]) const {
        __syncwarp();
#pragma unroll
        for (int Lh = 0; Lh < NL; Lh++)
#pragma unroll
            for (int h = 0; h < K; h++)
                xch_store((xr ^ ((Lh * K + h) << 4)) + Lh * 128, P[Lh * (RL / 2) + 2 * h],
                          P[Lh * (RL / 2) + 2 * h + 1]);
        __syncwarp();
#pragma unroll
        for (int q = 0; q < 8; q++) xch_load(xw ^ (q << 4), P[2 * q], P[2 * q + 1]);
    }
};

// Butterflies over the slice index of a vector held as runs (LaneRuns):
// the stages fwht_pairs<NL> runs across lanes, here in registers.
template <int NL>
__device__ __forceinline__ void fwht_runs(f32x2 (&P)[16]) {
    constexpr int H = 16 / NL;  // pairs per run
#pragma unroll
    for (int st = 1; st < NL; st <<= 1) {
#pragma unroll
        for (int Lh = 0; Lh < NL; Lh++) {
            if ((Lh & st) == 0) {
#pragma unroll
                for (int u = 0; u < H; u++) {
                    const f32x2 a = P[Lh * H + u], b = P[(Lh + st) * H + u];
                    P[Lh * H + u] = add2(a, b);
                    P[(Lh + st) * H + u] = sub2(a, b);
                }
            }
        }
    }
}

// ------------------------------------------------------ device errors ----

__device__ __forceinline__ void report(int32_t* err_word, int bits) {
    if (err_word) atomicOr(err_word, bits);
}

}  // namespace kvq
