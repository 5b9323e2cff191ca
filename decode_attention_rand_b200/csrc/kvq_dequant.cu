// kvq_dequant.cu - dequant kernel: packed codes -> fp16 head vectors.
//
// Reconstruction of "TurboAngle: Near-Lossless KV Cache Compression via
// Uniform Angle Quantization" (Abstract): each pair becomes
// r^ (cos theta^, sin theta^) with theta^ the centre of its angle bin, and the
// vector returns to the original domain through the inverse rotation
// D H / sqrt(d) (H symmetric, H H = d I).  r^ = c M / 255 (8-bit linear) or
// 2^(LO + c (HI - LO) / 15) (4-bit log space).
//
// Two kernels.  The fast one (d = 64, 128, 256 and L <= 256) keeps 32
// elements per lane, looks the bin centres up in a static shared-memory
// table and runs the butterfly stages over the lane index bits in registers
// after one exchange through shared memory (see dequant_fast_kernel).  The
// general one (any d and L) mirrors the encode kernel: one vector per group
// of NL lanes, EPL elements per lane, FWHT in registers plus shuffles,
// 128-bit stores; cos/sin of the L bin centres come from a shared-memory
// table (L <= 4096) or from sincospif for larger codebooks.
#include "kvq_internal.h"

namespace kvq {

template <int D>
struct DqCfg {
    static constexpr int EPL = D < 16 ? D : 16;
    static constexpr int NL = D / EPL;
    static constexpr int PPL = EPL / 2;
    static constexpr int VPW = 32 / NL;
};

constexpr int kDqWarps = 8;
constexpr int kDqTableMax = 4096;

struct DqArgs {
    PlaneDev in;
    const int8_t* signs;
    int64_t n_vec, T, pos0;
    CodecDev c;
    __half* y;
    float inv_sqrt_d;
    FastDiv tdiv;  // division by T (fast kernel: n_vec <= 2^31)
};

// Bits [0, 128) of a lane's code chunk that starts at bit `cb` of a row of
// `aw` words, as (lo, hi).
__device__ __forceinline__ void load_chunk(const uint32_t* row, int aw, int cb, uint64_t& lo,
                                           uint64_t& hi) {
    const int w0 = cb >> 5, sh = cb & 31;
    uint32_t w[5];
#pragma unroll
    for (int j = 0; j < 5; j++) w[j] = (w0 + j < aw) ? row[w0 + j] : 0u;
    const uint64_t a = (uint64_t)w[0] | (uint64_t)w[1] << 32;
    const uint64_t b = (uint64_t)w[2] | (uint64_t)w[3] << 32;
    const uint64_t c = (uint64_t)w[4];
    lo = sh ? ((a >> sh) | (b << (64 - sh))) : a;
    hi = sh ? ((b >> sh) | (c << (64 - sh))) : b;
}

__device__ __forceinline__ uint32_t chunk_code(uint64_t lo, uint64_t hi, int pos, int bits) {
    const uint64_t mask = (1ull << bits) - 1ull;
    uint64_t v;
    if (pos < 64) {
        v = lo >> pos;
        if (pos + bits > 64) v |= hi << (64 - pos);
    } else {
        v = hi >> (pos - 64);
    }
    return (uint32_t)(v & mask);
}

template <int D>
__global__ void __launch_bounds__(kDqWarps * 32)
dequant_kernel(DqArgs A) {
    using Cfg = DqCfg<D>;
    constexpr int EPL = Cfg::EPL, NL = Cfg::NL, PPL = Cfg::PPL, VPW = Cfg::VPW;
    __shared__ float2 cs_table[kDqTableMax];

    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int grp = lane / NL;
    const int lg = lane % NL;
    const int L = A.c.L;
    const int bits = A.c.bits;
    const int AW = A.c.angle_words;
    const bool use_table = L <= kDqTableMax;

    if (use_table) {
        for (int j = threadIdx.x; j < L; j += blockDim.x) {
            float s, c;
            sincospif((float)(2 * j + 1) / (float)L - 1.f, &s, &c);
            cs_table[j] = make_float2(c, s);
        }
    }
    __syncthreads();

    uint32_t negmask = 0;
#pragma unroll
    for (int e = 0; e < EPL; e++) negmask |= (A.signs[lg * EPL + e] < 0 ? 1u : 0u) << e;

    const int64_t n_warps_total = (int64_t)gridDim.x * kDqWarps;
    const int64_t n_warp_tiles = (A.n_vec + VPW - 1) / VPW;
    for (int64_t wt = (int64_t)blockIdx.x * kDqWarps + warp; wt < n_warp_tiles; wt += n_warps_total) {
        const int64_t v = wt * VPW + grp;
        const bool valid = v < A.n_vec;
        int64_t row = 0;
        if (valid) {
            const int64_t bh = v / A.T;
            row = bh * A.in.capacity + A.pos0 + (v - bh * A.T);
        }
        float z[EPL];
        if (valid) {
            uint64_t lo, hi;
            load_chunk(reinterpret_cast<const uint32_t*>(A.in.angles) + row * AW, AW,
                       lg * PPL * bits, lo, hi);
            int nc[PPL];
            float p0, p1;
            if (A.c.mode == KVQ_NORM_LIN8) {
                const uint8_t* src = A.in.norms + row * (D / 2) + lg * PPL;
#pragma unroll
                for (int i = 0; i < PPL; i++) nc[i] = src[i];
                p0 = half_bits_to_float(reinterpret_cast<const uint16_t*>(A.in.params)[row]) *
                     (1.f / 255.f);
                p1 = 0.f;
            } else {
                const uint8_t* src = A.in.norms + row * (D / 4) + lg * (PPL / 2);
#pragma unroll
                for (int i = 0; i < PPL; i++) nc[i] = (src[i / 2] >> (4 * (i & 1))) & 0xF;
                const uint32_t pr = reinterpret_cast<const uint32_t*>(A.in.params)[row];
                const float LO = half_bits_to_float((uint16_t)(pr & 0xFFFF));
                const float HI = half_bits_to_float((uint16_t)(pr >> 16));
                p0 = LO;
                p1 = (HI - LO) * (1.f / 15.f);
            }
#pragma unroll
            for (int i = 0; i < PPL; i++) {
                const int a = (int)chunk_code(lo, hi, i * bits, bits);
                const float r = A.c.mode == KVQ_NORM_LIN8 ? (float)nc[i] * p0
                                                           : exp2f(fmaf((float)nc[i], p1, p0));
                float c, s;
                if (use_table) {
                    const float2 t = cs_table[a];
                    c = t.x;
                    s = t.y;
                } else {
                    sincospif((float)(2 * a + 1) * (1.f / (float)L) - 1.f, &s, &c);
                }
                z[2 * i] = r * c;
                z[2 * i + 1] = r * s;
            }
        } else {
#pragma unroll
            for (int e = 0; e < EPL; e++) z[e] = 0.f;
        }
        fwht_local<EPL>(z);
        fwht_cross<EPL, NL>(z, lg);
        if (valid) {
            uint32_t packed[EPL / 2];
#pragma unroll
            for (int e = 0; e < EPL; e += 2) {
                float a0 = z[e] * A.inv_sqrt_d, a1 = z[e + 1] * A.inv_sqrt_d;
                a0 = ((negmask >> e) & 1u) ? -a0 : a0;
                a1 = ((negmask >> (e + 1)) & 1u) ? -a1 : a1;
                const __half2 h = __floats2half2_rn(a0, a1);
                packed[e / 2] = *reinterpret_cast<const uint32_t*>(&h);
            }
            __half* dst = A.y + v * D + lg * EPL;
            if constexpr (EPL == 16) {
                reinterpret_cast<uint4*>(dst)[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
                reinterpret_cast<uint4*>(dst)[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
            } else if constexpr (EPL == 8) {
                reinterpret_cast<uint4*>(dst)[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
            } else {
                reinterpret_cast<uint2*>(dst)[0] = make_uint2(packed[0], packed[1]);
            }
        }
    }
}

// ------------------------------------------------------------ fast path --
// d = 64, 128, 256 and L <= 256 (codes of B <= 8 bits, B a template
// parameter): 32 elements per lane, d/32 lanes per vector.  The butterfly
// inside each element pair is applied to the table instead of the data:
// (z[2i], z[2i+1]) = r (cos, sin) becomes r (cos + sin, cos - sin), the
// remaining index bits go through the packed fp32 transform, 1/sqrt(d) rides
// on r and the signs of D on the fp16 sign bits.

template <int D>
struct DqFastCfg {
    static constexpr int NL = D / 32;    // lanes per vector
    static constexpr int VPW = 32 / NL;  // vectors per warp tile
    static constexpr int S = D == 64 ? 6 : D == 128 ? 7 : 8;
};

constexpr int kDqFastBlocksPerSM = 3;  // registers for one tile ahead in flight

// The butterfly stages over the lane index bits run in registers after a
// transposition of each vector through shared memory (LaneRuns): lane l then
// holds, for every former lane index Lh, the run of RL = 32 / NL elements
// starting at Lh 32 + l RL, and stores it as 16-byte (8-byte for d = 256)
// words.

template <int D, int B>
__global__ void __launch_bounds__(kDqWarps * 32, kDqFastBlocksPerSM)
dequant_fast_kernel(DqArgs A) {
    // Launched as a programmatic dependent of the previous kernel on the
    // stream: the next kernel may start its own setup now, and this one builds
    // its table (from its arguments alone) while the previous one drains; no
    // global memory is read or written before griddepcontrol.wait.
    asm volatile("griddepcontrol.launch_dependents;");
    using Cfg = DqFastCfg<D>;
    constexpr int NL = Cfg::NL, VPW = Cfg::VPW, S = Cfg::S;
    // r-free (cos + sin, cos - sin) of each bin centre, 16 copies side by side
    // ([code][16]): lane l of a half warp reads copy l, so a lookup never
    // shares a bank within the half warp.  A static array: its base is a
    // compile-time address that the lookups carry in the load's immediate.
    __shared__ __align__(128) float2 tab[16 << B];
    extern __shared__ __align__(16) unsigned char xdyn[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int grp = lane / NL, lg = lane % NL;
    // 2^B entries, so that any B-bit pattern indexes inside the table (codes
    // of a valid cache are below L)
    const int L = A.c.L;
    for (int j = threadIdx.x; j < (1 << B); j += blockDim.x) {
        float sn, cs;
        sincospif((float)(2 * j + 1) / (float)L - 1.f, &sn, &cs);
        tab[j * 16] = make_float2(cs + sn, cs - sn);
    }
    __syncthreads();
    for (int i = threadIdx.x; i < (16 << B); i += blockDim.x)
        if (i & 15) tab[i] = tab[i & ~15];
    asm volatile("griddepcontrol.wait;" ::: "memory");
    uint32_t m[16];  // fp16 sign bits of D for this lane's output element pairs
#pragma unroll
    for (int w = 0; w < 16; w++) {
        // pair w is pair w % (RL / 2) of run w / (RL / 2)
        constexpr int RL = LaneRuns<NL>::RL;
        const int e = (w / (RL / 2)) * 32 + lg * RL + 2 * (w % (RL / 2));
        m[w] = (A.signs[e] < 0 ? 0x8000u : 0u) | (A.signs[e + 1] < 0 ? 0x80000000u : 0u);
    }
    // exchange buffer, 128-byte aligned: [warp][vector][lane][8 chunks]
    using T = LaneRuns<NL>;
    const T runs((((uint32_t)__cvta_generic_to_shared(xdyn) + 127u) & ~127u) +
                     (uint32_t)(warp * T::WARP_BYTES),
                 grp, lg);
    __syncthreads();
    // byte offset of the lane's replica (code c's entries span 128 bytes)
    const uint32_t tlo = (uint32_t)(lane & 15) * sizeof(float2);
    const int AW = A.c.angle_words;
    const bool lin8 = A.c.mode == KVQ_NORM_LIN8;
    const float isd = A.inv_sqrt_d;
    // this lane's 16 codes start at bit 16 B lg of the row
    const int wbase = (lg * 16 * B) >> 5, sh = (lg * 16 * B) & 31;
    const uint32_t n_tiles = (uint32_t)((A.n_vec + VPW - 1) / VPW);
    const uint32_t stride = gridDim.x * kDqWarps;
    // The code rows of a warp tile are loaded one iteration ahead: the loads
    // of tile wt + stride are in flight while tile wt is transformed.  Codes
    // are read once and the fp16 vectors written once: both carry the
    // evict-first hint (.cs).
    struct Rows {
        uint32_t w[5];   // angle words from the lane's first one
        uint4 nq;        // norm bytes (LIN8: 16, LOG4: 8 in .x/.y)
        uint32_t pr;     // parameters (LIN8: fp16 M, LOG4: fp16 LO | HI << 16)
    };
    auto fetch = [&](uint32_t wt, Rows& R) {
        const uint32_t v = wt * VPW + grp;
        const uint32_t vv = (int64_t)v < A.n_vec ? v : 0u;
        const uint32_t vt = fast_div(vv, A.tdiv);
        const int64_t row =
            (int64_t)vt * A.in.capacity + A.pos0 + (int64_t)(vv - vt * (uint32_t)A.T);
        const uint32_t* ar = reinterpret_cast<const uint32_t*>(A.in.angles) + row * AW;
#pragma unroll
        for (int j = 0; j < 5; j++) R.w[j] = wbase + j < AW ? __ldcs(ar + wbase + j) : 0u;
        if (lin8) {
            R.nq = __ldcs(reinterpret_cast<const uint4*>(A.in.norms + row * (D / 2) + lg * 16));
            R.pr = reinterpret_cast<const uint16_t*>(A.in.params)[row];
        } else {
            const uint2 q2 = __ldcs(reinterpret_cast<const uint2*>(A.in.norms + row * (D / 4) + lg * 8));
            R.nq = make_uint4(q2.x, q2.y, 0u, 0u);
            R.pr = reinterpret_cast<const uint32_t*>(A.in.params)[row];
        }
    };
    Rows nxt;
    uint32_t wt = blockIdx.x * kDqWarps + warp;
    if (wt < n_tiles) fetch(wt, nxt);
    for (; wt < n_tiles; wt += stride) {
        const Rows cur = nxt;
        if (wt + stride < n_tiles) fetch(wt + stride, nxt);
        const uint32_t v = wt * VPW + grp;
        const bool valid = (int64_t)v < A.n_vec;
        // angle codes aligned to the lane's first bit
        uint32_t W[4];
#pragma unroll
        for (int j = 0; j < 4; j++) W[j] = __funnelshift_r(cur.w[j], cur.w[j + 1], sh);
        // norms: r / sqrt(d) of each pair
        float r[16];
        if (lin8) {
            const uint32_t nw[4] = {cur.nq.x, cur.nq.y, cur.nq.z, cur.nq.w};
            const float sc = half_bits_to_float((uint16_t)cur.pr) * (1.f / 255.f) * isd;
#pragma unroll
            for (int k = 0; k < 16; k++)
                r[k] = (float)((nw[k >> 2] >> (8 * (k & 3))) & 0xFFu) * sc;
        } else {
            // log2(r / sqrt(d)) = LO - S / 2 + c (HI - LO) / 15 = f A + B with
            // f = 1 + c / 16 (the nibble as mantissa bits, no conversion),
            // A = 16 (HI - LO) / 15, B = LO - S / 2 - A
            const float LO = half_bits_to_float((uint16_t)(cur.pr & 0xFFFF));
            const float A16 = (half_bits_to_float((uint16_t)(cur.pr >> 16)) - LO) * (16.f / 15.f);
            const float B16 = LO - 0.5f * (float)S - A16;
#pragma unroll
            for (int k = 0; k < 16; k++) {
                const int sh4 = 4 * (k & 7);
                const uint32_t w = k < 8 ? cur.nq.x : cur.nq.y;
                const uint32_t mant = sh4 <= 19 ? (w << (19 - sh4)) : (w >> (sh4 - 19));
                const float f = __uint_as_float((mant & 0x00780000u) | 0x3F800000u);
                asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r[k]) : "f"(fmaf(f, A16, B16)));
            }
        }
        f32x2 P[16];
#pragma unroll
        for (int k = 0; k < 16; k++) {
            // code k moved to bits 7 .. 7 + B - 1 (times 128 bytes), the
            // replica offset or-ed in below them
            constexpr uint32_t mask = ((1u << B) - 1u) << 7;
            const int pos = k * B, wi = pos >> 5, bi = pos & 31;
            const uint32_t x = bi + B > 32 ? __funnelshift_r(W[wi], W[wi + 1], bi - 7)
                               : bi >= 7   ? W[wi] >> (bi - 7)
                                           : W[wi] << (7 - bi);
            const float2 t =
                *reinterpret_cast<const float2*>(reinterpret_cast<const char*>(tab) + ((x & mask) | tlo));
            P[k] = pack2(r[k] * t.x, r[k] * t.y);
        }
        fwht_pairs<1>(P, lg);  // the in-lane stages
        runs.to_runs(P);
        fwht_runs<NL>(P);      // the stages over the former lane bits
        if (valid) {
            uint32_t o[16];
#pragma unroll
            for (int k = 0; k < 16; k++) {
                const __half2 h = __floats2half2_rn(lo2(P[k]), hi2(P[k]));
                o[k] = *reinterpret_cast<const uint32_t*>(&h) ^ m[k];
            }
            __half* y = A.y + (size_t)v * D + lg * T::RL;
#pragma unroll
            for (int Lh = 0; Lh < NL; Lh++) {
                const uint32_t* oo = o + Lh * (T::RL / 2);
                if constexpr (T::RL == 4) {
                    __stcs(reinterpret_cast<uint2*>(y + Lh * 32), make_uint2(oo[0], oo[1]));
                } else {
#pragma unroll
                    for (int c = 0; c < T::RL / 8; c++)
                        __stcs(reinterpret_cast<uint4*>(y + Lh * 32) + c,
                               make_uint4(oo[4 * c], oo[4 * c + 1], oo[4 * c + 2], oo[4 * c + 3]));
                }
            }
        }
    }
}

template <int D>
static cudaError_t launch_dequant_fast_d(const DqArgs& a, int sm_count, cudaStream_t stream) {
    constexpr int VPW = DqFastCfg<D>::VPW;
    const int64_t tiles = (a.n_vec + VPW - 1) / VPW;
    int64_t blocks = (tiles + kDqWarps - 1) / kDqWarps;
    // one wave of resident blocks, each striding over the tiles (no partly
    // filled last wave)
    const int64_t cap = (int64_t)sm_count * kDqFastBlocksPerSM;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    const dim3 g((unsigned)blocks), b(kDqWarps * 32);
    // the exchange buffer (32 KB) and its alignment; the table (at most
    // 32 KB) is static
    const size_t smem = 128 + (size_t)kDqWarps * LaneRuns<D / 32>::WARP_BYTES;
    // programmatic dependent launch (see the kernel)
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr.val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = g;
    cfg.blockDim = b;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
#define KVQ_DQ(BB)                                                                          \
    case BB: {                                                                              \
        const cudaError_t e = cudaFuncSetAttribute(                                         \
            dequant_fast_kernel<D, BB>, cudaFuncAttributeMaxDynamicSharedMemorySize,        \
            (int)smem);                                                                     \
        if (e != cudaSuccess) return e;                                                     \
        const cudaError_t l = cudaLaunchKernelEx(&cfg, dequant_fast_kernel<D, BB>, a);      \
        if (l != cudaSuccess) return l;                                                     \
        break;                                                                              \
    }
    switch (a.c.bits) {
        KVQ_DQ(1) KVQ_DQ(2) KVQ_DQ(3) KVQ_DQ(4) KVQ_DQ(5) KVQ_DQ(6) KVQ_DQ(7) KVQ_DQ(8)
        default: return cudaErrorInvalidValue;
    }
#undef KVQ_DQ
    return cudaGetLastError();
}

template <int D>
static cudaError_t launch_dequant_d(const DqArgs& a, int sm_count, cudaStream_t stream) {
    constexpr int VPW = DqCfg<D>::VPW;
    const int64_t tiles = (a.n_vec + VPW - 1) / VPW;
    int64_t blocks = (tiles + kDqWarps - 1) / kDqWarps;
    const int64_t cap = (int64_t)sm_count * 4;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    dequant_kernel<D><<<(unsigned)blocks, kDqWarps * 32, 0, stream>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_dequant(const CodecDev& c, const int8_t* signs, const PlaneDev& in,
                           int64_t n_vec, int64_t T, int64_t pos0, __half* y, int sm_count,
                           cudaStream_t stream) {
    DqArgs a;
    a.in = in;
    a.signs = signs;
    a.n_vec = n_vec;
    a.T = T;
    a.pos0 = pos0;
    a.c = c;
    a.y = y;
    a.inv_sqrt_d = (float)(1.0 / sqrt((double)c.d));
    a.tdiv = make_fast_div(n_vec <= (1ll << 31) && T >= 1 ? (uint32_t)T : 1u);
    if ((c.d == 64 || c.d == 128 || c.d == 256) && c.L <= 256 && n_vec <= (1ll << 31) && T >= 1) {
        switch (c.d) {
            case 64: return launch_dequant_fast_d<64>(a, sm_count, stream);
            case 128: return launch_dequant_fast_d<128>(a, sm_count, stream);
            default: return launch_dequant_fast_d<256>(a, sm_count, stream);
        }
    }
    switch (c.d) {
        case 4: return launch_dequant_d<4>(a, sm_count, stream);
        case 8: return launch_dequant_d<8>(a, sm_count, stream);
        case 16: return launch_dequant_d<16>(a, sm_count, stream);
        case 32: return launch_dequant_d<32>(a, sm_count, stream);
        case 64: return launch_dequant_d<64>(a, sm_count, stream);
        case 128: return launch_dequant_d<128>(a, sm_count, stream);
        case 256: return launch_dequant_d<256>(a, sm_count, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace kvq
