// kvq_dequant.cu - dequant kernel: packed codes -> fp16 head vectors.
//
// Reconstruction of "TurboAngle: Near-Lossless KV Cache Compression via
// Uniform Angle Quantization" (Abstract): each pair becomes
// r^ (cos theta^, sin theta^) with theta^ the centre of its angle bin, and the
// vector returns to the original domain through the inverse rotation
// D H / sqrt(d) (H symmetric, H H = d I).  r^ = c M / 255 (8-bit linear) or
// 2^(LO + c (HI - LO) / 15) (4-bit log space).
//
// Work layout mirrors the encode kernel: one vector per group of NL lanes,
// EPL elements per lane, FWHT in registers plus shuffles, 128-bit stores.
// cos/sin of the L bin centres come from a shared-memory table (L <= 4096)
// or from sincospif for larger codebooks.
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
