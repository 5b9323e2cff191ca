// kvq_decode_impl.cuh - the split-K decode attention kernel (template), with
// the split combine fused in.  Instantiated per (head_dim, G) in the
// kvq_decode_d*_g*.cu files; dispatched from kvq_decode.cu.
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
//   - thread 0 streams tiles of kTT tokens of the six code arrays (K/V
//     angles, norms, params) into a 2..4-deep shared-memory ring with 1-D bulk
//     asynchronous copies (TMA, no multicast), tracked by "full" mbarriers
//     (transaction bytes) and recycled through "empty" mbarriers that every
//     warp arrives on; a stage is refilled one tile after it was released,
//     so the refill never waits on the warps still working; every wait is
//     bounded, a timeout is reported in the error word and the kernel drains
//     its copies and returns instead of trapping;
//   - consumer warps take blocks of consecutive tokens; a group of NL lanes
//     owns four tokens, each lane PP pairs of them and the matching pairs of
//     all G query heads of the KV head (GQA), so every unpacked code serves G
//     heads;
//   - the work per pair is kept to a handful of instructions: a key norm
//     byte becomes the float 1 + c 2^-15 in one byte permute, and with U =
//     (cos, sin) from the table, fma(f, U, -U) is 2^-15 c (cos, sin)
//     rounded once (no int-to-float conversion; the exact 2^-15 is undone in
//     the score scale, and equal K and V codebooks share one table); a value
//     norm nibble is
//     or-ed into the mantissa of 1.0 (f = 1 + c/16) and one FMA gives the
//     exponent LO + c (HI - LO)/15; table bases are folded into the load
//     address where the tables fit in static shared memory;
//   - partial scores meet in a transpose-reduce over the group in which every
//     lane sends the same register each round: a lane's query heads and token
//     order are permuted once, by its lane bits, so no per-round select is
//     needed; the softmax weights reach the value pass through a small
//     per-warp buffer in shared memory as (p, p) pairs;
//   - angle codes have compile-time widths (BK, BV in 5..8; 0 = runtime) so
//     a code becomes a table offset in two integer operations; bin-centre
//     cos/sin tables are replicated 16 times so a half-warp's 64-bit lookups
//     never share a bank;
//   - the online softmax rescales lazily, only when a score exceeds the
//     running reference max by more than 2^8;
//   - per-split partials (m, l, acc[d]) go to the workspace; the last CTA of a
//     (batch, KV head) to finish (atomic counter, no waiting) merges the
//     splits, divides by l, applies the inverse FWHT and D_V / sqrt(d).
#pragma once

#include <mutex>

#include "kvq_encode_impl.cuh"
#include "kvq_internal.h"

namespace kvq {

constexpr int kTT = 128;          // tokens per staged tile (paged caches; TT of an instance)
constexpr int kMaxStages = 4;     // ring depth (2..4, chosen per launch)
constexpr int kTPG = 4;           // tokens per group chunk
constexpr float kLazyThr = 8.f;   // log2 units
constexpr int kTabRep = 16;       // table replicas (one per half-warp lane)
constexpr int kTabShift = 7;      // log2(kTabRep * sizeof(float2))

// True when the two replicated cos/sin tables of fixed code widths (bk, bv)
// fit in static shared memory (48 KB).
constexpr bool decode_static_tables(int bk, int bv) {
    return bk > 0 && bv > 0 && ((1 << bk) + (1 << bv)) * kTabRep * 8 <= 48 * 1024;
}

// CTAS: resident CTAs per SM the instance is built for.  With one, a lane
// owns 32 / G pairs (at most 16) of each token; with two, half as many (at
// least 4), which halves its query and accumulator registers (4 G PP of
// them) so that two 8-warp CTAs fit beside each other on an SM.
template <int D, int G, int CTAS = 1, int TT = kTT>
struct DecCfg {
    static constexpr int P = D / 2;
    static constexpr int PP_MAX = CTAS == 1 ? 32 / G : (16 / G < 4 ? 4 : 16 / G);
    static constexpr int PP = PP_MAX > 16 ? 16 : PP_MAX;        // pairs per lane
    static constexpr int NL = P / PP;                          // lanes per token group
    static constexpr int GPW = 32 / NL;                        // groups per warp
    static constexpr int TW = GPW * kTPG;                      // tokens per warp block
    static constexpr int WARPS = (TT / TW) > 8 ? 8 : ((TT / TW) < 2 ? 2 : (TT / TW));
    static constexpr int THREADS = WARPS * 32;
    static constexpr int NG = WARPS * GPW;                     // groups per CTA
    static constexpr int V = kTPG * G;                         // partial sums per lane
    static constexpr int VF = V / NL;                          // final sums per lane
    static constexpr int PBUF = TW * G * 2;                    // floats of (p, p) per warp
    static_assert(VF >= 1, "group too wide");
    static_assert(PP % 4 == 0, "codes are unpacked four at a time");
    static_assert(TT % (TW * WARPS) == 0, "blocks must tile the stage");
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

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
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

// Bounded wait: false when `limit` tries ran out.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity,
                                                  uint32_t limit = kWaitLimit) {
    for (uint32_t it = 0; it < limit; ++it)
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

// Wait until the grids this one depends on have completed and their memory
// is visible (a no-op without a programmatic dependency).
__device__ __forceinline__ void griddep_wait() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

// Arrive on named barrier `id` without waiting (the producer side).
__device__ __forceinline__ void named_arrive(int id, int count) {
    asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// Barrier over `count` threads (a multiple of 32) of the CTA, id 1..15.
__device__ __forceinline__ void named_barrier(int id, int count) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// Orders this thread's generic-proxy global writes before later async-proxy
// (bulk copy) reads of them.
__device__ __forceinline__ void fence_proxy_async_global() {
    asm volatile("fence.proxy.async.global;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// ---------------------------------------------------------- clusters ----

// Barrier over every thread of every CTA of the cluster; release/acquire
// make each CTA's shared-memory writes before it visible to the others after.
__device__ __forceinline__ void cluster_barrier() {
    asm volatile(
        "barrier.cluster.arrive.release.aligned;\n\t"
        "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Address of the same shared-memory offset in cluster CTA `rank`.
__device__ __forceinline__ uint32_t dsmem_addr(uint32_t smem_addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_addr), "r"(rank));
    return r;
}

__device__ __forceinline__ float dsmem_f32(uint32_t addr) {
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
    return v;
}

__device__ __forceinline__ float2 dsmem_f32x2(uint32_t addr) {
    float2 v;
    asm volatile("ld.shared::cluster.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(addr)
                 : "memory");
    return v;
}

__device__ __forceinline__ float4 dsmem_f32x4(uint32_t addr) {
    float4 v;
    asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"(addr)
                 : "memory");
    return v;
}

// ------------------------------------------------------- group exchange --

// Reduce over the NL lanes of a group, halving the live entries each round:
// every lane adds its partner's v[i + half] to its own v[i].  For the result
// to be a transpose-reduce, slot i of lane lg must hold logical entry
// i ^ (lg * VF) (the caller arranges that once, by permuting the query heads
// and token order it computes into each slot); then on return v[0..VF) holds
// the group sums of the logical entries lg * VF + e.
template <int V, int NL>
__device__ __forceinline__ void xor_reduce(float (&v)[V]) {
#pragma unroll
    for (int r = 0; (NL >> (r + 1)) >= 1; r++) {
        const int o = NL >> (r + 1);
        const int half = V >> (r + 1);
#pragma unroll
        for (int i = 0; i < half; i++) v[i] += __shfl_xor_sync(KVQ_FULL_MASK, v[i + half], o);
    }
}

// Loads from the shared window at a 32-bit address (smem_u32); volatile, so
// that they stay behind the mbarrier wait that made the staged bytes valid.
template <int OFF = 0>
__device__ __forceinline__ uint32_t lds_u32(uint32_t a) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1+%2];" : "=r"(v) : "r"(a), "n"(OFF));
    return v;
}
template <int OFF = 0>
__device__ __forceinline__ uint2 lds_u64(uint32_t a) {
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2+%3];" : "=r"(v.x), "=r"(v.y) : "r"(a), "n"(OFF));
    return v;
}
template <int OFF = 0>
__device__ __forceinline__ uint4 lds_u128(uint32_t a) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4+%5];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(a), "n"(OFF));
    return v;
}
template <int OFF = 0>
__device__ __forceinline__ uint32_t lds_u16(uint32_t a) {
    unsigned short v;
    asm volatile("ld.shared.u16 %0, [%1+%2];" : "=h"(v) : "r"(a), "n"(OFF));
    return v;
}
template <int OFF = 0>
__device__ __forceinline__ uint32_t lds_u8(uint32_t a) {
    unsigned short v;
    asm volatile("ld.shared.u8 %0, [%1+%2];" : "=h"(v) : "r"(a), "n"(OFF));
    return v;
}
// Softmax weights handed from the score pass to the value pass of a warp:
// explicit shared accesses with a memory clobber, ordered by the __syncwarp
// on either side of the hand-off.
__device__ __forceinline__ void sts_pp(uint32_t a, float p) {
    asm volatile("st.shared.v2.f32 [%0], {%1, %1};" ::"r"(a), "f"(p) : "memory");
}
template <int OFF = 0>
__device__ __forceinline__ float4 lds_pp4(uint32_t a) {
    float4 v;
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4+%5];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"(a), "n"(OFF)
                 : "memory");
    return v;
}
__device__ __forceinline__ float2 lds_pp2(uint32_t a) {
    float2 v;
    asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(a) : "memory");
    return v;
}
__device__ __forceinline__ float2 lds_f2(uint32_t a) {
    float2 v;
    asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(a));
    return v;
}
template <int OFF = 0>
__device__ __forceinline__ float4 lds_f4(uint32_t a) {
    float4 v;
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4+%5];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"(a), "n"(OFF));
    return v;
}

// Shared addresses of the 16x replicated float2 table entries of this lane's
// PP angle codes: table + lane16 * 8 + code * 128, the codes being bits
// [cb, cb + PP*B) of the row at shared address `row` (wa = its first word:
// the row address plus 4 (cb >> 5); sh = cb & 31).  B > 0: compile-time
// width; B == 0: runtime width `bits`.
template <int PP, int B, bool TABC = false>
__device__ __forceinline__ void angle_addrs(uint32_t wa, int sh, int bits, uint32_t tab_lane,
                                            uint32_t (&off)[PP]) {
    if constexpr (B > 0) {
        constexpr int NB = PP * B;             // chunk bits
        constexpr int NW = (NB + 31) / 32;     // normalised words
        constexpr uint32_t mask = ((1u << B) - 1u) << kTabShift;
        uint32_t w[NW + 2];
        w[0] = lds_u32<0>(wa);
        if constexpr (NW >= 1) w[1] = lds_u32<4>(wa);
        if constexpr (NW >= 2) w[2] = lds_u32<8>(wa);
        if constexpr (NW >= 3) w[3] = lds_u32<12>(wa);
        if constexpr (NW >= 4) w[4] = lds_u32<16>(wa);
        static_assert(NW <= 4, "at most 128 code bits per lane");
        uint32_t n[NW + 1];
#pragma unroll
        for (int i = 0; i < NW; i++) n[i] = __funnelshift_r(w[i], w[i + 1], sh);
        n[NW] = 0u;
#pragma unroll
        for (int k = 0; k < PP; k++) {
            const int pos = k * B;             // compile-time after unrolling
            const int wi = pos >> 5, bi = pos & 31;
            uint32_t x;
            if (bi + B <= 32) {
                x = bi >= kTabShift ? (n[wi] >> (bi - kTabShift)) : (n[wi] << (kTabShift - bi));
            } else {
                x = __funnelshift_r(n[wi], n[wi + 1], bi - kTabShift);
            }
            // with a table at a compile-time address the lane's replica offset
            // (below bit kTabShift) is or-ed in with the mask, and the base
            // is left to the load's immediate (see tab_f2)
            off[k] = TABC ? ((x & mask) | tab_lane) : ((x & mask) + tab_lane);
        }
    } else {
        const uint32_t mask = (1u << bits) - 1u;
#pragma unroll
        for (int q = 0; q < PP / 4; q++) {
            const int pos = sh + q * 4 * bits;  // from the first word of the lane
            const uint32_t a = wa + 4u * (uint32_t)(pos >> 5);
            const uint32_t win = __funnelshift_r(lds_u32<0>(a), lds_u32<4>(a), pos & 31);
#pragma unroll
            for (int k = 0; k < 4; k++)
                off[4 * q + k] = (((win >> (k * bits)) & mask) << kTabShift) + tab_lane;
        }
    }
}

// Table entry at byte offset `off` of a table in static shared memory: a
// plain shared load, so the compiler can carry the table base in the load's
// immediate.  The tables are written before the barrier that precedes every
// lookup.
__device__ __forceinline__ float2 tab_f2(const float2* tab, uint32_t off) {
    return *reinterpret_cast<const float2*>(reinterpret_cast<const char*>(tab) + off);
}

// NBYTES bytes (1, 2, 4, 8, 16) at shared address a as little-endian words.
template <int NBYTES>
__device__ __forceinline__ void lds_bytes(uint32_t a, uint32_t (&w)[(NBYTES + 3) / 4]) {
    if constexpr (NBYTES == 16) {
        const uint4 q = lds_u128(a);
        w[0] = q.x; w[1] = q.y; w[2] = q.z; w[3] = q.w;
    } else if constexpr (NBYTES == 8) {
        const uint2 q = lds_u64(a);
        w[0] = q.x; w[1] = q.y;
    } else if constexpr (NBYTES == 4) {
        w[0] = lds_u32(a);
    } else if constexpr (NBYTES == 2) {
        w[0] = lds_u16(a);
    } else {
        static_assert(NBYTES == 1, "1, 2, 4, 8 or 16 bytes");
        w[0] = lds_u8(a);
    }
}

// ------------------------------------------------------------- kernel ---

template <int D, int G, int BK, int BV, int CTAS, int TT>
__global__ void __launch_bounds__(DecCfg<D, G, CTAS, TT>::THREADS, CTAS)
decode_kernel(DecodeArgs A) {
    // A kernel launched after this one as its programmatic dependent (the
    // next layer's or step's decode) may start its setup once every CTA here
    // has started: it touches no global memory before griddepcontrol.wait,
    // which returns only when this grid has completed and its writes are
    // visible, so it overlaps its barrier setup and tables with this tail.
    asm volatile("griddepcontrol.launch_dependents;");
    using Cfg = DecCfg<D, G, CTAS, TT>;
    constexpr int P = Cfg::P, PP = Cfg::PP, NL = Cfg::NL, GPW = Cfg::GPW, NG = Cfg::NG;
    constexpr int WARPS = Cfg::WARPS, TW = Cfg::TW;
    constexpr int V = Cfg::V, VF = Cfg::VF;
    constexpr int EPQ = D / 32;
    constexpr int CONSUMERS = WARPS * 32;

    // cos/sin tables: in static shared memory when both widths are fixed and
    // the tables fit (their address is then a constant of the load), in the
    // dynamic allocation otherwise
    constexpr bool kStatic = decode_static_tables(BK, BV);
    __shared__ __align__(128) float2 s_tab[kStatic ? ((1 << BK) + (1 << BV)) * kTabRep : 1];
    extern __shared__ __align__(16) unsigned char smem[];
    const int NST = A.nstages;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);           // [kMaxStages]
    uint64_t* empty = full + kMaxStages;                          // [kMaxStages]
    int* sflag = reinterpret_cast<int*>(smem + 16 * kMaxStages);  // timeout, last
    // table sizes: compile-time for fixed widths (so are the table addresses)
    const int nK = 1 << (BK > 0 ? BK : A.kc.bits), nV = 1 << (BV > 0 ? BV : A.vc.bits);
    unsigned char* dyn = smem + 16 * kMaxStages + 16;
    // key table (cos, sin) [2^bK][16], value table (cos, sin) [2^bV][16]
    // equal codebooks share one dynamic table (the key path uses it unscaled)
    const bool share = !kStatic && A.kc.L == A.vc.L;
    float2* tabK = kStatic ? s_tab : reinterpret_cast<float2*>(dyn);
    float2* tabV = share ? tabK : tabK + nK * kTabRep;
    if (!kStatic) dyn += sizeof(float2) * kTabRep * (size_t)(share ? nK : nK + nV);
    float* qs = reinterpret_cast<float*>(dyn);                    // [G][D]
    uint32_t* encst = reinterpret_cast<uint32_t*>(qs + G * D);    // [2][kEncStageWords]
    float* pbuf_all = reinterpret_cast<float*>(encst + 2 * kEncStageWords);  // [WARPS][PBUF]
    unsigned char* stages = smem + A.stage_offset;                // [kStages][stage]

    const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    // ---- token range of this split -----------------------------------------
    // Copies start before ctx_len is known: they cover the split up to the
    // host bound min(max_ctx, capacity); tokens past ctx_len[b] are masked.
    const int64_t lim = A.max_ctx < A.K.capacity ? A.max_ctx : A.K.capacity;
    const int64_t t0 = (int64_t)split * A.split_len;
    const int64_t t1m = (t0 + A.split_len < lim) ? t0 + A.split_len : lim;
    const int ntiles_max = t1m > t0 ? (int)((t1m - t0 + TT - 1) / TT) : 0;
    if (tid == 0) {
        for (int s = 0; s < NST; s++) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], WARPS);
        }
        mbar_fence_init();
        sflag[0] = 0;
        sflag[1] = 0;
    }
    __syncthreads();

    // ---- producer lane: the first NST tiles go out before the prologue ------
    int issued = 0;  // tiles issued (producer lane 0)
    auto issue_tile = [&](int tile) {
        const int rbK = A.kc.angle_words * 4, rbV = A.vc.angle_words * 4;
        const int s = tile % NST;
        const int64_t tt0 = t0 + (int64_t)tile * TT;
        // a tile never crosses a page: pages hold whole 128-token tiles and
        // paged splits start on a multiple of 128
        bool bad = false;
        const int64_t rowK = plane_row(A.K, b, kvh, tt0, &bad);
        const int64_t rowV = plane_row(A.V, b, kvh, tt0, &bad);
        if (bad) report(A.err_word, KVQ_DEVERR_PAGE_RANGE);
        const uint8_t* srcs[6] = {A.K.angles + rowK * rbK, A.K.norms + rowK * A.kc.norm_bytes,
                                  A.K.params + rowK * A.kc.param_bytes, A.V.angles + rowV * rbV,
                                  A.V.norms + rowV * A.vc.norm_bytes,
                                  A.V.params + rowV * A.vc.param_bytes};
        const int rbs[6] = {rbK, A.kc.norm_bytes, A.kc.param_bytes, rbV, A.vc.norm_bytes,
                            A.vc.param_bytes};
        const int64_t left = t1m - tt0;
        const int n16 = (int)(((left < TT ? left : TT) + 15) / 16 * 16);
        uint32_t bytes = 0;
#pragma unroll
        for (int k = 0; k < 6; k++) bytes += (uint32_t)(n16 * rbs[k]);
        fence_proxy_async();
        mbar_expect_tx(&full[s], bytes);
        unsigned char* dst = stages + (size_t)s * A.stage_bytes;
#pragma unroll
        for (int k = 0; k < 6; k++)
            bulk_g2s(dst + A.lay[k], srcs[k], (uint32_t)(n16 * rbs[k]), &full[s]);
    };
    // tile t + NST - 1 is issued once tile t - 1 is released, so NST - 1 tiles
    // are in flight ahead of the one being consumed
    // Launched as a programmatic dependent of the previous kernel on the
    // stream (the previous layer's or step's decode), the kernel may start
    // before that one ends: nothing it reads from global memory (codes, q,
    // ctx_len, signs) is touched before griddepcontrol.wait; the barrier setup
    // and the cos/sin tables overlap the previous kernel's tail.  After a
    // separate append launch (append_pending) everything but the new row is
    // already final when the kernel starts, so only that row's tile waits.
    // Fused append (kvq_decode_step): the split holding the new token (position
    // ctx_len[b] - 1) encodes it with warps 0 and 1 while the other warps build
    // the tables and rotate q; the tile holding it, and the ones after, are
    // copied in only after it is written.  Without an append all warps share
    // the tables and q.
    // the two-CTA instance carries no append code (its registers would not
    // fit); its kvq_decode_step runs the append as a launch of its own first
    const bool fused = CTAS == 1 && A.k_new != nullptr;
    // append_kernel ran just before (see DecodeArgs::append_pending): only the
    // tile holding the new row waits for it, every other read starts at once
    const bool pending = A.append_pending != 0;
    const int w0 = fused ? 2 : 0;  // first warp of the table / q' work
    int64_t ctx_in = 0;
    bool append = false;           // warps 0 and 1 of a fused launch
    if (fused && warp < 2) {
        griddep_wait();
        ctx_in = A.ctx_len[b];
        append = ctx_in >= 1 && ctx_in <= lim && ctx_in - 1 >= t0 && ctx_in - 1 < t1m;
    }
    int hold = ntiles_max;  // (thread 0) first tile that waits for the append
    if (tid == 0) {
        if (pending) {
            const int64_t c = A.ctx_len[b];
            if (c >= 1 && c <= lim && c - 1 >= t0 && c - 1 < t1m) hold = (int)((c - 1 - t0) / TT);
        } else {
            griddep_wait();
            if (append) hold = (int)((ctx_in - 1 - t0) / TT);
        }
        for (; issued < NST - 1 && issued < ntiles_max && issued < hold; issued++) issue_tile(issued);
        if (pending && issued < NST - 1 && issued < ntiles_max) {
            griddep_wait();
            hold = ntiles_max;
            for (; issued < NST - 1 && issued < ntiles_max; issued++) issue_tile(issued);
        }
        // from here on only a pending append's tile waits (in the refill)
        if (!pending || hold >= ntiles_max) hold = 1 << 30;
    }
    if (fused && warp < 2) {
        if constexpr (CTAS == 1) if (append) {
            // the same encode_tile as kvq_encode, one vector per warp
            using ECfg = EncCfg<D>;
            EncArgs E = warp == 0 ? A.enc_k : A.enc_v;
            const int64_t bh = (int64_t)b * A.H_kv + kvh;
            E.x = (warp == 0 ? A.k_new : A.v_new) + bh * D;
            E.n_vec = 1;
            E.T = 1;
            E.pos0 = ctx_in - 1;
            E.bh0 = bh;
            E.out = warp == 0 ? A.K : A.V;
            E.err_word = A.err_word;
            uint32_t* est = encst + warp * kEncStageWords;
            for (int i = lane; i < kEncStageWords; i += 32) est[i] = 0u;
            __syncwarp();
            const int elg = lane % ECfg::NL, egrp = lane / ECfg::NL;
            uint32_t smask[ECfg::PPL];
            lane_sign_masks<D>(E.signs, elg, smask);
            (void)encode_tile<D, true>(E, 0, smask, est, angle_margin(E), lane, egrp, elg);
            fence_proxy_async_global();
        }
        named_barrier(1, 64);
        if (tid == 0 && append)
            for (; issued < NST - 1 && issued < ntiles_max; issued++) issue_tile(issued);
    }

    // ---- tables and q' (overlap the first copies and the append) -------------
    // tabV follows tabK (or is tabK), so the tables are one array of nTab
    // entries of kTabRep replicas.  Each bin centre is computed once, into
    // replica 0; the other replicas are then copied by consecutive threads
    // writing consecutive addresses (no bank conflicts).
    if (warp >= w0) {
        const int nthr = CONSUMERS - 32 * w0, t = tid - 32 * w0;
        const int nTab = tabV == tabK ? nK : nK + nV;
#pragma unroll 1
        for (int e = t; e < nTab; e += nthr) {
            const bool isK = e < nK;
            const int a = isK ? e : e - nK;
            float s, c;
            sincospif((float)(2 * a + 1) / (float)(isK ? A.kc.L : A.vc.L) - 1.f, &s, &c);
            tabK[e * kTabRep] = make_float2(c, s);
        }
        named_barrier(2, nthr);
#pragma unroll 1
        for (int idx = t; idx < nTab * kTabRep; idx += nthr)
            if (idx % kTabRep) tabK[idx] = tabK[idx - idx % kTabRep];
        if (!pending) griddep_wait();
        ctx_in = A.ctx_len[b];
        for (int h = warp - w0; h < G; h += WARPS - w0) {
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
            if constexpr (EPQ == 4) {
                reinterpret_cast<float4*>(qs + h * D)[lane] =
                    make_float4(v[0] * isd, v[1] * isd, v[2] * isd, v[3] * isd);
            } else {
#pragma unroll
                for (int e = 0; e < EPQ; e++) qs[h * D + lane * EPQ + e] = v[e] * isd;
            }
        }
    }
    int64_t ctx = ctx_in;
    if (ctx < 0 || ctx > lim) {
        if (split == 0 && kvh == 0 && tid == 0) report(A.err_word, KVQ_DEVERR_CTX_RANGE);
        ctx = ctx < 0 ? 0 : lim;
    }
    const int64_t t1 = t1m < ctx ? t1m : ctx;
    const int span = t1 > t0 ? (int)(t1 - t0) : 0;  // a split is far shorter than 2^31 tokens
    const int ntiles = t1 > t0 ? (int)((t1 - t0 + TT - 1) / TT) : 0;
    // every issued tile is consumed (tiles past the context are fully masked)
    const int nloop = ntiles > (NST - 1 < ntiles_max ? NST - 1 : ntiles_max)
                          ? ntiles
                          : (NST - 1 < ntiles_max ? NST - 1 : ntiles_max);
    if (fused) {
        // the table / q' warps start on the tiles at once; the append warps
        // join when done (barrier 3: the others only arrive, they do not wait)
        if (warp >= w0) {
            named_barrier(2, CONSUMERS - 32 * w0);
            named_arrive(3, CONSUMERS);
        } else {
            named_barrier(3, CONSUMERS);
        }
    } else {
        __syncthreads();
    }

    const int grp = lane / NL, lg = lane % NL;
    // Slot (j, h) of a lane's partial scores holds the logical entry
    // (j ^ JX, h ^ HX) (token slot, head) so that xor_reduce needs no selects;
    // after it, final entry e is logical M + e: token slot (M + e) / G, head
    // (M + e) % G, with softmax reference mh[e].
    const int M = lg * VF;
    const int HX = M % G, JX = M / G;
    const int bitsK = BK > 0 ? BK : A.kc.bits, bitsV = BV > 0 ? BV : A.vc.bits;
    const int cbK = lg * PP * bitsK, cbV = lg * PP * bitsV;
    // all staged data is addressed by 32-bit shared-window offsets; row
    // strides are compile-time constants for the fixed code widths
    const int rbK = 4 * (BK > 0 ? (P * BK + 31) / 32 : A.kc.angle_words);
    const int rbV = 4 * (BV > 0 ? (P * BV + 31) / 32 : A.vc.angle_words);
    const uint32_t lane_off = (uint32_t)(lane & 15) * 8u;
    // static tables: both table addresses are compile-time constants (tabV
    // follows 2^BK key entries), so lookups take the lane offset alone
    constexpr bool kTabC = kStatic;
    const uint32_t tKl = kTabC ? lane_off : smem_u32(tabK) + lane_off;
    const uint32_t tVl = kTabC ? lane_off : smem_u32(tabV) + lane_off;
    const uint32_t wK = 4u * (uint32_t)(cbK >> 5), wV = 4u * (uint32_t)(cbV >> 5);
    const int shK = cbK & 31, shV = cbV & 31;
    const uint32_t stages32 = smem_u32(stages);
    // ---- merge the NG group states of this CTA (reuses the stage memory) --
    // accumulators as [G][PP][NG * 2 NL + pad]: a warp writes one (h, k) row
    // segment of 32 consecutive float2 (no bank conflicts), and the pad puts
    // the next k row on the other half of the banks for the summing pass
    constexpr int ROW = NG * 2 * NL + 16;
    float* gm = reinterpret_cast<float*>(stages);  // [NG][G]  running maxima
    float* gl = gm + NG * G;                      // [NG][G]  denominators, then weights
    float* gacc = gl + NG * G;                    // [G][PP][ROW]
    float* hml = gacc + G * PP * ROW;             // [G][2]   CTA max and denominator

    const int gidx = warp * GPW + grp;
    float2 acc[G][PP];
    float mref[G];
    float lpart[VF];
#pragma unroll
    for (int h = 0; h < G; h++) {
        mref[h] = -INFINITY;
#pragma unroll
        for (int k = 0; k < PP; k++) acc[h][k] = make_float2(0.f, 0.f);
    }
#pragma unroll
    for (int e = 0; e < VF; e++) lpart[e] = 0.f;

    float mh[VF];  // softmax reference of final entry e
#pragma unroll
    for (int e = 0; e < VF; e++) mh[e] = -INFINITY;
    // [TW][G] (p, p) of this warp's block
    const uint32_t pbuf = smem_u32(pbuf_all + warp * Cfg::PBUF);

    {
        float2 q2[G][PP];
#pragma unroll
        for (int h = 0; h < G; h++)
#pragma unroll
            for (int k = 0; k < PP; k++) {
                const float2 qq = reinterpret_cast<const float2*>(qs + (h ^ HX) * D)[lg * PP + k];
                q2[h][k] = qq;
            }

        for (int tile = 0; tile < nloop; tile++) {
            const int s = tile % NST;
            const bool got = mbar_wait_bounded(&full[s], (uint32_t)(tile / NST) & 1u, A.wait_limit);
            if (!__all_sync(KVQ_FULL_MASK, got)) {
                if (lane == 0) atomicOr(&sflag[0], 1);
                break;
            }
            if (__any_sync(KVQ_FULL_MASK, *((volatile int*)&sflag[0]) != 0)) break;
            const uint32_t st = stages32 + (uint32_t)(s * A.stage_bytes);
            const uint32_t sKa = st + A.lay[0] + wK, sKn = st + A.lay[1] + lg * PP;
            const uint32_t sKp = st + A.lay[2];
            const uint32_t sVa = st + A.lay[3] + wV, sVn = st + A.lay[4] + lg * (PP / 2);
            const uint32_t sVp = st + A.lay[5];
            const int left = span - tile * TT;  // tokens of the split from this tile on
            const int ntok = left < TT ? left : TT;

            for (int blk = warp; blk * TW < ntok; blk += WARPS) {
                // -- scores: this lane's partial dot products, slot (j, h) --
                // token slot j ^ JX (rows consecutive across the warp), head h ^ HX
                float part[V];
#pragma unroll
                for (int j = 0; j < kTPG; j++) {
                    const int t = blk * TW + (j ^ JX) * GPW + grp;
                    uint32_t off[PP];
                    angle_addrs<PP, BK, kTabC>(sKa + (uint32_t)(t * rbK), shK, bitsK, tKl, off);
                    uint32_t nw[(PP + 3) / 4];
                    lds_bytes<PP>(sKn + (uint32_t)(t * P), nw);
                    float2 dot[G];
#pragma unroll
                    for (int k = 0; k < PP; k++) {
                        // norm byte c -> f = 1 + c 2^-15 (bytes 0x3F 0x80 c 0x00);
                        // with U = (cos, sin) from the table, fma(f, U, -U) =
                        // (f - 1) U = 2^-15 c (cos, sin), rounded once (the
                        // 2^-15 is exact and undone in the score scale); the
                        // first pair starts the accumulators (no zeroing)
                        const float f = __uint_as_float(
                            __byte_perm(nw[k / 4], 0x3F800000u, 0x7604u | ((k % 4) << 4)));
                        const float2 U = kTabC ? tab_f2(tabK, off[k]) : lds_f2(off[k]);
                        const float2 xy =
                            __ffma2_rn(make_float2(f, f), U, make_float2(-U.x, -U.y));
#pragma unroll
                        for (int h = 0; h < G; h++)
                            dot[h] = k == 0 ? __fmul2_rn(q2[h][k], xy) : __ffma2_rn(q2[h][k], xy, dot[h]);
                    }
#pragma unroll
                    for (int h = 0; h < G; h++) part[j * G + h] = dot[h].x + dot[h].y;
                }
                xor_reduce<V, NL>(part);
                // -- scale by M/255 * tau * log2(e), mask, lazy softmax reference
                bool need = false;
#pragma unroll
                for (int e = 0; e < VF; e++) {
                    const int t = blk * TW + ((M + e) / G) * GPW + grp;
                    const float Mk = half_bits_to_float((uint16_t)lds_u16(sKp + 2u * (uint32_t)t));
                    // M/255, times 2^15 for the key products' 2^-15
                    float sv = part[e] * (Mk * (32768.f / 255.f)) * A.scale_log2;
                    sv = t < ntok ? sv : -INFINITY;
                    part[e] = sv;
                    need |= sv > mh[e] + kLazyThr;
                }
                if (__any_sync(KVQ_FULL_MASK, need)) {
                    float mx[G];
#pragma unroll
                    for (int h = 0; h < G; h++) mx[h] = -INFINITY;
#pragma unroll
                    for (int e = 0; e < VF; e++) {
                        const int h = (M + e) % G;
#pragma unroll
                        for (int hh = 0; hh < G; hh++)
                            if (hh == h) mx[hh] = fmaxf(mx[hh], part[e]);
                    }
#pragma unroll
                    for (int h = 0; h < G; h++) {
                        mx[h] = group_max<NL>(mx[h]);
                        const float mn = fmaxf(mref[h], mx[h]);
                        const float al = (mn == -INFINITY) ? 0.f : ex2(mref[h] - mn);
                        const float2 al2 = make_float2(al, al);
#pragma unroll
                        for (int k = 0; k < PP; k++) acc[h][k] = __fmul2_rn(acc[h][k], al2);
#pragma unroll
                        for (int e = 0; e < VF; e++)
                            if ((M + e) % G == h) lpart[e] *= al;
                        mref[h] = mn;
                    }
#pragma unroll
                    for (int e = 0; e < VF; e++) {
                        const int h = (M + e) % G;
                        float m = mref[0];
#pragma unroll
                        for (int hh = 1; hh < G; hh++) m = (hh == h) ? mref[hh] : m;
                        mh[e] = m;
                    }
                }
                // -- softmax weights to this warp's buffer as (p, p) pairs --
                __syncwarp();  // the previous block's value pass is done with it
#pragma unroll
                for (int e = 0; e < VF; e++) {
                    const int idx = M + e;
                    const float p = part[e] == -INFINITY ? 0.f : ex2(part[e] - mh[e]);
                    lpart[e] += p;
                    sts_pp(pbuf + 8u * (uint32_t)(((idx / G) * GPW + grp) * G + idx % G), p);
                }
                __syncwarp();
                // -- values: acc[h] += p[t][h] * r^ (cos, sin), rotated domain --
#pragma unroll
                for (int j = 0; j < kTPG; j++) {
                    const int tl = j * GPW + grp;
                    const int t = blk * TW + tl;
                    float2 pw[G];
                    if constexpr (G == 1) {
                        pw[0] = lds_pp2(pbuf + 8u * (uint32_t)tl);
                    } else {
                        const uint32_t pa = pbuf + 8u * (uint32_t)(tl * G);
                        float4 v = lds_pp4<0>(pa);
                        pw[0] = make_float2(v.x, v.y);
                        pw[1] = make_float2(v.z, v.w);
                        if constexpr (G >= 4) {
                            v = lds_pp4<16>(pa);
                            pw[2] = make_float2(v.x, v.y);
                            pw[3] = make_float2(v.z, v.w);
                        }
                        if constexpr (G >= 8) {
                            v = lds_pp4<32>(pa);
                            pw[4] = make_float2(v.x, v.y);
                            pw[5] = make_float2(v.z, v.w);
                            v = lds_pp4<48>(pa);
                            pw[6] = make_float2(v.x, v.y);
                            pw[7] = make_float2(v.z, v.w);
                        }
                    }
                    uint32_t off[PP];
                    angle_addrs<PP, BV, kTabC>(sVa + (uint32_t)(t * rbV), shV, bitsV, tVl, off);
                    uint32_t nw[(PP / 2 + 3) / 4];
                    lds_bytes<PP / 2>(sVn + (uint32_t)(t * (P / 2)), nw);
                    const uint32_t pr = lds_u32(sVp + 4u * (uint32_t)t);
                    const float LO = half_bits_to_float((uint16_t)(pr & 0xFFFF));
                    // log2 r^ = LO + c (HI - LO)/15 = f A + B with f = 1 + c/16,
                    // A = 16 (HI - LO)/15, B = LO - A
                    float A16 = (half_bits_to_float((uint16_t)(pr >> 16)) - LO) * (16.f / 15.f);
                    float B16 = LO - A16;
                    // rows past the context hold stale bytes: make their r^ finite
                    // (their softmax weight is already 0)
                    A16 = t < ntok ? A16 : 0.f;
                    B16 = t < ntok ? B16 : -64.f;
#pragma unroll
                    for (int k = 0; k < PP; k++) {
                        // nibble k of the word -> mantissa bits 19..22 of 1.0
                        const int sh = 4 * (k % 8);
                        const uint32_t w = nw[k / 8];
                        const uint32_t mant = sh <= 19 ? (w << (19 - sh)) : (w >> (sh - 19));
                        const float f = __uint_as_float((mant & 0x00780000u) | 0x3F800000u);
                        const float r = ex2(fmaf(f, A16, B16));
                        const float2 cs = kTabC ? tab_f2(tabV, off[k]) : lds_f2(off[k]);
                        const float2 xy = __fmul2_rn(make_float2(r, r), cs);
#pragma unroll
                        for (int h = 0; h < G; h++) acc[h][k] = __ffma2_rn(pw[h], xy, acc[h][k]);
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
            // refill: tile + NST - 1 goes into the stage tile - 1 used, once every
            // warp has released it (normally already true)
            if (tid == 0 && issued < nloop && issued == tile + NST - 1) {
                const int nxt = issued;
                const int sn = nxt % NST;
                bool ok = true;
                if (nxt >= NST)
                    ok = mbar_wait_bounded(&empty[sn], (uint32_t)((nxt / NST) - 1) & 1u,
                                           A.wait_limit);
                if (ok) {
                    if (nxt >= hold) {
                        griddep_wait();  // the append's rows are written
                        hold = 1 << 30;
                    }
                    issue_tile(nxt);
                    issued = nxt + 1;
                } else {
                    atomicOr(&sflag[0], 1);
                }
            }
        }
    }

    __syncthreads();
    if (sflag[0]) {
        // a wait ran out: report, then wait (bounded) for the copies still in
        // flight before the shared memory is released; this CTA contributes
        // nothing to the output
        if (tid == 0) {
            report(A.err_word, KVQ_DEVERR_TIMEOUT);
            // the newest tile of each stage covers the older ones
            for (int t = issued - NST > 0 ? issued - NST : 0; t < issued; t++)
                (void)mbar_wait_bounded(&full[t % NST], (uint32_t)(t / NST) & 1u);
        }
        __syncthreads();
#pragma unroll
        for (int h = 0; h < G; h++) {
            mref[h] = -INFINITY;
#pragma unroll
            for (int k = 0; k < PP; k++) acc[h][k] = make_float2(0.f, 0.f);
        }
#pragma unroll
        for (int e = 0; e < VF; e++) lpart[e] = 0.f;
    }

    {
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
            for (int k = 0; k < PP; k++)
                reinterpret_cast<float2*>(gacc + (h * PP + k) * ROW)[gidx * NL + lg] =
                    acc[h][k];
    }
    __syncthreads();
    // per head: the CTA max, each group's weight 2^(m_g - max), the denominator
    for (int h = warp; h < G; h += WARPS) {
        float mx = -INFINITY;
        for (int g = lane; g < NG; g += 32) mx = fmaxf(mx, gm[g * G + h]);
        mx = group_max<32>(mx);
        float sl = 0.f;
        for (int g = lane; g < NG; g += 32) {
            const float w = mx == -INFINITY ? 0.f : ex2(gm[g * G + h] - mx);
            sl += w * gl[g * G + h];
            gl[g * G + h] = w;
        }
        sl = group_sum<32>(sl);
        if (lane == 0) {
            hml[2 * h] = mx;
            hml[2 * h + 1] = sl;
        }
    }
    __syncthreads();

    const int S = A.num_splits;
    float* stats = A.ws + ws_counter_floats(A.B, A.H_q);
    float* accs = stats + ws_stat_floats(A.B, A.H_q, S);
    // clustered launch: this CTA's partial stays in its own shared memory,
    // [G][D + 4] = acc[D], m, l (16-byte aligned rows)
    float* part = hml + (2 * G + 3) / 4 * 4;
    // thread -> (h, k, lg, c) with (lg, c) fastest: consecutive threads read
    // consecutive floats of a row; element j = 2 (lg PP + k) + c
    for (int idx = tid; idx < G * D; idx += CONSUMERS) {
        const int lc = idx % (2 * NL), hk = idx / (2 * NL);
        const int h = hk / PP, k = hk % PP;
        const int j = 2 * ((lc >> 1) * PP + k) + (lc & 1);
        const float* row = gacc + hk * ROW + lc;
        float a0 = 0.f, a1 = 0.f;
        int g = 0;
        for (; g + 2 <= NG; g += 2) {
            a0 = fmaf(gl[g * G + h], row[g * 2 * NL], a0);
            a1 = fmaf(gl[(g + 1) * G + h], row[(g + 1) * 2 * NL], a1);
        }
        for (; g < NG; g++) a0 = fmaf(gl[g * G + h], row[g * 2 * NL], a0);
        if (A.cluster) {
            part[h * (D + 4) + j] = a0 + a1;
            if (j == 0) {
                part[h * (D + 4) + D] = hml[2 * h];
                part[h * (D + 4) + D + 1] = hml[2 * h + 1];
            }
        } else {
            const int64_t slot = ((int64_t)b * A.H_q + (int64_t)kvh * G + h) * S + split;
            accs[slot * D + j] = a0 + a1;
            if (j == 0) {
                stats[slot * 2] = hml[2 * h];
                stats[slot * 2 + 1] = hml[2 * h + 1];
            }
        }
    }

    // ---- clustered launch: the splits of this (b, KV head) are one cluster
    // and merge through distributed shared memory: cluster CTA r takes heads
    // r, r + S, ... (one warp per head), reading every split's partial
    if (A.cluster) {
        cluster_barrier();
        const uint32_t part_s = smem_u32(part);
        for (int h = split + S * warp; h < G; h += S * WARPS) {
            const int64_t hq = (int64_t)b * A.H_q + (int64_t)kvh * G + h;
            const uint32_t row = part_s + (uint32_t)(h * (D + 4)) * 4u;
            float m_l = -INFINITY, l_l = 0.f;  // lane s holds split s (S <= 32)
            if (lane < S) {
                const uint32_t rr = dsmem_addr(row, (uint32_t)lane);
                m_l = dsmem_f32(rr + 4u * D);
                l_l = dsmem_f32(rr + 4u * (D + 1));
            }
            const float mx = group_max<32>(m_l);
            const float w_l = (lane < S && mx != -INFINITY) ? ex2(m_l - mx) : 0.f;
            const float sl = group_sum<32>(w_l * l_l);
            float v[EPQ];
#pragma unroll
            for (int e = 0; e < EPQ; e++) v[e] = 0.f;
#pragma unroll 4
            for (int sp = 0; sp < S; sp++) {
                const float w = __shfl_sync(KVQ_FULL_MASK, w_l, sp);
                const uint32_t ra = dsmem_addr(row, (uint32_t)sp) + 4u * (uint32_t)(lane * EPQ);
                if constexpr (EPQ == 4) {
                    const float4 x = dsmem_f32x4(ra);
                    v[0] = fmaf(w, x.x, v[0]);
                    v[1] = fmaf(w, x.y, v[1]);
                    v[2] = fmaf(w, x.z, v[2]);
                    v[3] = fmaf(w, x.w, v[3]);
                } else {
                    const float2 x = dsmem_f32x2(ra);
                    v[0] = fmaf(w, x.x, v[0]);
                    v[1] = fmaf(w, x.y, v[1]);
                }
            }
            const float inv = sl > 0.f ? 1.f / sl : 0.f;
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
        // no CTA leaves while another may still read its partial
        cluster_barrier();
        return;
    }

    // partials only (kvq_decode_attn_partials): the caller merges them
    if (A.partials_only) return;

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
    // one warp per head: the common max and denominator over the splits (lane
    // s holds split s), the weighted sum of the split accumulators, the inverse
    // FWHT, D_V / sqrt(d), the store
    for (int h = warp; h < G; h += WARPS) {
        const int64_t hq = (int64_t)b * A.H_q + (int64_t)kvh * G + h;
        const float* stp = stats + hq * S * 2;
        const float* ac = accs + hq * S * D + lane * EPQ;
        float mx = -INFINITY;
        for (int s = lane; s < S; s += 32) mx = fmaxf(mx, __ldcg(stp + 2 * s));
        mx = group_max<32>(mx);
        float sl = 0.f;
        float v[EPQ];
#pragma unroll
        for (int e = 0; e < EPQ; e++) v[e] = 0.f;
        if (mx != -INFINITY) {
            for (int c0 = 0; c0 < S; c0 += 32) {
                const int s_l = c0 + lane;
                const float w_l = s_l < S ? ex2(__ldcg(stp + 2 * s_l) - mx) : 0.f;
                sl += s_l < S ? w_l * __ldcg(stp + 2 * s_l + 1) : 0.f;
                const int n = S - c0 < 32 ? S - c0 : 32;
                if constexpr (EPQ == 4) {
#pragma unroll 8
                    for (int k = 0; k < n; k++) {
                        const float w = __shfl_sync(KVQ_FULL_MASK, w_l, k);
                        const float4 x =
                            __ldcg(reinterpret_cast<const float4*>(ac + (int64_t)(c0 + k) * D));
                        v[0] = fmaf(w, x.x, v[0]);
                        v[1] = fmaf(w, x.y, v[1]);
                        v[2] = fmaf(w, x.z, v[2]);
                        v[3] = fmaf(w, x.w, v[3]);
                    }
                } else {
#pragma unroll 8
                    for (int k = 0; k < n; k++) {
                        const float w = __shfl_sync(KVQ_FULL_MASK, w_l, k);
                        const float2 x =
                            __ldcg(reinterpret_cast<const float2*>(ac + (int64_t)(c0 + k) * D));
                        v[0] = fmaf(w, x.x, v[0]);
                        v[1] = fmaf(w, x.y, v[1]);
                    }
                }
            }
        }
        sl = group_sum<32>(sl);
        const float inv = sl > 0.f ? 1.f / sl : 0.f;
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

// Shared-memory plan of one launch (ring depth 4, 3 or 2, whichever fits in
// `avail` bytes of dynamic shared memory); returns 0 bytes when even two
// stages do not fit.
template <int D, int G, int BK, int BV, int CTAS, int TT>
inline size_t decode_smem_plan(DecodeArgs& a, size_t avail, int min_stages) {
    using Cfg = DecCfg<D, G, CTAS, TT>;
    size_t off = 16 * kMaxStages + 16;
    if (!decode_static_tables(BK, BV))  // one table when the codebooks are equal
        off += sizeof(float2) * kTabRep *
               (size_t)(a.kc.L == a.vc.L ? (1 << a.kc.bits) : (1 << a.kc.bits) + (1 << a.vc.bits));
    off += sizeof(float) * G * D + sizeof(uint32_t) * 2 * kEncStageWords +
           sizeof(float) * Cfg::WARPS * Cfg::PBUF;
    off = (off + 15) / 16 * 16;
    a.stage_offset = (int)off;
    const int rb[6] = {a.kc.angle_words * 4, a.kc.norm_bytes, a.kc.param_bytes,
                       a.vc.angle_words * 4, a.vc.norm_bytes, a.vc.param_bytes};
    int sb = 0;
    for (int k = 0; k < 6; k++) {
        a.lay[k] = sb;
        // +16: the last row's code window may read one word past its region
        sb += (TT * rb[k] + 16 + 15) / 16 * 16;
    }
    a.stage_bytes = sb;
    const size_t merge =
        sizeof(float) * ((size_t)2 * Cfg::NG * G +
                         (size_t)G * Cfg::PP * (Cfg::NG * 2 * Cfg::NL + 16) +
                         (size_t)(2 * G + 3) / 4 * 4 + (size_t)G * (D + 4));
    for (int ns = kMaxStages; ns >= min_stages; ns--) {
        size_t ring = (size_t)ns * sb;
        if (ring < merge) ring = merge;
        if (off + ring <= avail) {
            a.nstages = ns;
            return off + ring;
        }
    }
    return 0;
}

// Largest cluster the combine uses (non-portable beyond 8 CTAs).
constexpr int kMaxClusterSplits = 16;

// Per-device launch facts of one kernel instance, set up once under a lock:
// SM count, the dynamic shared memory left beside its static tables, and how
// many clusters of S CTAs can be resident at once for a given dynamic size
// (the generic-width instance's size varies with the code widths).
struct DecodeLaunchCache {
    std::mutex lock;
    bool init[64] = {};
    int sm_count[64] = {};
    size_t avail[64] = {};
    struct Entry {
        int dev, S;
        size_t smem;
        int n;
    };
    Entry entries[256];
    int n_entries = 0;
};

template <int D, int G, int BK, int BV, int CTAS, int TT = kTT>
inline cudaError_t launch_decode_kernel(DecodeArgs a, cudaStream_t stream, int min_stages = 2) {
    using Cfg = DecCfg<D, G, CTAS, TT>;
    auto kernel = decode_kernel<D, G, BK, BV, CTAS, TT>;
    static DecodeLaunchCache cache;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    size_t avail;
    int sm_count;
    {
        std::lock_guard<std::mutex> g(cache.lock);
        if (!cache.init[dev]) {
            cudaFuncAttributes fa;
            e = cudaFuncGetAttributes(&fa, kernel);
            if (e != cudaSuccess) return e;
            // per CTA: 227 KB, or half the SM's 228 KB less the 1 KB the
            // system reserves per CTA when two share the SM
            const size_t dyn = (CTAS == 1 ? 227 * 1024 : 228 * 1024 / 2 - 1024) -
                               fa.sharedSizeBytes;
            e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dyn);
            if (e != cudaSuccess) return e;
            e = cudaFuncSetAttribute(kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
            if (e != cudaSuccess) return e;
            int n = 0;
            e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
            if (e != cudaSuccess) return e;
            cache.sm_count[dev] = n;
            cache.avail[dev] = dyn;
            cache.init[dev] = true;
        }
        avail = cache.avail[dev];
        sm_count = cache.sm_count[dev];
    }
    const size_t smem = decode_smem_plan<D, G, BK, BV, CTAS, TT>(a, avail, min_stages);
    if (smem == 0) return cudaErrorInvalidConfiguration;
    dim3 grid((unsigned)a.num_splits, (unsigned)a.H_kv, (unsigned)a.B);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(Cfg::THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)a.num_splits;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    // programmatic dependent launch: see griddep_wait in the kernel
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    // the cluster combine pays off only when every cluster of the launch is
    // resident at once (it saves the L2 round trip of the last-CTA combine);
    // the GPC layout admits only a few large clusters at a time, so ask the
    // occupancy calculator rather than count SMs
    const int S = a.num_splits;
    a.cluster = 0;
    if (S <= kMaxClusterSplits && !a.partials_only &&
        (int64_t)a.B * a.H_kv * S <= (int64_t)sm_count) {
        int n = -1;
        {
            std::lock_guard<std::mutex> g(cache.lock);
            for (int i = 0; i < cache.n_entries; i++)
                if (cache.entries[i].dev == dev && cache.entries[i].S == S &&
                    cache.entries[i].smem == smem)
                    n = cache.entries[i].n;
        }
        if (n < 0) {
            cfg.attrs = attr;
            cfg.numAttrs = 1;
            const cudaError_t q = cudaOccupancyMaxActiveClusters(&n, kernel, &cfg);
            if (q != cudaSuccess) {
                (void)cudaGetLastError();
                n = 0;
            }
            std::lock_guard<std::mutex> g(cache.lock);
            if (cache.n_entries < 256) cache.entries[cache.n_entries++] = {dev, S, smem, n};
        }
        a.cluster = (int64_t)a.B * a.H_kv <= (int64_t)n;
    }
    cfg.attrs = a.cluster ? attr : attr + 1;
    cfg.numAttrs = a.cluster ? 2 : 1;
    e = cudaLaunchKernelEx(&cfg, kernel, a);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

// The append of kvq_decode_step as its own launch (kvq_decode_generic.cu),
// for the instances that carry no append code.
cudaError_t launch_append(const DecodeArgs& a, cudaStream_t stream);

// The two-CTA instance of fixed widths (bk, bv): for G up to 4 with codes of
// 5..7 bits (its tables then fit in static shared memory beside a ring of
// tiles in half an SM), on a paged cache, when the launch needs more than one
// wave of one-CTA launches.  On a contiguous cache the one-CTA instance with
// 256-token tiles is as fast per layer and keeps the append fused (one launch
// per layer instead of two): the Mistral-shaped 32-layer step took 8.38 ms
// that way against 8.49 ms with this instance.
inline bool decode_two_ctas(const DecodeArgs& a, int G, int sm_count) {
    return G <= 4 && a.kc.bits >= 5 && a.kc.bits <= 7 && a.vc.bits >= 5 && a.vc.bits <= 7 &&
           a.K.pages != nullptr && (int64_t)a.B * a.H_kv * a.num_splits > (int64_t)sm_count;
}

// One CTA per SM with 256-token tiles where the ring still gets three stages,
// the cache is contiguous (a paged cache guarantees whole pages only for
// 128-token tiles) and a split spans more than one such tile, else 128-token
// tiles.  Longer tiles halve the per-tile cost of the copy pipeline: the ring
// streamed 1.45x faster with the compute taken out, and layers ran 11-12 %
// faster.  A split of at most 256 tokens would be one tile, copied in whole
// before any compute; as two tiles the second's copy overlaps the first's
// compute (a one-wave launch of 228-token splits: 14.5 -> 13.8 us).
template <int D, int G, int BK, int BV>
inline cudaError_t launch_one_cta(const DecodeArgs& a, cudaStream_t stream) {
    if (a.K.pages == nullptr && a.V.pages == nullptr && a.split_len > 256) {
        const cudaError_t e = launch_decode_kernel<D, G, BK, BV, 1, 256>(a, stream, 3);
        if (e != cudaErrorInvalidConfiguration) return e;
    }
    return launch_decode_kernel<D, G, BK, BV, 1>(a, stream);
}

// Fast kernels for code widths 5..8 (codebooks of 17..256 entries), the
// runtime-width kernel for anything else.
template <int D, int G>
inline cudaError_t launch_decode_dg(const DecodeArgs& a, cudaStream_t stream) {
    const int bk = a.kc.bits, bv = a.vc.bits;
    if constexpr (G <= 4) {
        if (decode_two_ctas(a, G, device_sm_count())) {
            DecodeArgs b = a;
            if (a.k_new) {
                const cudaError_t e = launch_append(a, stream);
                if (e != cudaSuccess) return e;
                b.k_new = b.v_new = nullptr;
                b.append_pending = 1;
            }
#define KVQ_BB2(X, Y) \
    if (bk == X && bv == Y) return launch_decode_kernel<D, G, X, Y, 2>(b, stream);
            KVQ_BB2(5, 5) KVQ_BB2(5, 6) KVQ_BB2(5, 7)
            KVQ_BB2(6, 5) KVQ_BB2(6, 6) KVQ_BB2(6, 7)
            KVQ_BB2(7, 5) KVQ_BB2(7, 6) KVQ_BB2(7, 7)
#undef KVQ_BB2
        }
    }
#define KVQ_BB(X, Y) \
    if (bk == X && bv == Y) return launch_one_cta<D, G, X, Y>(a, stream);
    KVQ_BB(5, 5) KVQ_BB(5, 6) KVQ_BB(5, 7) KVQ_BB(5, 8)
    KVQ_BB(6, 5) KVQ_BB(6, 6) KVQ_BB(6, 7) KVQ_BB(6, 8)
    KVQ_BB(7, 5) KVQ_BB(7, 6) KVQ_BB(7, 7) KVQ_BB(7, 8)
    KVQ_BB(8, 5) KVQ_BB(8, 6) KVQ_BB(8, 7) KVQ_BB(8, 8)
#undef KVQ_BB
    return launch_decode_kernel<D, G, 0, 0, 1>(a, stream);
}

}  // namespace kvq
