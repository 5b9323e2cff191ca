// kvq_encode.cu - the encode/append kernels and their launcher: the streaming
// kernel of kvq_encode_fast.cuh where it applies, else the general one (the
// per-tile encoding of kvq_encode_impl.cuh, shared with the fused append).
#include "kvq_encode_fast.cuh"

namespace kvq {

template <int D>
__global__ void __launch_bounds__(kEncWarps * 32, kEncBlocksPerSM)
encode_kernel(EncPair PA) {
    // a kernel launched as this one's programmatic dependent (the decode of
    // the same step) may start its own setup now; it waits for this grid to
    // finish before reading anything this grid writes
    asm volatile("griddepcontrol.launch_dependents;");
    const EncArgs A = blockIdx.y ? PA.a[1] : PA.a[0];
    using Cfg = EncCfg<D>;
    constexpr int NL = Cfg::NL, PPL = Cfg::PPL, VPW = Cfg::VPW;
    __shared__ uint32_t stage[kEncWarps][kEncStageWords];

    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int grp = lane / NL;
    const int lg = lane % NL;

    uint32_t* st = stage[warp];
    for (int i = lane; i < kEncStageWords; i += 32) st[i] = 0u;
    uint32_t smask[PPL];
    lane_sign_masks<D>(A.signs, lg, smask);
    const float du = angle_margin(A);

    const int64_t n_warps_total = (int64_t)gridDim.x * kEncWarps;
    const int64_t n_warp_tiles = (A.n_vec + VPW - 1) / VPW;
    for (int64_t wt = (int64_t)blockIdx.x * kEncWarps + warp; wt < n_warp_tiles; wt += n_warps_total)
        (void)encode_tile<D, true>(A, wt, smask, st, du, lane, grp, lg);
}

template <int D>
static cudaError_t launch_encode_d(const EncPair& pa, int n_args, int sm_count,
                                   cudaStream_t stream) {
    constexpr int VPW = EncCfg<D>::VPW;
    int64_t n_max = pa.a[0].n_vec;
    if (n_args > 1 && pa.a[1].n_vec > n_max) n_max = pa.a[1].n_vec;
    const int64_t tiles = (n_max + VPW - 1) / VPW;
    int64_t blocks = (tiles + kEncWarps - 1) / kEncWarps;
    const int64_t cap = (int64_t)sm_count * kEncBlocksPerSM * 4 / n_args;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    encode_kernel<D><<<dim3((unsigned)blocks, (unsigned)n_args), kEncWarps * 32, 0, stream>>>(pa);
    return cudaGetLastError();
}

// The streaming and fixup kernels of kvq_encode_fast.cuh cover d = 64, 128,
// 256 and L % 8 == 0 with 16 <= L <= 256, for at most 2^31 vectors.
static bool fast_ok(const EncodeJob& j) {
    const int d = j.c.d, L = j.c.L;
    return (d == 64 || d == 128 || d == 256) && L % 8 == 0 && L >= 16 && L <= 256 &&
           j.n_vec <= (1ll << 31) && j.T >= 1;
}

template <int D>
static cudaError_t launch_encode_fast_d(const EncPair& pa, int n_args, int sm_count,
                                        cudaStream_t stream) {
    constexpr int VPW = FastCfg<D>::VPW;
    int64_t n_max = pa.a[0].n_vec;
    if (n_args > 1 && pa.a[1].n_vec > n_max) n_max = pa.a[1].n_vec;
    const int64_t tiles = (n_max + VPW - 1) / VPW;
    int64_t blocks = (tiles + kFastWarps - 1) / kFastWarps;
    const int64_t cap = (int64_t)sm_count * kFastBlocksPerSM * 4 / n_args;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    encode_fast_kernel<D>
        <<<dim3((unsigned)blocks, (unsigned)n_args), kFastWarps * 32, 0, stream>>>(pa);
    // the fixup pass: one warp per 128 vectors, two blocks per SM at most
    int64_t fblocks = ((n_max + 127) / 128 + kFastWarps - 1) / kFastWarps;
    if (fblocks > 2 * sm_count / n_args) fblocks = 2 * sm_count / n_args;
    if (fblocks < 1) fblocks = 1;
    encode_fixup_kernel<D>
        <<<dim3((unsigned)fblocks, (unsigned)n_args), kFastWarps * 32, 0, stream>>>(pa);
    return cudaGetLastError();
}

EncArgs encode_args(const CodecDev& c, const int8_t* signs) {
    EncArgs a = {};
    a.signs = signs;
    a.c = c;
    a.inv_sqrt_d = (float)(1.0 / sqrt((double)c.d));
    a.bins_per_rad = (float)((double)c.L / (2.0 * kPi));
    a.tdiv = make_fast_div(1);
    a.small = 1;
    return a;
}

static EncArgs make_args(const EncodeJob& j) {
    EncArgs a = encode_args(j.c, j.signs);
    a.x = j.x;
    a.n_vec = j.n_vec;
    a.T = j.T;
    a.pos0 = j.pos0;
    a.out = j.out;
    a.err_word = j.err_word;
    a.small = j.n_vec < (1ll << 32) && j.T >= 1 && j.T < (1ll << 32);
    a.tdiv = make_fast_div(a.small ? (uint32_t)j.T : 1u);
    return a;
}

cudaError_t launch_encode_jobs(const EncodeJob* jobs, int n_jobs, int sm_count,
                               cudaStream_t stream) {
    if (n_jobs < 1 || n_jobs > 2) return cudaErrorInvalidValue;
    if (n_jobs == 2 && jobs[0].c.d != jobs[1].c.d) return cudaErrorInvalidValue;
    EncPair pa;
    pa.a[0] = make_args(jobs[0]);
    pa.a[1] = n_jobs == 2 ? make_args(jobs[1]) : pa.a[0];
    if (fast_ok(jobs[0]) && (n_jobs == 1 || fast_ok(jobs[1]))) {
        switch (jobs[0].c.d) {
            case 64: return launch_encode_fast_d<64>(pa, n_jobs, sm_count, stream);
            case 128: return launch_encode_fast_d<128>(pa, n_jobs, sm_count, stream);
            case 256: return launch_encode_fast_d<256>(pa, n_jobs, sm_count, stream);
            default: break;
        }
    }
    switch (jobs[0].c.d) {
        case 4: return launch_encode_d<4>(pa, n_jobs, sm_count, stream);
        case 8: return launch_encode_d<8>(pa, n_jobs, sm_count, stream);
        case 16: return launch_encode_d<16>(pa, n_jobs, sm_count, stream);
        case 32: return launch_encode_d<32>(pa, n_jobs, sm_count, stream);
        case 64: return launch_encode_d<64>(pa, n_jobs, sm_count, stream);
        case 128: return launch_encode_d<128>(pa, n_jobs, sm_count, stream);
        case 256: return launch_encode_d<256>(pa, n_jobs, sm_count, stream);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_encode(const CodecDev& c, const int8_t* signs, const __half* x, int64_t n_vec,
                          int64_t T, int64_t pos0, const PlaneDev& out, int sm_count,
                          cudaStream_t stream) {
    const EncodeJob j{c, signs, x, n_vec, T, pos0, out, nullptr};
    return launch_encode_jobs(&j, 1, sm_count, stream);
}

}  // namespace kvq
