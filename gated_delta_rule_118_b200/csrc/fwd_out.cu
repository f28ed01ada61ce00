// fwd_out.cu -- the windowed output kernel: one CTA of 128 threads per
// (batch, head, chunk) of a window, running the chunk outputs of out_body.cuh
// on the records of the prep kernel and the state images of the chain kernel.
#include "launch.h"
#include "out_body.cuh"

namespace gdn2 {
namespace {

using namespace sm100;
using namespace outp;

constexpr int kOutThreads = 128;

template <int DV>
struct OutKernelLayout {
    static constexpr int BAR = OutLayout<DV>::DATA;
    static constexpr int SLOT = BAR + 16;
    static constexpr int BYTES = SLOT + 16 + 1024;
};

template <int DV>
__global__ void __launch_bounds__(kOutThreads)
out_kernel(const __grid_constant__ CUtensorMap tm_g, const uint8_t *__restrict__ ws, const uint8_t *__restrict__ sx,
           bf16 *__restrict__ o, const OutEpi epi, int Tlen, int H, int c0, int WC, unsigned int *err)
{
    using K = OutKernelLayout<DV>;
    using R = Record<DV>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5;
    const int cw = blockIdx.x, h = blockIdx.y, bi = blockIdx.z;
    const long idx = ((long)bi * H + h) * WC + cw;
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + K::BAR);
    uint32_t *slot = reinterpret_cast<uint32_t *>(sm + K::SLOT);

    if (tid == 0) {
        mbar_init(bar, 1);
        mbar_init(bar + 1, 1);
        fence_mbar_init();
        out_issue_loads<DV>(sm, bar, ws + idx * R::BYTES, sx + idx * SxSlot<DV>::BYTES, epi.g ? &tm_g : nullptr,
                            (c0 + cw) * kChunk, h, bi);
    }
    if (warp == 0) {
        tmem_alloc(slot, OutLayout<DV>::TMEM_COLS);
        tmem_relinquish();
    }
    // windows write disjoint outputs: the next window's output kernel may start early
    allow_dependent_launch();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *slot;
    const int ct0 = (c0 + cw) * kChunk;
    uint32_t phase = 0;
    const long row0 = (((long)bi * Tlen + ct0) * H + h) * (long)DV;
    out_chunk<DV, kOutThreads>(sm, tmem, tid, 0, bar, bar + 1, phase, o + row0, Tlen - ct0, (long)H * DV, epi, err);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, OutLayout<DV>::TMEM_COLS);
    }
}

template <int DV>
cudaError_t launch_out_impl(const FwdArgs &a, const CUtensorMap *tm_g, const uint8_t *ws, const uint8_t *sx, int c0,
                            int ncw, int WC, bool overlap)
{
    using L = OutKernelLayout<DV>;
    auto kern = out_kernel<DV>;
    static std::atomic<unsigned long long> smem_set{0};
    cudaError_t e = ensure_smem_limit(kern, L::BYTES, smem_set);
    if (e != cudaSuccess) return e;
    LaunchCfg lc(dim3(ncw, a.H, a.B), dim3(kOutThreads), L::BYTES, a.stream, overlap);
    const OutEpi epi{a.g, a.norm_weight, a.eps};
    return cudaLaunchKernelEx(&lc.cfg, kern, *tm_g, ws, sx, (bf16 *)a.o, epi, a.T, a.H, c0, WC, a.err);
}

}  // namespace

cudaError_t launch_out(const FwdArgs &a, const CUtensorMap *tm_g, const uint8_t *ws, const uint8_t *sx, int c0,
                       int ncw, int WC, bool overlap)
{
    return a.dv == 128 ? launch_out_impl<128>(a, tm_g, ws, sx, c0, ncw, WC, overlap)
                       : launch_out_impl<64>(a, tm_g, ws, sx, c0, ncw, WC, overlap);
}

}  // namespace gdn2
