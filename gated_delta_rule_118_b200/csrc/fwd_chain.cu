// fwd_chain.cu -- the windowed chain kernel: one CTA per (batch, head, value
// tile) walks the chunks of one window through the chain of chain_body.cuh,
// reading the records the window's prep kernel wrote and exporting the state
// images for the window's output kernel.
#include "chain_body.cuh"
#include "launch.h"

namespace gdn2 {
namespace {

using namespace sm100;
using namespace chain;

template <int DV, int DVT>
__global__ void __launch_bounds__(kChainThreads, 1)
chain_kernel(const uint8_t *__restrict__ ws, uint8_t *__restrict__ sx_out, const float *S_in, float *S_out,
             int H, int ncw, int WC, unsigned int *err)
{
    using L = ChainLayout<DV, DVT>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5;
    const int tile = blockIdx.x, h = blockIdx.y, bi = blockIdx.z;
    uint32_t *slot = reinterpret_cast<uint32_t *>(sm + L::SLOT);
    const long pair = (long)bi * H + h;

    if (tid == 0) chain_init<DV, DVT>(sm);
    if (warp == 0) {
        tmem_alloc(slot, L::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *slot;
    // This window's chain is resident: the next window's prep may take the other
    // SMs.  Then wait for this window's prep (its records, and through its own
    // final wait the previous chain and the state it carries).
    allow_dependent_launch();
    wait_prior_grid();

    const WindowFlow<DV> f{ws + pair * WC * (long)Record<DV>::BYTES, sx_out + pair * WC * (long)SxSlot<DV>::BYTES};
    chain_run<DV, DVT>(sm, tmem, tid, f, S_in, S_out, pair, tile, ncw, err);

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, L::TMEM_COLS);
    }
}

}  // namespace

template <int DV, int DVT>
cudaError_t launch_chain_impl(const FwdArgs &a, const uint8_t *ws, uint8_t *sx, const float *S_in, float *S_out,
                              int ncw, int WC, bool overlap)
{
    using L = ChainLayout<DV, DVT>;
    auto kern = chain_kernel<DV, DVT>;
    static std::atomic<unsigned long long> smem_set{0};
    cudaError_t e = ensure_smem_limit(kern, L::BYTES, smem_set);
    if (e != cudaSuccess) return e;
    dim3 grid(DV / DVT, a.H, a.B);
    LaunchCfg lc(grid, dim3(kChainThreads), L::BYTES, a.stream, overlap);
    return cudaLaunchKernelEx(&lc.cfg, kern, ws, sx, S_in, S_out, a.H, ncw, WC, a.err);
}

cudaError_t launch_chain(const FwdArgs &a, int dvt, const uint8_t *ws, uint8_t *sx, const float *S_in,
                         float *S_out, int ncw, int WC, bool overlap)
{
    if (a.dv == 128) {
        if (dvt == 128) return launch_chain_impl<128, 128>(a, ws, sx, S_in, S_out, ncw, WC, overlap);
        return launch_chain_impl<128, 64>(a, ws, sx, S_in, S_out, ncw, WC, overlap);
    }
    return launch_chain_impl<64, 64>(a, ws, sx, S_in, S_out, ncw, WC, overlap);
}

}  // namespace gdn2
