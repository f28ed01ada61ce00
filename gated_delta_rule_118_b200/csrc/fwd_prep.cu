// fwd_prep.cu -- the windowed prep kernel: one CTA of 256 threads per
// (batch, head, chunk) of a window, two CTAs per SM, running the chunk prep of
// prep_body.cuh (the state-independent part of the chunkwise forward).
#include <cuda.h>

#include "launch.h"
#include "prep_body.cuh"

namespace gdn2 {
namespace {

using namespace sm100;
using namespace prep;

// TP: the backward's prep, which also keeps every chunk's T, P and the low
// part of T in `tp` (kTpBytes per chunk, indexed like the records).
template <int DV, bool TP>
__global__ void __launch_bounds__(kPrepThreads, 2)
prep_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
            const __grid_constant__ CUtensorMap tm_b, const __grid_constant__ CUtensorMap tm_la,
            const bf16 *__restrict__ vg, const bf16 *__restrict__ wg, const GateSrc gs, uint8_t *__restrict__ ws,
            int Tlen, int H, int c0, int WC, unsigned int *err, uint8_t *__restrict__ tp)
{
    using L = PrepLayout;
    using R = Record<DV>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5;
    const int cw = blockIdx.x, h = blockIdx.y, bi = blockIdx.z;
    const int t0 = (c0 + cw) * kChunk;
    uint64_t *bar_tma = reinterpret_cast<uint64_t *>(sm + L::BAR);
    uint64_t *bar_mma = bar_tma + 1;
    uint32_t *slot = reinterpret_cast<uint32_t *>(sm + L::SLOT);
    const long idx = ((long)bi * H + h) * WC + cw;
    uint8_t *rec = ws + idx * (long)R::BYTES;

    if (tid == 0) {
        mbar_init(bar_tma, 1);
        mbar_init(bar_mma, 1);
        fence_mbar_init();
        prep_issue_loads(sm, bar_tma, &tm_q, &tm_k, &tm_b, &tm_la, t0, h, bi, gs.layout);
    }
    if (warp == 0) {
        tmem_alloc(slot, L::TMEM_COLS);
        tmem_relinquish();
    }
    // chunks are independent: the next window's prep may start filling SMs
    allow_dependent_launch();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *slot;
    uint32_t mma_phase = 0;
    prep_chunk<DV, TP>(sm, tmem, tid, 0, bar_tma, 0, bar_mma, mma_phase, vg, wg, gs, rec, Tlen, H, t0, h, bi, err,
                       TP ? tp + idx * kTpBytes : nullptr);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, L::TMEM_COLS);
    }
    // When launched behind the previous window's chain, end only after it: the
    // next chain waits for this grid and so also for the state it carries.
    wait_prior_grid();
}

}  // namespace

template <int DV, bool TP>
cudaError_t launch_prep_impl(const FwdArgs &a, const CUtensorMap *maps, uint8_t *ws, int c0, int ncw, int WC,
                             bool overlap, uint8_t *tp)
{
    using L = PrepLayout;
    auto kern = prep_kernel<DV, TP>;
    static std::atomic<unsigned long long> smem_set{0};
    cudaError_t e = ensure_smem_limit(kern, L::BYTES, smem_set);
    if (e != cudaSuccess) return e;
    LaunchCfg lc(dim3(ncw, a.H, a.B), dim3(kPrepThreads), L::BYTES, a.stream, overlap);
    const GateSrc gs{(const bf16 *)a.b, a.log_alpha, a.layout};
    return cudaLaunchKernelEx(&lc.cfg, kern, maps[0], maps[1], maps[2], maps[3], (const bf16 *)a.v,
                              (const bf16 *)a.w, gs, ws, a.T, a.H, c0, WC, a.err, tp);
}

cudaError_t launch_prep(const FwdArgs &a, const CUtensorMap *maps, uint8_t *ws, int c0, int ncw, int WC, bool overlap,
                        uint8_t *tp)
{
    if (tp)
        return a.dv == 128 ? launch_prep_impl<128, true>(a, maps, ws, c0, ncw, WC, overlap, tp)
                           : launch_prep_impl<64, true>(a, maps, ws, c0, ncw, WC, overlap, tp);
    return a.dv == 128 ? launch_prep_impl<128, false>(a, maps, ws, c0, ncw, WC, overlap, nullptr)
                       : launch_prep_impl<64, false>(a, maps, ws, c0, ncw, WC, overlap, nullptr);
}

}  // namespace gdn2
