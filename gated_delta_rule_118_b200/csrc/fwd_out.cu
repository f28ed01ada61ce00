// fwd_out.cu -- the outputs of the chunkwise forward (bf16 inputs).
//
// The query reads the updated state ("Gated DeltaNet-2", iplexlaw.co.kr,
// section "Decisiones independientes en dos ejes"); in the chunkwise form the
// outputs of a chunk are
//   O = P T Z + (Qhat - P T Ehat) Diag(e^{Gamma_r}) S = PT Z + QS Sx,
// with PT, Z and QS from the chunk's prep record and Sx the bf16 image of the
// incoming state exported by the chain kernel.  Nothing here is sequential in
// the chunk index, so one CTA per (batch, head, chunk) accumulates the two
// products in tensor memory (M = 64 tokens, N = dv; K = 64 tokens, then K = dk)
// and writes its 64 output rows.
#include "launch.h"
#include "tc_common.cuh"

namespace gdn2 {
namespace {

using namespace sm100;

constexpr int kOutThreads = 128;

template <int DV>
struct OutLayout {
    static constexpr int QS = 0;                    // QS [64][128] K-major, no swizzle
    static constexpr int PT = 16384;                // PT [64][64] K-major, no swizzle
    static constexpr int Z = 24576;                 // Z, DV/64 blocks of [64][64] (MN-major)
    static constexpr int SX = Z + 64 * DV * 2;      // Sx [128][DV] (MN-major, no swizzle)
    static constexpr int TX = SX + 128 * DV * 2;
    static constexpr int BAR = TX;
    static constexpr int SLOT = BAR + 16;
    static constexpr int BYTES = SLOT + 16 + 1024;
    static_assert(SX % 1024 == 0, "swizzle atoms");
};

template <int DV>
__global__ void __launch_bounds__(kOutThreads)
out_kernel(const uint8_t *__restrict__ ws, const uint8_t *__restrict__ sx, bf16 *__restrict__ o, int Tlen,
           int H, int c0, int WC, unsigned int *err)
{
    using L = OutLayout<DV>;
    using R = Record<DV>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int cw = blockIdx.x, h = blockIdx.y, bi = blockIdx.z;
    const long idx = ((long)bi * H + h) * WC + cw;
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + L::BAR);
    uint32_t *slot = reinterpret_cast<uint32_t *>(sm + L::SLOT);
    const uint32_t sbase = smem_u32(sm);

    if (tid == 0) {
        mbar_init(bar, 1);
        mbar_init(bar + 1, 1);
        fence_mbar_init();
        const uint8_t *rec = ws + idx * R::BYTES;
        mbar_arrive_expect_tx(bar, (uint32_t)L::TX);
        bulk_load(sm + L::QS, rec + R::QS, 16384, bar);
        bulk_load(sm + L::PT, rec + R::PT, 8192, bar);
        bulk_load(sm + L::Z, rec + R::Z, 64 * DV * 2, bar);
        bulk_load(sm + L::SX, sx + idx * SxSlot<DV>::BYTES, 128 * DV * 2, bar);
    }
    if (warp == 0) {
        tmem_alloc(slot, DV);
        tmem_relinquish();
    }
    // windows write disjoint outputs: the next window's output kernel may start early
    allow_dependent_launch();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *slot;

    bool ok = (tid == 0) ? mbar_wait(bar, 0, err) : true;
    if (tid == 0 && ok) {
        const uint32_t id = idesc_bf16(64, DV, 0, 1);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
            umma_bf16(tmem, smem_desc(sbase + L::PT + ks * 2048, 1024, 128, kSwNone),
                      smem_desc(sbase + L::Z + ks * 2048, 8192, 1024, kSw128), id, ks > 0);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
            umma_bf16(tmem, smem_desc(sbase + L::QS + ks * 2048, 1024, 128, kSwNone),
                      smem_desc(sbase + L::SX + ks * 256, 128, 2048, kSwNone), id, 1);
        umma_commit(bar + 1);
        ok = mbar_wait(bar + 1, 0, err);
    }
    ok = __syncthreads_and(ok) != 0;
    if (ok) {
        tc_fence_after();
        // M = 64 accumulator: row 16*warp + l sits in TMEM lane 32*warp + l (l < 16)
        const int t = warp * 16 + lane;
        const int ct0 = (c0 + cw) * kChunk;
        const bool live = lane < 16 && t < Tlen - ct0;
        bf16 *dst = o + (((long)bi * Tlen + ct0 + t) * H + h) * (long)DV;
        const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16);
#pragma unroll
        for (int j = 0; j < DV; j += 32) {
            float a[16], b[16];
            tmem_ld16(lane_addr + j, a);
            tmem_ld16(lane_addr + j + 16, b);
            tmem_ld_wait();
            if (live) {
                *reinterpret_cast<uint4 *>(dst + j) = pack8(a);
                *reinterpret_cast<uint4 *>(dst + j + 8) = pack8(a + 8);
                *reinterpret_cast<uint4 *>(dst + j + 16) = pack8(b);
                *reinterpret_cast<uint4 *>(dst + j + 24) = pack8(b + 8);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, DV);
    }
}

template <int DV>
cudaError_t launch_out_impl(const FwdArgs &a, const uint8_t *ws, const uint8_t *sx, int c0, int ncw, int WC,
                            bool overlap)
{
    using L = OutLayout<DV>;
    auto kern = out_kernel<DV>;
    static std::atomic<unsigned long long> smem_set{0};
    cudaError_t e = ensure_smem_limit(kern, L::BYTES, smem_set);
    if (e != cudaSuccess) return e;
    LaunchCfg lc(dim3(ncw, a.H, a.B), dim3(kOutThreads), L::BYTES, a.stream, overlap);
    return cudaLaunchKernelEx(&lc.cfg, kern, ws, sx, (bf16 *)a.o, a.T, a.H, c0, WC, a.err);
}

}  // namespace

cudaError_t launch_out(const FwdArgs &a, const uint8_t *ws, const uint8_t *sx, int c0, int ncw, int WC, bool overlap)
{
    return a.dv == 128 ? launch_out_impl<128>(a, ws, sx, c0, ncw, WC, overlap)
                       : launch_out_impl<64>(a, ws, sx, c0, ncw, WC, overlap);
}

}  // namespace gdn2
