// fwd_chain.cu -- the state-carrying part of the chunkwise forward (bf16 inputs).
//
// The chunks of a sequence are passed in order, the state of one chunk being
// the input of the next ("Gated DeltaNet-2", iplexlaw.co.kr, section
// "Procesamiento del token y entrenamiento paralelo").  With the prep records
// of fwd_prep.cu (G, N and the decays of each chunk) one chunk is an affine map
// of the state:
//   Sref = e^{Gamma_r} S
//   S   <- e^{Gamma_C} S + N - G Sref          (one tcgen05 UMMA, M = dk = 128)
// so the serial path through the sequence is one tensor-core round trip per
// chunk: 8 UMMA instructions (K = 16 each) and one epilogue.  The state stays
// fp32 in registers; its bf16 image Sref goes to shared memory (the next
// UMMA's operand) and to the workspace, where the output kernel reads it.
//
// One CTA owns one (batch, head, DVT-wide value tile); a whole 128-column tile
// costs the tensor core about as much per instruction as a narrow one, so wide
// tiles keep the number of SMs on the serial path small.  Warp roles:
//   warps 0-7  state: thread (i, half) owns key row i, columns [half*DVT/2, +DVT/2)
//   warp  8    producer: streams the records through a ring of shared stages
#include "launch.h"
#include "tc_common.cuh"

namespace gdn2 {
namespace {

using namespace sm100;

constexpr int kChainThreads = 288;
constexpr int kStateThreads = 256;
constexpr int kDK = 128;

template <int DV, int DVT>
struct ChainLayout {
    static constexpr int NB = DVT / 64;                       // 64-column blocks in the tile
    static constexpr int HALF = DVT / 2;                      // columns per state thread
    // one stage: GC | NC tile (NB blocks of [128][64], 128-byte swizzle) | DEC
    static constexpr int S_GC = 0, S_NC = 32768;
    static constexpr int S_DEC = S_NC + NB * 16384;
    static constexpr int STAGE_TX = S_DEC + 1024;
    static constexpr int STAGE = align_up(STAGE_TX, 1024);
    static constexpr int SRB = NB * 16384;                    // one Sref buffer
    static constexpr int NS = (4 * STAGE + 2 * SRB + 2048 <= 232448) ? 4
                              : (3 * STAGE + 2 * SRB + 2048 <= 232448) ? 3 : 2;  // ring depth
    static constexpr int SR = NS * STAGE;                     // two Sref buffers, NB blocks of [128][64] each
    static constexpr int BAR = SR + 2 * SRB;
    static constexpr int NBAR = 2 * NS + 1;                   // full[NS], empty[NS], s_done
    static constexpr int SLOT = BAR + 8 * NBAR;
    static constexpr int BYTES = SLOT + 16 + 1024;
    static constexpr uint32_t TMEM_COLS = DVT < 32 ? 32 : DVT;
    static_assert(BYTES <= 232448, "shared memory");
};

template <int DV, int DVT>
__global__ void __launch_bounds__(kChainThreads, 1)
chain_kernel(const uint8_t *__restrict__ ws, uint8_t *__restrict__ sref_out, const float *S_in, float *S_out,
             int H, int ncw, int WC, unsigned int *err)
{
    using L = ChainLayout<DV, DVT>;
    using R = Record<DV>;
    constexpr int NS = L::NS, HALF = L::HALF, NB = L::NB;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int tile = blockIdx.x, h = blockIdx.y, bi = blockIdx.z;
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + L::BAR);
    uint64_t *full = bars, *empty = bars + NS, *s_done = bars + 2 * NS;
    uint32_t *slot = reinterpret_cast<uint32_t *>(sm + L::SLOT);
    const uint32_t sbase = smem_u32(sm);
    const long pair = (long)bi * H + h;
    const uint8_t *recs = ws + pair * WC * (long)R::BYTES;
    uint8_t *srefs = sref_out + pair * WC * (long)SrefSlot<DV>::BYTES;

    if (tid == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(full + s, 1);
            mbar_init(empty + s, 1);
        }
        mbar_init(s_done, 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(slot, L::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *slot;

    if (warp == 8) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            for (int cw = 0; cw < ncw; ++cw) {
                const int s = cw % NS;
                if (cw >= NS) mbar_wait(empty + s, ((cw / NS) - 1) & 1, err);
                uint8_t *st = sm + s * L::STAGE;
                const uint8_t *rec = recs + (long)cw * R::BYTES;
                mbar_arrive_expect_tx(full + s, (uint32_t)L::STAGE_TX);
                bulk_load(st + L::S_GC, rec + R::GC, 32768, full + s);
                bulk_load(st + L::S_NC, rec + R::NC + tile * NB * 16384, NB * 16384, full + s);
                bulk_load(st + L::S_DEC, rec + R::DEC, 1024, full + s);
            }
        }
    } else {
        // ------------------------------------------------------------ state
        const int i = tid & 127, half = tid >> 7;
        const int col0 = half * HALF;  // first column (within the tile) of this thread
        const uint32_t lane_addr = tmem + ((uint32_t)((warp & 3) * 32) << 16) + col0;
        float S[HALF];
#pragma unroll
        for (int j = 0; j < HALF; ++j) S[j] = 0.f;
        if (S_in) {
            const float *src = S_in + (pair * kDK + i) * DV + tile * DVT + col0;
#pragma unroll
            for (int j = 0; j < HALF; j += 4) {
                const float4 v4 = *reinterpret_cast<const float4 *>(src + j);
                S[j] = v4.x; S[j + 1] = v4.y; S[j + 2] = v4.z; S[j + 3] = v4.w;
            }
        }
        // Sref of chunk cw: written to shared memory (operand of the next UMMA) on
        // the serial path, then exported to the workspace for the output kernel
        // while that UMMA runs.
        auto sref_pack = [&](int cw, int j) {
            const float egr = reinterpret_cast<const float *>(sm + (cw % NS) * L::STAGE + L::S_DEC)[kDK + i];
            float f[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) f[u] = egr * S[j + u];
            return pack8(f);
        };
        // Sref(cw) lives in buffer cw & 1, already in the layout of the exported slot.
        auto write_sref = [&](int cw) {
            uint8_t *sr = sm + L::SR + (cw & 1) * L::SRB;
#pragma unroll
            for (int j = 0; j < HALF; j += 8) {
                const int c = col0 + j;
                *reinterpret_cast<uint4 *>(sr + (c >> 6) * 16384 + swz_off(i, (c & 63) * 2, 128)) = sref_pack(cw, j);
            }
        };
        // One thread copies the whole buffer to the workspace (blocks of this tile only).
        auto export_sref = [&](int cw) {
            bulk_store(srefs + (long)cw * SrefSlot<DV>::BYTES + tile * NB * 16384, sm + L::SR + (cw & 1) * L::SRB,
                       (uint32_t)L::SRB);
            bulk_commit();
        };
        if (ncw > 0) {
            mbar_wait(full, 0, err);
            write_sref(0);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        named_bar(1, kStateThreads);
        // UMMA descriptors (start addresses are in 16-byte units, so offsets add directly)
        const uint64_t bdesc0 = smem_desc(sbase + L::SR, 16384, 1024, kSw128);
        const uint64_t adesc0 = smem_desc(sbase + L::S_GC, 16, 1024, kSw128);

        const uint32_t ids = idesc_bf16(128, DVT, 0, 1);
        for (int cw = 0; cw < ncw; ++cw) {
            const int s = cw % NS;
            const uint8_t *st = sm + s * L::STAGE;
            if (tid == 0) {
                tc_fence_after();
                // descriptor start addresses are in 16-byte units: offsets add directly
                const uint64_t ga = adesc0 + (uint64_t)((s * L::STAGE) >> 4);
                const uint64_t gb = bdesc0 + (uint64_t)(((cw & 1) * L::SRB) >> 4);
#pragma unroll
                for (int ks = 0; ks < kDK / 16; ++ks)
                    umma_bf16(tmem, ga + (uint64_t)((((ks >> 2) * 16384) + (ks & 3) * 32) >> 4),
                              gb + (uint64_t)((ks * 2048) >> 4), ids, ks > 0);
                umma_commit(s_done);
                export_sref(cw);
            }
            mbar_wait(s_done, cw & 1, err);
            tc_fence_after();
            {
                const float gci = reinterpret_cast<const float *>(st + L::S_DEC)[i];
                const uint8_t *nc = st + L::S_NC;
#pragma unroll
                for (int j = 0; j < HALF; j += 16) {
                    float gs[16], n[16];
                    tmem_ld16(lane_addr + j, gs);
                    const int c = col0 + j;
                    const uint8_t *nb = nc + (c >> 6) * 16384;
                    unpack8(*reinterpret_cast<const uint4 *>(nb + swz_off(i, (c & 63) * 2, 128)), n);
                    unpack8(*reinterpret_cast<const uint4 *>(nb + swz_off(i, (c & 63) * 2 + 16, 128)), n + 8);
                    tmem_ld_wait();
#pragma unroll
                    for (int u = 0; u < 16; ++u) S[j + u] = gci * S[j + u] + n[u] - gs[u];
                }
            }
            if (cw + 1 < ncw) {
                mbar_wait(full + (cw + 1) % NS, ((cw + 1) / NS) & 1, err);
                write_sref(cw + 1);
            }
            fence_proxy_async_smem();
            tc_fence_before();
            // the export of Sref(cw - 1) read the buffer that the next iteration rewrites
            if (tid == 0) bulk_wait_read_all();
            named_bar(1, kStateThreads);
            if (tid == 0) mbar_arrive(empty + s);
        }
        if (tid == 0) bulk_wait_all();
        if (S_out) {
            float *dst = S_out + (pair * kDK + i) * DV + tile * DVT + col0;
#pragma unroll
            for (int j = 0; j < HALF; j += 4)
                *reinterpret_cast<float4 *>(dst + j) = make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, L::TMEM_COLS);
    }
}

}  // namespace

template <int DV, int DVT>
cudaError_t launch_chain_impl(const FwdArgs &a, const uint8_t *ws, uint8_t *sref, const float *S_in, float *S_out,
                              int ncw, int WC)
{
    using L = ChainLayout<DV, DVT>;
    auto kern = chain_kernel<DV, DVT>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::BYTES);
    if (e != cudaSuccess) return e;
    dim3 grid(DV / DVT, a.H, a.B);
    kern<<<grid, kChainThreads, L::BYTES, a.stream>>>(ws, sref, S_in, S_out, a.H, ncw, WC, a.err);
    return cudaGetLastError();
}

cudaError_t launch_chain(const FwdArgs &a, int dvt, const uint8_t *ws, uint8_t *sref, const float *S_in,
                         float *S_out, int ncw, int WC)
{
    if (a.dv == 128) {
        if (dvt == 128) return launch_chain_impl<128, 128>(a, ws, sref, S_in, S_out, ncw, WC);
        return launch_chain_impl<128, 64>(a, ws, sref, S_in, S_out, ncw, WC);
    }
    return launch_chain_impl<64, 64>(a, ws, sref, S_in, S_out, ncw, WC);
}

}  // namespace gdn2
