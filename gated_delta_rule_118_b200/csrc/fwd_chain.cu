// fwd_chain.cu -- the state-carrying part of the chunkwise forward (bf16 inputs).
//
// The chunks of a sequence are passed in order, the state of one chunk being
// the input of the next ("Gated DeltaNet-2", iplexlaw.co.kr, section
// "Procesamiento del token y entrenamiento paralelo").  With the prep records
// of fwd_prep.cu one chunk is an affine map of the state:
//   S <- e^{Gamma_C} S + D,    D = Y Z + NG Sx,    Sx = bf16(S)
// D is accumulated in tensor memory by two groups of tcgen05 UMMAs: Y Z (4
// instructions, M = dk, K = 64 tokens) does not depend on the state and is
// issued a chunk ahead; NG Sx (8 instructions, K = dk) is the only tensor-core
// work on the serial path.  The state stays fp32 in registers; its bf16 image
// Sx goes to shared memory (operand of the next UMMA) and to the workspace,
// where the output kernel reads it.
//
// One CTA owns one (batch, head, DVT-wide value tile); a whole 128-column tile
// costs the tensor core about as much per instruction as a narrow one, so wide
// tiles keep the number of SMs on the serial path small.  Warp roles:
//   warps 0-7  state: thread (i, half) owns key row i, columns [half*DVT/2, +DVT/2)
//   warp  8    producer: streams the records through a ring of shared stages
//   warp  9    MMA issuer (one elected lane)
#include "launch.h"
#include "tc_common.cuh"

namespace gdn2 {
namespace {

using namespace sm100;

constexpr int kChainThreads = 320;
constexpr int kStateThreads = 256;
constexpr int kSyncThreads = 288;  // state warps + MMA warp
constexpr int kDK = 128;

template <int DV, int DVT>
struct ChainLayout {
    static constexpr int NB = DVT / 64;                       // 64-column blocks in the tile
    static constexpr int HALF = DVT / 2;                      // columns per state thread
    // one stage: NG | Y | Z tile (NB blocks of [64 tokens][64 values])
    static constexpr int S_NG = 0, S_Y = 32768, S_Z = 49152;
    static constexpr int STAGE = S_Z + NB * 8192;
    static constexpr int SRB = NB * 16384;                    // one Sx buffer: NB blocks of [128][64]
    static constexpr int NSR = 3;                             // Sx buffers
    static constexpr int FIXED = NSR * SRB + 2048 + 1024;     // Sx buffers, decays, barriers, alignment
    static constexpr int NS = (4 * STAGE + 4 * 512 + FIXED <= 232448) ? 4
                              : (3 * STAGE + 3 * 512 + FIXED <= 232448) ? 3 : 2;  // ring depth
    static constexpr int SR = NS * STAGE;
    static constexpr int DECR = SR + NSR * SRB;               // [NS][128] fp32 e^{Gamma_C}
    static constexpr int BAR = DECR + NS * 512;
    static constexpr int NBAR = 2 * NS + 1;                   // full[NS], empty[NS], s_done
    static constexpr int SLOT = BAR + 8 * NBAR;
    static constexpr int BYTES = SLOT + 16 + 1024;
    static constexpr uint32_t TMEM_COLS = 2 * DVT;            // two D buffers
    static_assert(BYTES <= 232448, "shared memory");
    static_assert(STAGE % 1024 == 0 && SR % 1024 == 0 && SRB % 1024 == 0, "swizzle atoms");
};

template <int DV, int DVT>
__global__ void __launch_bounds__(kChainThreads, 1)
chain_kernel(const uint8_t *__restrict__ ws, uint8_t *__restrict__ sx_out, const float *S_in, float *S_out,
             int H, int ncw, int WC, unsigned int *err)
{
    using L = ChainLayout<DV, DVT>;
    using R = Record<DV>;
    constexpr int NS = L::NS, HALF = L::HALF, NB = L::NB, NSR = L::NSR;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int tile = blockIdx.x, h = blockIdx.y, bi = blockIdx.z;
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + L::BAR);
    uint64_t *full = bars, *empty = bars + NS, *s_done = bars + 2 * NS;
    uint32_t *slot = reinterpret_cast<uint32_t *>(sm + L::SLOT);
    const float *decr = reinterpret_cast<const float *>(sm + L::DECR);
    const uint32_t sbase = smem_u32(sm);
    const long pair = (long)bi * H + h;
    const uint8_t *recs = ws + pair * WC * (long)R::BYTES;
    uint8_t *sxs = sx_out + pair * WC * (long)SxSlot<DV>::BYTES;

    if (tid == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(full + s, 1);
            mbar_init(empty + s, 2);  // the state warps (decays read) and the tensor core (operands read)
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
                if (cw >= NS && !mbar_wait(empty + s, ((cw / NS) - 1) & 1, err)) break;
                uint8_t *st = sm + s * L::STAGE;
                const uint8_t *rec = recs + (long)cw * R::BYTES;
                mbar_arrive_expect_tx(full + s, (uint32_t)(L::STAGE + 512));
                bulk_load(st + L::S_NG, rec + R::NG, 32768, full + s);
                bulk_load(st + L::S_Y, rec + R::Y, 16384, full + s);
                bulk_load(st + L::S_Z, rec + R::Z + tile * NB * 8192, NB * 8192, full + s);
                bulk_load(sm + L::DECR + s * 512, rec + R::DEC, 512, full + s);
            }
        }
    } else if (warp == 9) {
        // ------------------------------------------------------------ MMA issuer
        const uint32_t idd = idesc_bf16(128, DVT, 0, 1);
        // descriptor start addresses are in 16-byte units: byte offsets >> 4 add directly
        const uint64_t ng0 = smem_desc(sbase + L::S_NG, 16, 1024, kSw128);
        const uint64_t y0 = smem_desc(sbase + L::S_Y, 16, 1024, kSw128);
        const uint64_t z0 = smem_desc(sbase + L::S_Z, 8192, 1024, kSw128);
        const uint64_t sx0 = smem_desc(sbase + L::SR, 16384, 1024, kSw128);
        bool ok = true;
        // D[cw & 1] = Y Z of chunk cw
        auto issue_yz = [&](int cw) {
            const int s = cw % NS;
            ok = ok && mbar_wait(full + s, (cw / NS) & 1, err);
            if (!ok) return;
            tc_fence_after();
            const uint64_t so = (uint64_t)((s * L::STAGE) >> 4);
            const uint32_t d = tmem + (uint32_t)((cw & 1) * DVT);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                umma_bf16(d, y0 + so + (uint64_t)((ks * 32) >> 4), z0 + so + (uint64_t)((ks * 2048) >> 4), idd, ks > 0);
        };
        if (lane == 0 && ncw > 0) issue_yz(0);
        for (int cw = 0; cw < ncw; ++cw) {
            named_bar(1, kSyncThreads);  // Sx(cw) is in its buffer; D[(cw + 1) & 1] has been read
            if (lane == 0) {
                tc_fence_after();
                const int s = cw % NS;
                const uint64_t so = (uint64_t)((s * L::STAGE) >> 4);
                const uint64_t bo = (uint64_t)(((cw % NSR) * L::SRB) >> 4);
                const uint32_t d = tmem + (uint32_t)((cw & 1) * DVT);
                if (ok) {
#pragma unroll
                    for (int ks = 0; ks < kDK / 16; ++ks)
                        umma_bf16(d, ng0 + so + (uint64_t)((((ks >> 2) * 16384) + (ks & 3) * 32) >> 4),
                                  sx0 + bo + (uint64_t)((ks * 2048) >> 4), idd, 1);
                }
                umma_commit(s_done);
                if (cw + NS < ncw) umma_commit(empty + s);
                if (cw + 1 < ncw) issue_yz(cw + 1);
            }
            __syncwarp();
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
        // Sx(cw) lives in buffer cw % NSR, already in the layout of the exported slot.
        auto write_sx = [&](int cw) {
            uint8_t *sr = sm + L::SR + (cw % NSR) * L::SRB;
#pragma unroll
            for (int j = 0; j < HALF; j += 8) {
                const int c = col0 + j;
                *reinterpret_cast<uint4 *>(sr + (c >> 6) * 16384 + swz_off(i, (c & 63) * 2, 128)) = pack8(S + j);
            }
        };
        // e^{Gamma_C} of chunk cw for this row, once its stage has landed (after a
        // wait has given up, the rest of the walk only runs to its end)
        bool live = true;
        auto decay = [&](int cw) {
            live = live && mbar_wait(full + cw % NS, (cw / NS) & 1, err);
            return decr[(cw % NS) * 128 + i];
        };
        float gc = 1.f;
        if (ncw > 0) {
            write_sx(0);
            gc = decay(0);
        }
        fence_proxy_async_smem();
        for (int cw = 0; cw < ncw; ++cw) {
            const int s = cw % NS;
            named_bar(1, kSyncThreads);  // every state thread has read the decays of chunk cw
            if (tid == 0) {
                if (cw + NS < ncw) mbar_arrive(empty + s);
                // one thread copies the whole buffer to the workspace (blocks of this tile only)
                bulk_store(sxs + (long)cw * SxSlot<DV>::BYTES + tile * NB * 16384, sm + L::SR + (cw % NSR) * L::SRB,
                           (uint32_t)L::SRB);
                bulk_commit();
            }
            mbar_wait(s_done, cw & 1, err);
            tc_fence_after();
            {
                const uint32_t dcol = (uint32_t)((cw & 1) * DVT);
#pragma unroll
                for (int j = 0; j < HALF; j += 32) {
                    float d0[16], d1[16];
                    tmem_ld16(lane_addr + dcol + j, d0);
                    tmem_ld16(lane_addr + dcol + j + 16, d1);
                    tmem_ld_wait();
#pragma unroll
                    for (int u = 0; u < 16; ++u) {
                        S[j + u] = gc * S[j + u] + d0[u];
                        S[j + 16 + u] = gc * S[j + 16 + u] + d1[u];
                    }
                }
            }
            if (cw + 1 < ncw) {
                write_sx(cw + 1);
                gc = decay(cw + 1);
            }
            fence_proxy_async_smem();
            tc_fence_before();
            // the buffer written next iteration was exported two chunks ago: that copy
            // must have finished reading it (only the latest export may still be running)
            if (tid == 0) asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
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
cudaError_t launch_chain_impl(const FwdArgs &a, const uint8_t *ws, uint8_t *sx, const float *S_in, float *S_out,
                              int ncw, int WC)
{
    using L = ChainLayout<DV, DVT>;
    auto kern = chain_kernel<DV, DVT>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::BYTES);
    if (e != cudaSuccess) return e;
    dim3 grid(DV / DVT, a.H, a.B);
    kern<<<grid, kChainThreads, L::BYTES, a.stream>>>(ws, sx, S_in, S_out, a.H, ncw, WC, a.err);
    return cudaGetLastError();
}

cudaError_t launch_chain(const FwdArgs &a, int dvt, const uint8_t *ws, uint8_t *sx, const float *S_in,
                         float *S_out, int ncw, int WC)
{
    if (a.dv == 128) {
        if (dvt == 128) return launch_chain_impl<128, 128>(a, ws, sx, S_in, S_out, ncw, WC);
        return launch_chain_impl<128, 64>(a, ws, sx, S_in, S_out, ncw, WC);
    }
    return launch_chain_impl<64, 64>(a, ws, sx, S_in, S_out, ncw, WC);
}

}  // namespace gdn2
