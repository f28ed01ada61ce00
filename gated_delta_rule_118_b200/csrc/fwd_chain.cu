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
//   warps 0-7  state: thread (i, g) owns key row i, columns [g*COLS, +COLS)
//   warp  8    issues NG Sx (one elected lane)
//   warp  9    producer: streams the records through a ring of shared stages
//   warp  10   issues Y Z (one elected lane)
// The serial path per chunk is: UMMA completion -> tensor-memory load and state
// update -> Sx to shared memory -> one mbarrier arrival per state warp -> UMMA
// issue.  Everything else (the Sx export, stage refills, the next Y Z) runs
// beside it; the decays come straight from L2 into registers three chunks ahead,
// so the state warps never wait for a stage (a stage takes microseconds to land).  Issuing a UMMA blocks the issuing thread while the
// tensor pipe is busy, so the two groups of UMMAs come from different warps,
// ordered by mbarriers: NG Sx of chunk c issued -> Y Z of chunk c + 1 (queued
// right behind it, it runs beside the epilogue of chunk c) -> Y Z done ->
// NG Sx of chunk c + 1.
#include "launch.h"
#include "tc_common.cuh"

namespace gdn2 {
namespace {

using namespace sm100;

constexpr int kStateWarps = 8;
constexpr int kMmaWarp = kStateWarps, kProducerWarp = kStateWarps + 1, kYzWarp = kStateWarps + 2;
constexpr int kChainThreads = 32 * (kStateWarps + 3);
constexpr int kDK = 128;

template <int DV, int DVT>
struct ChainLayout {
    static constexpr int NB = DVT / 64;                       // 64-column blocks of Z in the tile
    static constexpr int COLS = DVT / (kStateWarps / 4);      // columns per state thread
    // one stage: NG | Y | Z tile (NB blocks of [64 tokens][64 values])
    static constexpr int S_NG = 0, S_Y = 32768, S_Z = 49152;
    static constexpr int STAGE = S_Z + NB * 8192;
    // Sx buffer: [128][DVT], no swizzle.  One is enough: Sx of chunk c + 1 is
    // written after the UMMA that read Sx of chunk c has completed.
    static constexpr int SRB = DVT * 256;
    static constexpr int FIXED = SRB + 2048 + 1024;           // Sx buffer, barriers, alignment
    static constexpr int NS = (4 * STAGE + FIXED <= 232448) ? 4 : (3 * STAGE + FIXED <= 232448) ? 3 : 2;
    static constexpr int SR = NS * STAGE;
    static constexpr int BAR = SR + SRB;
    static constexpr int NBAR = 2 * NS + 5;  // full[NS], empty[NS], s_done, sx_full, yz_done[2], s_issued
    static constexpr int SLOT = BAR + 8 * NBAR;
    static constexpr int BYTES = SLOT + 16 + 1024;
    static constexpr uint32_t TMEM_COLS = 2 * DVT;            // two D buffers
    static_assert(BYTES <= 232448, "shared memory");
    static_assert(STAGE % 1024 == 0 && SR % 1024 == 0, "swizzle atoms");
};

template <int DV, int DVT>
__global__ void __launch_bounds__(kChainThreads, 1)
chain_kernel(const uint8_t *__restrict__ ws, uint8_t *__restrict__ sx_out, const float *S_in, float *S_out,
             int H, int ncw, int WC, unsigned int *err)
{
    using L = ChainLayout<DV, DVT>;
    using R = Record<DV>;
    constexpr int NS = L::NS, COLS = L::COLS, NB = L::NB;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int tile = blockIdx.x, h = blockIdx.y, bi = blockIdx.z;
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + L::BAR);
    uint64_t *full = bars, *empty = bars + NS, *s_done = bars + 2 * NS, *sx_full = bars + 2 * NS + 1;
    uint64_t *yz_done = bars + 2 * NS + 2, *s_issued = bars + 2 * NS + 4;
    uint32_t *slot = reinterpret_cast<uint32_t *>(sm + L::SLOT);
    const uint32_t sbase = smem_u32(sm);
    const long pair = (long)bi * H + h;
    const uint8_t *recs = ws + pair * WC * (long)R::BYTES;
    uint8_t *sxs = sx_out + pair * WC * (long)SxSlot<DV>::BYTES;

    if (tid == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(full + s, 1);
            mbar_init(empty + s, 1);  // the tensor core has read the stage's operands
        }
        mbar_init(s_done, 1);
        mbar_init(sx_full, kStateWarps);
        for (int b = 0; b < 2; ++b) mbar_init(yz_done + b, 1);
        mbar_init(s_issued, 1);
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
    // This window's chain is resident: the next window's prep may take the other
    // SMs.  Then wait for this window's prep (its records, and through its own
    // final wait the previous chain and the state it carries).
    allow_dependent_launch();
    wait_prior_grid();

    if (warp == kProducerWarp) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            for (int cw = 0; cw < ncw; ++cw) {
                const int s = cw % NS;
                if (cw >= NS && !mbar_wait(empty + s, ((cw / NS) - 1) & 1, err)) break;
                uint8_t *st = sm + s * L::STAGE;
                const uint8_t *rec = recs + (long)cw * R::BYTES;
                mbar_arrive_expect_tx(full + s, (uint32_t)L::STAGE);
                bulk_load(st + L::S_NG, rec + R::NG, 32768, full + s);
                bulk_load(st + L::S_Y, rec + R::Y, 16384, full + s);
                bulk_load(st + L::S_Z, rec + R::Z + tile * NB * 8192, NB * 8192, full + s);
            }
        }
    } else if (warp == kYzWarp) {
        // ------------------------------------------------------------ Y Z issuer
        if (lane == 0) {
            const uint32_t idd = idesc_bf16(128, DVT, 0, 1);
            const uint64_t y0 = smem_desc(sbase + L::S_Y, 2048, 128, kSwNone);  // no-swizzle K chunks of 128 rows
            const uint64_t z0 = smem_desc(sbase + L::S_Z, 8192, 1024, kSw128);
            bool ok = true;
            for (int cw = 0; cw < ncw; ++cw) {
                const int s = cw % NS, b = cw & 1;
                ok = ok && mbar_wait(full + s, (cw / NS) & 1, err);
                // right behind NG Sx of chunk cw - 1, whose issue also means that
                // the epilogue of chunk cw - 2 has read D[b]
                if (cw >= 1) ok = ok && mbar_wait(s_issued, (cw - 1) & 1, err);
                tc_fence_after();
                if (ok) {
                    const uint64_t so = (uint64_t)((s * L::STAGE) >> 4);
                    const uint32_t d = tmem + (uint32_t)(b * DVT);
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
                        umma_bf16(d, y0 + so + (uint64_t)((ks * 4096) >> 4), z0 + so + (uint64_t)((ks * 2048) >> 4),
                                  idd, ks > 0);
                }
                umma_commit(yz_done + b);
            }
        }
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ NG Sx issuer
        if (lane == 0) {
            const uint32_t idd = idesc_bf16(128, DVT, 0, 1);
            // descriptor start addresses are in 16-byte units: byte offsets >> 4 add directly
            const uint64_t ng0 = smem_desc(sbase + L::S_NG, 2048, 128, kSwNone);
            const uint64_t sx0 = smem_desc(sbase + L::SR, 128, 2048, kSwNone);   // MN-major, 8-row K groups
            bool ok = true;
            for (int cw = 0; cw < ncw; ++cw) {
                const int s = cw % NS, b = cw & 1;
                // Sx(cw) is in its buffer and D[(cw + 1) & 1] has been read
                ok = ok && mbar_wait(sx_full, cw & 1, err);
                ok = ok && mbar_wait(yz_done + b, (cw >> 1) & 1, err);
                tc_fence_after();
                if (ok) {
                    const uint64_t so = (uint64_t)((s * L::STAGE) >> 4);
                    const uint32_t d = tmem + (uint32_t)(b * DVT);
#pragma unroll
                    for (int ks = 0; ks < kDK / 16; ++ks)
                        umma_bf16(d, ng0 + so + (uint64_t)((ks * 4096) >> 4), sx0 + (uint64_t)((ks * 256) >> 4), idd, 1);
                }
                umma_commit(s_done);
                if (cw + NS < ncw) umma_commit(empty + s);
                mbar_arrive(s_issued);
            }
        }
    } else {
        // ------------------------------------------------------------ state
        const int i = tid & 127, grp = tid >> 7;
        const int col0 = grp * COLS;  // first column (within the tile) of this thread
        const uint32_t lane_addr = tmem + ((uint32_t)((warp & 3) * 32) << 16) + col0;
        float S[COLS];
#pragma unroll
        for (int j = 0; j < COLS; ++j) S[j] = 0.f;
        if (S_in) {
            const float *src = S_in + (pair * kDK + i) * DV + tile * DVT + col0;
#pragma unroll
            for (int j = 0; j < COLS; j += 4) {
                const float4 v4 = *reinterpret_cast<const float4 *>(src + j);
                S[j] = v4.x; S[j + 1] = v4.y; S[j + 2] = v4.z; S[j + 3] = v4.w;
            }
        }
        // Sx(cw) -> the Sx buffer (the next UMMA's operand), signal the MMA warp,
        // then copy the same 16-byte pieces to the exported slot (every warp store
        // covers 512 contiguous bytes).
        auto publish_sx = [&](int cw) {
            uint4 px[COLS / 8];
#pragma unroll
            for (int j = 0; j < COLS; j += 8) px[j / 8] = pack8(S + j);
            uint8_t *sr = sm + L::SR;
#pragma unroll
            for (int j = 0; j < COLS; j += 8) *reinterpret_cast<uint4 *>(sr + sx_off(i, col0 + j)) = px[j / 8];
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(sx_full);
            uint8_t *dst = sxs + (long)cw * SxSlot<DV>::BYTES;
#pragma unroll
            for (int j = 0; j < COLS; j += 8)
                *reinterpret_cast<uint4 *>(dst + sx_off(i, tile * DVT + col0 + j)) = px[j / 8];
        };
        // e^{Gamma_C} of chunk cw for this row, read from the record three chunks ahead
        auto decay = [&](int cw) {
            return cw < ncw ? __ldg(reinterpret_cast<const float *>(recs + (long)cw * R::BYTES + R::DEC) + i) : 1.f;
        };
        float gc = decay(0), g1 = decay(1), g2 = decay(2);
        if (ncw > 0) publish_sx(0);
        for (int cw = 0; cw < ncw; ++cw) {
            const float gn = g1;
            g1 = g2;
            g2 = decay(cw + 3);
            mbar_wait(s_done, cw & 1, err);
            tc_fence_after();
            {
                float d[COLS];
                const uint32_t da = lane_addr + (uint32_t)((cw & 1) * DVT);
                if constexpr (COLS % 32 == 0) {
#pragma unroll
                    for (int j = 0; j < COLS; j += 32) tmem_ld32(da + j, *reinterpret_cast<float(*)[32]>(d + j));
                } else {
#pragma unroll
                    for (int j = 0; j < COLS; j += 16) tmem_ld16(da + j, *reinterpret_cast<float(*)[16]>(d + j));
                }
                tmem_ld_wait();
#pragma unroll
                for (int u = 0; u < COLS; ++u) S[u] = gc * S[u] + d[u];
            }
            gc = gn;
            if (cw + 1 < ncw) publish_sx(cw + 1);
        }
        if (S_out) {
            float *dst = S_out + (pair * kDK + i) * DV + tile * DVT + col0;
#pragma unroll
            for (int j = 0; j < COLS; j += 4)
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
