// fwd_chain_out.cu -- the windowed chain with the chunk outputs computed in the
// same CTA, for wide batches (chains on most SMs, prep and chain taking turns).
//
// Per chunk c the tensor core runs, in issue order, NG Sx(c) into D[c & 1] (the
// serial product of chain_body.cuh), the next chunk's Y Z, and the outputs
//   O(c) = PT Z + QS Sx(c)       (M = 64 tokens, N = DVT; K = 64, then K = dk)
// into O[c & 1], from the same state image Sx(c) in shared memory ("Gated
// DeltaNet-2", iplexlaw.co.kr, section "Decisiones independientes en dos ejes":
// the query reads the updated state).  The window's outputs need no kernel of
// their own, and the state images never leave the SM: the records' QS and PT
// ride in each stage beside NG, Y and Z.
//
// One state-image buffer: Sx(c + 1) is written once the output products of
// chunk c, which read Sx(c), have completed (the serial path gains their
// duration, the window loses its output pass).  Warps:
//   0-7   state: thread (i, g) owns key row i, columns [g COLS, +COLS)
//   8     NG Sx, then the outputs (one lane)
//   9     producer: the records through a ring of two shared stages
//   10    Y Z (one lane)
//   12-15 output writers (tensor-memory lane quarters 0-3)
#include "launch.h"
#include "tc_common.cuh"

namespace gdn2 {
namespace chainout {

using namespace sm100;

constexpr int kStateWarps = 8;
constexpr int kMmaWarp = 8, kProducerWarp = 9, kYzWarp = 10, kOutWarp0 = 12;
constexpr int kThreads = 512;
constexpr int kDK = 128;

template <int DV, int DVT>
struct Layout {
    static constexpr int NB = DVT / 64;                    // 64-column blocks of Z in the tile
    static constexpr int COLS = DVT / (kStateWarps / 4);   // columns per state thread
    // one stage: NG | Y | QS | PT | Z tile; the stage's decays in an array of their own
    static constexpr int S_NG = 0, S_Y = 32768, S_QS = 49152, S_PT = 65536, S_Z = 73728;
    static constexpr int STAGE = S_Z + NB * 8192;
    static constexpr int NS = 2;
    static constexpr int SRB = DVT * 256;                   // the state image [128][DVT]
    static constexpr int DEC_BYTES = kDK * 4;
    static constexpr int SR = NS * STAGE;
    static constexpr int DECR = SR + SRB;
    static constexpr int BAR = DECR + NS * DEC_BYTES;
    // full[NS], empty[NS], s_done, sx_full, yz_done[2], s_issued, o_done[2], o_free[2]
    static constexpr int NBAR = 2 * NS + 9;
    static constexpr int SLOT = BAR + 8 * NBAR;            // tensor-memory address
    static constexpr int DATA = SLOT + 16;
    static constexpr int BYTES = DATA + 1024;
    static constexpr uint32_t TMEM_COLS = 4 * DVT;         // D[2], O[2]
    static_assert(BYTES <= 232448, "shared memory");
    static_assert(STAGE % 1024 == 0 && SR % 1024 == 0, "swizzle atoms");
    static_assert(COLS % 32 == 0, "whole 32-column tensor-memory loads");
};

template <int DV, int DVT>
__global__ void __launch_bounds__(kThreads, 1)
chain_out_kernel(const uint8_t *__restrict__ ws, const float *S_in, float *S_out, bf16 *__restrict__ o, int Tlen,
                 int H, int c0, int ncw, int WC, unsigned int *err)
{
    using L = Layout<DV, DVT>;
    using R = Record<DV>;
    constexpr int NS = L::NS, COLS = L::COLS, NB = L::NB;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int tile = blockIdx.x, h = blockIdx.y, bi = blockIdx.z;
    const long pair = (long)bi * H + h;
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + L::BAR);
    uint64_t *full = bars, *empty = bars + NS, *s_done = bars + 2 * NS, *sx_full = bars + 2 * NS + 1;
    uint64_t *yz_done = bars + 2 * NS + 2, *s_issued = bars + 2 * NS + 4;
    uint64_t *o_done = bars + 2 * NS + 5, *o_free = bars + 2 * NS + 7;
    uint32_t *slot = reinterpret_cast<uint32_t *>(sm + L::SLOT);
    const uint32_t sbase = smem_u32(sm);
    const uint8_t *recs = ws + pair * WC * (long)R::BYTES;

    if (tid == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(full + s, 1);                      // the producer's bytes
            mbar_init(empty + s, 1 + kStateWarps);       // the UMMAs (one commit) and every state warp
        }
        mbar_init(s_done, 1);
        mbar_init(sx_full, kStateWarps);
        for (int b = 0; b < 2; ++b) {
            mbar_init(yz_done + b, 1);
            mbar_init(o_done + b, 1);
            mbar_init(o_free + b, 4);                    // the four writer warps
        }
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
    // the window's prep (its records, and through its own final wait the
    // previous chain and the state it carries)
    wait_prior_grid();
    const uint32_t d_cols = 0, o_cols = 2 * DVT;  // D[b] at b DVT, O[b] at 2 DVT + b DVT

    if (warp == kProducerWarp) {
        if (lane == 0) {
            int issued = 0;
            for (int cw = 0; cw < ncw; ++cw) {
                const int s = cw % NS;
                if (cw >= NS && !mbar_wait(empty + s, ((cw / NS) - 1) & 1, err)) break;
                uint8_t *st = sm + s * L::STAGE;
                const uint8_t *rec = recs + (long)cw * R::BYTES;
                mbar_arrive_expect_tx(full + s, (uint32_t)(L::STAGE + L::DEC_BYTES));
                bulk_load(st + L::S_NG, rec + R::NG, 32768, full + s);
                bulk_load(st + L::S_Y, rec + R::Y, 16384, full + s);
                bulk_load(st + L::S_QS, rec + R::QS, 16384, full + s);
                bulk_load(st + L::S_PT, rec + R::PT, 8192, full + s);
                bulk_load(st + L::S_Z, rec + R::Z + tile * NB * 8192, NB * 8192, full + s);
                bulk_load(sm + L::DECR + s * L::DEC_BYTES, rec + R::DEC, L::DEC_BYTES, full + s);
                issued = cw + 1;
            }
            // copies in flight land before the CTA may leave
            for (int c = issued > NS ? issued - NS : 0; c < issued; ++c) mbar_wait(full + c % NS, (c / NS) & 1, err);
        }
    } else if (warp == kYzWarp) {
        if (lane == 0) {
            const uint32_t idd = idesc_bf16(128, DVT, 0, 1);
            const uint64_t y0 = smem_desc(sbase + L::S_Y, 2048, 128, kSwNone);
            const uint64_t z0 = smem_desc(sbase + L::S_Z, 8192, 1024, kSw128);
            bool ok = true;
            for (int cw = 0; cw < ncw; ++cw) {
                const int s = cw % NS, b = cw & 1;
                ok = ok && mbar_wait(full + s, (cw / NS) & 1, err);
                // right behind NG Sx of chunk cw - 1, whose issue also means that the
                // state warps have read D[b] of chunk cw - 2
                if (cw >= 1) ok = ok && mbar_wait(s_issued, (cw - 1) & 1, err);
                tc_fence_after();
                if (ok) {
                    const uint64_t so = (uint64_t)((s * L::STAGE) >> 4);
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
                        umma_bf16(tmem + d_cols + (uint32_t)(b * DVT), y0 + so + (uint64_t)((ks * 4096) >> 4),
                                  z0 + so + (uint64_t)((ks * 2048) >> 4), idd, ks > 0);
                }
                umma_commit(yz_done + b);
            }
        }
    } else if (warp == kMmaWarp) {
        if (lane == 0) {
            const uint32_t idd = idesc_bf16(128, DVT, 0, 1), ido = idesc_bf16(64, DVT, 0, 1);
            const uint64_t ng0 = smem_desc(sbase + L::S_NG, 2048, 128, kSwNone);
            const uint64_t qs0 = smem_desc(sbase + L::S_QS, 1024, 128, kSwNone);
            const uint64_t pt0 = smem_desc(sbase + L::S_PT, 1024, 128, kSwNone);
            const uint64_t z0 = smem_desc(sbase + L::S_Z, 8192, 1024, kSw128);
            const uint64_t sx0 = smem_desc(sbase + L::SR, 128, 2048, kSwNone);
            bool ok = true;
            for (int cw = 0; cw < ncw; ++cw) {
                const int s = cw % NS, b = cw & 1;
                ok = ok && mbar_wait(sx_full, cw & 1, err);
                ok = ok && mbar_wait(yz_done + b, (cw >> 1) & 1, err);
                tc_fence_after();
                const uint64_t so = (uint64_t)((s * L::STAGE) >> 4);
                if (ok) {
#pragma unroll
                    for (int ks = 0; ks < kDK / 16; ++ks)
                        umma_bf16(tmem + d_cols + (uint32_t)(b * DVT), ng0 + so + (uint64_t)((ks * 4096) >> 4),
                                  sx0 + (uint64_t)((ks * 256) >> 4), idd, 1);
                }
                umma_commit(s_done);
                mbar_arrive(s_issued);
                // the outputs of chunk cw into O[b], once the writers have read O[b] of chunk cw - 2
                if (cw >= 2) ok = ok && mbar_wait(o_free + b, ((cw >> 1) - 1) & 1, err);
                tc_fence_after();
                if (ok) {
                    const uint32_t od = tmem + o_cols + (uint32_t)(b * DVT);
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
                        umma_bf16(od, pt0 + so + (uint64_t)((ks * 2048) >> 4), z0 + so + (uint64_t)((ks * 2048) >> 4),
                                  ido, ks > 0);
#pragma unroll
                    for (int ks = 0; ks < kDK / 16; ++ks)
                        umma_bf16(od, qs0 + so + (uint64_t)((ks * 2048) >> 4), sx0 + (uint64_t)((ks * 256) >> 4),
                                  ido, 1);
                }
                // o_done: the outputs are in O[b] and Sx(cw) is free; empty: stage s is read
                umma_commit(o_done + b);
                if (cw + NS < ncw) umma_commit(empty + s);
            }
        }
    } else if (warp >= kOutWarp0) {
        // M = 64 accumulator: token 16 q + l sits in tensor-memory lane 32 q + l (l < 16)
        const int q = warp & 3;
        const uint32_t lane_base = tmem + ((uint32_t)(q * 32) << 16) + o_cols;
        bool ok = true;
        for (int cw = 0; cw < ncw; ++cw) {
            const int b = cw & 1, t = q * 16 + lane, t0 = (c0 + cw) * kChunk;
            ok = ok && mbar_wait(o_done + b, (cw >> 1) & 1, err);
            tc_fence_after();
            const bool on = ok && lane < 16 && t < Tlen - t0;
            bf16 *row = o + (((long)bi * Tlen + t0 + t) * H + h) * (long)DV + tile * DVT;
#pragma unroll
            for (int j = 0; j < DVT; j += 32) {
                float a[32];
                tmem_ld32(lane_base + (uint32_t)(b * DVT + j), a);
                tmem_ld_wait();
                if (on) {
#pragma unroll
                    for (int u = 0; u < 32; u += 8) *reinterpret_cast<uint4 *>(row + j + u) = pack8(a + u);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(o_free + b);
        }
    } else if (warp < kStateWarps) {
        const int i = tid & 127, grp = tid >> 7;
        const int col0 = grp * COLS;
        const uint32_t lane_addr = tmem + ((uint32_t)((warp & 3) * 32) << 16) + d_cols + col0;
        const float *decr = reinterpret_cast<const float *>(sm + L::DECR);
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
        auto publish_sx = [&]() {
            uint8_t *sr = sm + L::SR;
#pragma unroll
            for (int j = 0; j < COLS; j += 8) *reinterpret_cast<uint4 *>(sr + sx_off(i, col0 + j)) = pack8(S + j);
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(sx_full);
        };
        bool ok = true;
        if (ncw > 0) publish_sx();
        for (int cw = 0; cw < ncw; ++cw) {
            const int s = cw % NS, b = cw & 1;
            ok = ok && mbar_wait(s_done, cw & 1, err);
            // the stage's decays (its bytes have landed: the UMMAs that just
            // completed read it), then release the stage to the producer
            ok = ok && mbar_wait(full + s, (cw / NS) & 1, err);
            tc_fence_after();
            const float gc = decr[s * kDK + i];
            __syncwarp();
            if (lane == 0 && cw + NS < ncw) mbar_arrive(empty + s);
            const uint32_t da = lane_addr + (uint32_t)(b * DVT);
#pragma unroll
            for (int hh = 0; hh < COLS; hh += 32) {
                float d[32];
                tmem_ld32(da + hh, d);
                tmem_ld_wait();
#pragma unroll
                for (int u = 0; u < 32; ++u) S[hh + u] = gc * S[hh + u] + d[u];
            }
            if (cw + 1 < ncw) {
                // Sx(cw + 1) over Sx(cw) once the output products of chunk cw have read it
                ok = ok && mbar_wait(o_done + b, (cw >> 1) & 1, err);
                tc_fence_after();
                publish_sx();
            }
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

template <int DV, int DVT>
cudaError_t launch_impl(const FwdArgs &a, const uint8_t *ws, const float *S_in, float *S_out, int c0, int ncw, int WC,
                        bool overlap)
{
    using L = Layout<DV, DVT>;
    auto kern = chain_out_kernel<DV, DVT>;
    static std::atomic<unsigned long long> smem_set{0};
    cudaError_t e = ensure_smem_limit(kern, L::BYTES, smem_set);
    if (e != cudaSuccess) return e;
    LaunchCfg lc(dim3(DV / DVT, a.H, a.B), dim3(kThreads), L::BYTES, a.stream, overlap);
    return cudaLaunchKernelEx(&lc.cfg, kern, ws, S_in, S_out, (bf16 *)a.o, a.T, a.H, c0, ncw, WC, a.err);
}

}  // namespace chainout

cudaError_t launch_chain_out(const FwdArgs &a, int dvt, const uint8_t *ws, const float *S_in, float *S_out, int c0,
                             int ncw, int WC, bool overlap)
{
    if (a.dv == 128) {
        if (dvt == 128) return chainout::launch_impl<128, 128>(a, ws, S_in, S_out, c0, ncw, WC, overlap);
        return chainout::launch_impl<128, 64>(a, ws, S_in, S_out, c0, ncw, WC, overlap);
    }
    return chainout::launch_impl<64, 64>(a, ws, S_in, S_out, c0, ncw, WC, overlap);
}

}  // namespace gdn2
