// fwd_tc.cu -- chunkwise forward for bf16 inputs on the sm_100a tensor cores.
//
// The chunkwise (WY) form with chunks of 64 tokens ("Gated DeltaNet-2",
// iplexlaw.co.kr, section "Procesamiento del token y entrenamiento paralelo";
// gist.science, section 3 "Efficient chunkwise parallel training"): per chunk,
// with Gamma the chunk-local cumulative log-decay (fp32) and r the midpoint,
//   Ehat = e^{Gamma-Gamma_r} b k   Qhat = e^{Gamma-Gamma_r} q
//   Khat = e^{Gamma_r-Gamma} k     Ktil = e^{Gamma_C-Gamma} k      Z = w v
//   A = strict_lower(Ehat Khat^T)  P = lower(Qhat Khat^T)  T = (I + A)^{-1}
//   Sref = e^{Gamma_r} S
//   U = T Z - (T Ehat) Sref        O = P T Z + (Qhat - P T Ehat) Sref
//   S <- e^{Gamma_C} S + Ktil^T U
// which equals the token recurrence up to rounding.
//
// One CTA owns one (batch, head, DVT-wide value tile) and walks the chunks of
// its sequence in order.  Every product is a tcgen05 UMMA with bf16 operands
// staged in shared memory and fp32 accumulators in tensor memory:
//   Gram   [Ehat;Qhat] Khat^T         M=128 N=64  K=DK   -> A (rows 0-63), P (64-127)
//   PT     P T                        M=64  N=64  K=64
//   WU     [T;PT] [Ehat | Z]          M=128 N=DK, DVT   -> [W;PW], [U0;PU0]
//   chain  [-W;Q'] Sref (+= [U0;PU0]) M=128 N=DVT K=DK  -> [U;O]
//   dS     Ktil^T U                   M=DK  N=DVT K=64
// Only the last two depend on the state carried from the previous chunk.  The
// triangular solve runs in fp32 on CUDA cores (one column of T per thread).
// Inputs arrive by TMA (4-D maps over [B][T][H][d]; tokens past T are
// zero-filled), double-buffered so chunk c+1 loads while chunk c computes.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "launch.h"
#include "sm100.cuh"

namespace gdn2 {
namespace {

using namespace sm100;
using bf16 = __nv_bfloat16;

constexpr int kTcThreads = 128;
constexpr int kTmemCols = 512;
constexpr float kLog2e = 1.4426950408889634f;

__host__ __device__ constexpr int align_up(int x, int a) { return (x + a - 1) / a * a; }

// Shared-memory plan (byte offsets from a 1024-byte aligned base).
template <int DK, int DVT>
struct TcLayout {
    static constexpr int KB = DK / 64;           // 64-channel blocks (128-byte rows)
    static constexpr int TILE = 64 * 128;        // [64 rows][128 B] = 8 KB
    static constexpr int VROW = DVT * 2;         // bytes per row of a [64][DVT] bf16 tile
    // input stage (TMA destination)
    static constexpr int Q = 0;
    static constexpr int K = Q + KB * TILE;
    static constexpr int Bg = K + KB * TILE;
    static constexpr int LA = Bg + KB * TILE;    // fp32 [64][DK], unswizzled
    static constexpr int V = LA + 64 * DK * 4;   // bf16 [64][DVT], unswizzled
    static constexpr int W = V + 64 * VROW;
    static constexpr int STAGE_BYTES = W + 64 * VROW;
    // operands
    static constexpr int EQ = align_up(STAGE_BYTES, 1024);   // [Ehat;Qhat] -> [-W;Q'], per block 2 tiles
    static constexpr int KH = EQ + KB * 2 * TILE;            // Khat; then fp32 A for the solve
    static constexpr int KT = KH + align_up(KB * TILE > 64 * 64 * 4 ? KB * TILE : 64 * 64 * 4, 1024);
    static constexpr int PO = KT + KB * TILE;                // P  [64][64] bf16
    static constexpr int TO = PO + TILE;                     // [T;PT] [128][64] bf16
    static constexpr int ZO = TO + 2 * TILE;                 // Z  [64][DVT]
    static constexpr int UO = ZO + align_up(64 * VROW, 1024);// U  [64][DVT]
    static constexpr int SR = UO + align_up(64 * VROW, 1024);// Sref [DK][DVT]
    static constexpr int GC = SR + align_up(DK * VROW, 1024);// e^{Gamma_C} fp32 [DK]
    static constexpr int GR = GC + DK * 4;                   // e^{Gamma_r}
    static constexpr int BAR = GR + DK * 4;                  // 2 mbarriers
    static constexpr int SLOT = BAR + 16;                    // TMEM base address
    static constexpr int BYTES = SLOT + 16 + 1024;           // + alignment slack
    // tensor-memory columns
    static constexpr uint32_t TM_G = 0, TM_PT = 64, TM_W = 128, TM_R1 = 128 + DK, TM_R3 = 128 + DK + DVT;
    static_assert(TM_R3 + DVT <= kTmemCols, "tensor memory plan");
};

// 16-byte vector of 8 bf16 built from 8 floats.
__device__ __forceinline__ uint4 pack8(const float *f)
{
    uint4 r;
    __nv_bfloat162 h;
    h = __floats2bfloat162_rn(f[0], f[1]); r.x = *reinterpret_cast<uint32_t *>(&h);
    h = __floats2bfloat162_rn(f[2], f[3]); r.y = *reinterpret_cast<uint32_t *>(&h);
    h = __floats2bfloat162_rn(f[4], f[5]); r.z = *reinterpret_cast<uint32_t *>(&h);
    h = __floats2bfloat162_rn(f[6], f[7]); r.w = *reinterpret_cast<uint32_t *>(&h);
    return r;
}

__device__ __forceinline__ void unpack8(uint4 v, float *f)
{
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 p = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w[i]));
        f[2 * i] = p.x;
        f[2 * i + 1] = p.y;
    }
}

__device__ __forceinline__ float ld_bf16(const uint8_t *p) { return __bfloat162float(*reinterpret_cast<const bf16 *>(p)); }
__device__ __forceinline__ void st_bf16(uint8_t *p, float x) { *reinterpret_cast<bf16 *>(p) = __float2bfloat16_rn(x); }

// fp32 64x64 matrix in shared memory, 16-byte chunks XOR-swizzled by row so
// that row-per-thread float4 stores do not collide on banks.
__device__ __forceinline__ int af_off(int t, int s) { return t * 64 + ((((s >> 2) ^ (t & 15)) << 2) | (s & 3)); }

template <int DK, int DVT>
__global__ void __launch_bounds__(kTcThreads, 1)
fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
              const __grid_constant__ CUtensorMap tm_b, const __grid_constant__ CUtensorMap tm_la,
              const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_w,
              const float *S0, bf16 *__restrict__ o, float *S_T, int Tlen, int H, int DV,
              unsigned int *err)
{
    using L = TcLayout<DK, DVT>;
    constexpr int KB = L::KB, TILE = L::TILE, VROW = L::VROW, C = kChunk;
    static_assert(DK == 128, "the tensor-core path is written for dk = 128");

    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int tile = blockIdx.x, h = blockIdx.y, bi = blockIdx.z;
    uint64_t *bar_tma = reinterpret_cast<uint64_t *>(sm + L::BAR);
    uint64_t *bar_mma = bar_tma + 1;
    uint32_t *slot = reinterpret_cast<uint32_t *>(sm + L::SLOT);
    float *gcs = reinterpret_cast<float *>(sm + L::GC);
    float *grs = reinterpret_cast<float *>(sm + L::GR);
    float *Af = reinterpret_cast<float *>(sm + L::KH);
    const uint32_t sbase = smem_u32(sm);

    if (tid == 0) {
        mbar_init(bar_tma, 1);
        mbar_init(bar_mma, 1);
        fence_mbar_init();
        prefetch_tmap(&tm_q); prefetch_tmap(&tm_k); prefetch_tmap(&tm_b);
        prefetch_tmap(&tm_la); prefetch_tmap(&tm_v); prefetch_tmap(&tm_w);
    }
    if (warp == 0) {
        tmem_alloc(slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *slot;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;

    // State rows: thread i owns row i (key channel i) of this value tile, fp32.
    const long pair = (long)bi * H + h;
    float S[DVT];
#pragma unroll
    for (int j = 0; j < DVT; ++j) S[j] = 0.f;
    if (S0) {
        const float *src = S0 + (pair * DK + tid) * DV + tile * DVT;
#pragma unroll
        for (int j = 0; j < DVT; j += 4) {
            const float4 v4 = *reinterpret_cast<const float4 *>(src + j);
            S[j] = v4.x; S[j + 1] = v4.y; S[j + 2] = v4.z; S[j + 3] = v4.w;
        }
    }

    const int nch = (Tlen + C - 1) / C;
    uint32_t tma_phase = 0, mma_phase = 0;
    bool tma_inflight = false, mma_inflight = false, ok = true;

    auto issue_loads = [&](int c) {
        mbar_arrive_expect_tx(bar_tma, (uint32_t)L::STAGE_BYTES);
        const int t0 = c * C;
#pragma unroll
        for (int kb = 0; kb < KB; ++kb) {
            tma_load_4d(sm + L::Q + kb * TILE, &tm_q, bar_tma, kb * 64, h, t0, bi);
            tma_load_4d(sm + L::K + kb * TILE, &tm_k, bar_tma, kb * 64, h, t0, bi);
            tma_load_4d(sm + L::Bg + kb * TILE, &tm_b, bar_tma, kb * 64, h, t0, bi);
        }
        tma_load_4d(sm + L::LA, &tm_la, bar_tma, 0, h, t0, bi);
        tma_load_4d(sm + L::V, &tm_v, bar_tma, tile * DVT, h, t0, bi);
        tma_load_4d(sm + L::W, &tm_w, bar_tma, tile * DVT, h, t0, bi);
    };
    // Every thread waits on an MMA commit; the CTA aborts together if any wait gave up.
    auto wait_mma = [&]() -> bool {
        const bool mine = mbar_wait(bar_mma, mma_phase, err);
        mma_phase ^= 1;
        mma_inflight = false;
        tc_fence_after();
        return __syncthreads_and(mine) != 0;
    };

    if (tid == 0 && nch > 0) {
        issue_loads(0);
        tma_inflight = true;
    }

    for (int c = 0; c < nch && ok; ++c) {
        const int t0 = c * C;
        const int Lc = min(C, Tlen - t0);

        // ------------------------------------------------ wait for the chunk's inputs
        {
            const bool mine = mbar_wait(bar_tma, tma_phase, err);
            tma_phase ^= 1;
            if (tid == 0) tma_inflight = false;
            if (!__syncthreads_and(mine)) { ok = false; break; }
        }

        // ------------------------------------------------ Gamma, factors, Z, Sref
        {
            const int i = tid;  // key channel
            float *la = reinterpret_cast<float *>(sm + L::LA);  // log_alpha, overwritten by Gamma
            const int rm = min(C / 2, Lc);
            float g = 0.f, gr = 0.f;
#pragma unroll 16
            for (int t = 0; t < C; ++t) {
                g += la[t * DK + i];
                la[t * DK + i] = g;
                if (t == rm - 1) gr = g;
            }
            const float gc = g;
            gcs[i] = expf(gc);
            const float egr = expf(gr);
            grs[i] = egr;
            const float egcr = exp2f((gc - gr) * kLog2e);
            const int kb = i >> 6, cb = (i & 63) * 2;
            uint8_t *q_in = sm + L::Q + kb * TILE, *k_in = sm + L::K + kb * TILE, *b_in = sm + L::Bg + kb * TILE;
            uint8_t *eq = sm + L::EQ + kb * 2 * TILE;
            uint8_t *kh = sm + L::KH + kb * TILE, *kt = sm + L::KT + kb * TILE;
            unsigned int bad = 0;
#pragma unroll 8
            for (int t = 0; t < C; ++t) {
                const uint32_t off = swz_off(t, cb, 128);
                const float x = la[t * DK + i] - gr;
                bad |= (fabsf(x) > kMaxHalfChunkLogDecay);
                const float up = exp2f(x * kLog2e), dn = exp2f(-x * kLog2e);
                const float kv = ld_bf16(k_in + off);
                st_bf16(eq + off, up * ld_bf16(b_in + off) * kv);
                st_bf16(eq + TILE + off, up * ld_bf16(q_in + off));
                st_bf16(kh + off, dn * kv);
                st_bf16(kt + off, egcr * dn * kv);
            }
            if (bad) atomicOr(err, kErrRange);
            // Sref row i = e^{Gamma_r} S_i
#pragma unroll
            for (int j = 0; j < DVT; j += 8) {
                float f[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) f[u] = egr * S[j + u];
                *reinterpret_cast<uint4 *>(sm + L::SR + swz_off(i, j * 2, VROW)) = pack8(f);
            }
            // Z = w v
            const bf16 *vin = reinterpret_cast<const bf16 *>(sm + L::V);
            const bf16 *win = reinterpret_cast<const bf16 *>(sm + L::W);
            for (int idx = tid; idx < C * DVT; idx += kTcThreads) {
                const int t = idx / DVT, j = idx % DVT;
                st_bf16(sm + L::ZO + swz_off(t, j * 2, VROW),
                        __bfloat162float(vin[idx]) * __bfloat162float(win[idx]));
            }
        }
        fence_proxy_async_smem();
        __syncthreads();

        // ------------------------------------------------ next chunk's loads; Gram MMA
        if (tid == 0) {
            if (c + 1 < nch) {
                issue_loads(c + 1);
                tma_inflight = true;
            }
            tc_fence_after();
            const uint32_t id = idesc_bf16(128, 64, 0, 0);
#pragma unroll
            for (int ks = 0; ks < DK / 16; ++ks) {
                const uint32_t koff = (ks & 3) * 32;
                const uint64_t ad = smem_desc(sbase + L::EQ + (ks >> 2) * 2 * TILE + koff, 16, 1024, kSw128);
                const uint64_t bd = smem_desc(sbase + L::KH + (ks >> 2) * TILE + koff, 16, 1024, kSw128);
                umma_bf16(tmem + L::TM_G, ad, bd, id, ks > 0);
            }
            umma_commit(bar_mma);
            mma_inflight = true;
        }
        if (!wait_mma()) { ok = false; break; }

        // ------------------------------------------------ A (fp32, for the solve) and P (bf16 operand)
        {
            const int t = tid & 63;
            float r[64];
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
                float part[16];
                tmem_ld16(tmem + lane_base + L::TM_G + q4 * 16, part);
#pragma unroll
                for (int u = 0; u < 16; ++u) r[q4 * 16 + u] = part[u];
            }
            tmem_ld_wait();
            if (warp < 2) {  // rows of A: strictly lower
#pragma unroll
                for (int s = 0; s < 64; s += 4) {
                    float4 v4;
                    v4.x = (s + 0 < t) ? r[s + 0] : 0.f;
                    v4.y = (s + 1 < t) ? r[s + 1] : 0.f;
                    v4.z = (s + 2 < t) ? r[s + 2] : 0.f;
                    v4.w = (s + 3 < t) ? r[s + 3] : 0.f;
                    *reinterpret_cast<float4 *>(Af + af_off(t, s)) = v4;
                }
            } else {         // rows of P: lower including the diagonal
#pragma unroll
                for (int s = 0; s < 64; s += 8) {
                    float f[8];
#pragma unroll
                    for (int u = 0; u < 8; ++u) f[u] = (s + u <= t) ? r[s + u] : 0.f;
                    *reinterpret_cast<uint4 *>(sm + L::PO + swz_off(t, s * 2, 128)) = pack8(f);
                }
            }
        }
        tc_fence_before();
        __syncthreads();

        // ------------------------------------------------ T = (I + A)^{-1}: one column per thread
        if (tid < 64) {
            const int j = tid;
            float x[64];
#pragma unroll
            for (int t = 0; t < 64; ++t) {
                float acc0 = (t == j) ? 1.f : 0.f, acc1 = 0.f;
#pragma unroll
                for (int s = 0; s < (t & ~3); s += 4) {
                    const float4 a4 = *reinterpret_cast<const float4 *>(Af + af_off(t, s));
                    acc0 -= a4.x * x[s] + a4.z * x[s + 2];
                    acc1 -= a4.y * x[s + 1] + a4.w * x[s + 3];
                }
#pragma unroll
                for (int s = t & ~3; s < t; ++s) acc0 -= Af[af_off(t, s)] * x[s];
                x[t] = acc0 + acc1;
            }
#pragma unroll
            for (int t = 0; t < 64; ++t) st_bf16(sm + L::TO + swz_off(t, j * 2, 128), x[t]);
        }
        fence_proxy_async_smem();
        __syncthreads();

        // ------------------------------------------------ PT = P T  (M = 64)
        if (tid == 0) {
            tc_fence_after();
            const uint32_t id = idesc_bf16(64, 64, 0, 1);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                const uint64_t ad = smem_desc(sbase + L::PO + ks * 32, 16, 1024, kSw128);
                const uint64_t bd = smem_desc(sbase + L::TO + ks * 16 * 128, 8192, 1024, kSw128);
                umma_bf16(tmem + L::TM_PT, ad, bd, id, ks > 0);
            }
            umma_commit(bar_mma);
            mma_inflight = true;
        }
        if (!wait_mma()) { ok = false; break; }
        {
            float r[64];
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
                float part[16];
                tmem_ld16(tmem + lane_base + L::TM_PT + q4 * 16, part);
#pragma unroll
                for (int u = 0; u < 16; ++u) r[q4 * 16 + u] = part[u];
            }
            tmem_ld_wait();
            if (lane < 16) {  // M = 64 accumulator: row 16*warp + lane lives in TMEM lane 32*warp + lane
                const int row = 64 + warp * 16 + lane;
#pragma unroll
                for (int s = 0; s < 64; s += 8)
                    *reinterpret_cast<uint4 *>(sm + L::TO + swz_off(row, s * 2, 128)) = pack8(&r[s]);
            }
        }
        tc_fence_before();
        fence_proxy_async_smem();
        __syncthreads();

        // ------------------------------------------------ [W;PW] = [T;PT] Ehat,  [U0;PU0] = [T;PT] Z
        if (tid == 0) {
            tc_fence_after();
            const uint32_t idw = idesc_bf16(128, DK, 0, 1);
            const uint32_t idz = idesc_bf16(128, DVT, 0, 1);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                const uint64_t ad = smem_desc(sbase + L::TO + ks * 32, 16, 1024, kSw128);
                const uint64_t be = smem_desc(sbase + L::EQ + ks * 16 * 128, 2 * TILE, 1024, kSw128);
                umma_bf16(tmem + L::TM_W, ad, be, idw, ks > 0);
                const uint64_t bz = smem_desc(sbase + L::ZO + ks * 16 * VROW, 8 * VROW, 8 * VROW, swz_mode(VROW));
                umma_bf16(tmem + L::TM_R1, ad, bz, idz, ks > 0);
            }
            umma_commit(bar_mma);
            mma_inflight = true;
        }
        if (!wait_mma()) { ok = false; break; }

        // ------------------------------------------------ -W over Ehat; Q' = Qhat - PW over Qhat
        {
            const int t = tid & 63;
            const int half = warp >> 1;  // 0: W rows, 1: PW rows
#pragma unroll
            for (int kb = 0; kb < KB; ++kb) {
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    float part[16];
                    tmem_ld16(tmem + lane_base + L::TM_W + kb * 64 + q4 * 16, part);
                    tmem_ld_wait();
                    uint8_t *base = sm + L::EQ + kb * 2 * TILE + half * TILE;
#pragma unroll
                    for (int u8 = 0; u8 < 16; u8 += 8) {
                        const uint32_t off = swz_off(t, (q4 * 16 + u8) * 2, 128);
                        float f[8];
                        if (half == 0) {
#pragma unroll
                            for (int u = 0; u < 8; ++u) f[u] = -part[u8 + u];
                        } else {
                            float qh[8];
                            unpack8(*reinterpret_cast<const uint4 *>(base + off), qh);
#pragma unroll
                            for (int u = 0; u < 8; ++u) f[u] = qh[u] - part[u8 + u];
                        }
                        *reinterpret_cast<uint4 *>(base + off) = pack8(f);
                    }
                }
            }
        }
        tc_fence_before();
        fence_proxy_async_smem();
        __syncthreads();

        // ------------------------------------------------ chain: [U;O] = [U0;PU0] + [-W;Q'] Sref
        if (tid == 0) {
            tc_fence_after();
            const uint32_t id = idesc_bf16(128, DVT, 0, 1);
#pragma unroll
            for (int ks = 0; ks < DK / 16; ++ks) {
                const uint64_t ad = smem_desc(sbase + L::EQ + (ks >> 2) * 2 * TILE + (ks & 3) * 32, 16, 1024, kSw128);
                const uint64_t bd = smem_desc(sbase + L::SR + ks * 16 * VROW, 8 * VROW, 8 * VROW, swz_mode(VROW));
                umma_bf16(tmem + L::TM_R1, ad, bd, id, 1);
            }
            umma_commit(bar_mma);
            mma_inflight = true;
        }
        if (!wait_mma()) { ok = false; break; }
        {
            const int t = tid & 63;
            float r[DVT];
#pragma unroll
            for (int j = 0; j < DVT; j += 16) {
                float part[16];
                tmem_ld16(tmem + lane_base + L::TM_R1 + j, part);
#pragma unroll
                for (int u = 0; u < 16; ++u) r[j + u] = part[u];
            }
            tmem_ld_wait();
            if (warp < 2) {  // U -> operand of the state update
#pragma unroll
                for (int j = 0; j < DVT; j += 8)
                    *reinterpret_cast<uint4 *>(sm + L::UO + swz_off(t, j * 2, VROW)) = pack8(&r[j]);
            } else if (t < Lc) {  // O -> global
                bf16 *dst = o + (((long)bi * Tlen + t0 + t) * H + h) * (long)DV + tile * DVT;
#pragma unroll
                for (int j = 0; j < DVT; j += 8) *reinterpret_cast<uint4 *>(dst + j) = pack8(&r[j]);
            }
        }
        tc_fence_before();
        fence_proxy_async_smem();
        __syncthreads();

        // ------------------------------------------------ dS = Ktil^T U
        if (tid == 0) {
            tc_fence_after();
            const uint32_t id = idesc_bf16(128, DVT, 1, 1);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                const uint64_t ad = smem_desc(sbase + L::KT + ks * 16 * 128, TILE, 1024, kSw128);
                const uint64_t bd = smem_desc(sbase + L::UO + ks * 16 * VROW, 8 * VROW, 8 * VROW, swz_mode(VROW));
                umma_bf16(tmem + L::TM_R3, ad, bd, id, ks > 0);
            }
            umma_commit(bar_mma);
            mma_inflight = true;
        }
        if (!wait_mma()) { ok = false; break; }
        {
            const float gci = gcs[tid];
#pragma unroll
            for (int j = 0; j < DVT; j += 16) {
                float part[16];
                tmem_ld16(tmem + lane_base + L::TM_R3 + j, part);
                tmem_ld_wait();
#pragma unroll
                for (int u = 0; u < 16; ++u) S[j + u] = gci * S[j + u] + part[u];
            }
        }
        tc_fence_before();
        __syncthreads();
    }

    if (ok && S_T) {
        float *dst = S_T + (pair * DK + tid) * DV + tile * DVT;
#pragma unroll
        for (int j = 0; j < DVT; j += 4)
            *reinterpret_cast<float4 *>(dst + j) = make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]);
    }

    // Leave nothing in flight: on an aborted run, drain (bounded) before freeing TMEM.
    if (tid == 0) {
        if (tma_inflight) mbar_wait(bar_tma, tma_phase, err);
        if (mma_inflight) mbar_wait(bar_mma, mma_phase, err);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// ------------------------------------------------------------------ host side
PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// 4-D map over a [B][T][H][d] tensor: dims (d, H, T, B), box (box_d, 1, 64, 1).
bool make_map(CUtensorMap *m, const void *base, CUtensorMapDataType dt, int esize, int d, int H, int T, int B,
              int box_d, CUtensorMapSwizzle swz)
{
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    cuuint64_t strides[3] = {(cuuint64_t)d * esize, (cuuint64_t)H * d * esize, (cuuint64_t)T * H * d * esize};
    cuuint32_t box[4] = {(cuuint32_t)box_d, 1, 64, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    return fn(m, dt, 4, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int DK, int DVT>
cudaError_t launch(const FwdArgs &a)
{
    using L = TcLayout<DK, DVT>;
    CUtensorMap mq, mk, mb, ml, mv, mw;
    const auto BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    if (!make_map(&mq, a.q, BF, 2, DK, a.H, a.T, a.B, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&mk, a.k, BF, 2, DK, a.H, a.T, a.B, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&mb, a.b, BF, 2, DK, a.H, a.T, a.B, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&ml, a.log_alpha, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, DK, a.H, a.T, a.B, DK,
                  CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !make_map(&mv, a.v, BF, 2, a.dv, a.H, a.T, a.B, DVT, CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !make_map(&mw, a.w, BF, 2, a.dv, a.H, a.T, a.B, DVT, CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    auto kern = fwd_tc_kernel<DK, DVT>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::BYTES);
    if (e != cudaSuccess) return e;
    dim3 grid(a.dv / DVT, a.H, a.B);
    kern<<<grid, kTcThreads, L::BYTES, a.stream>>>(mq, mk, mb, ml, mv, mw, a.S0, (bf16 *)a.o, a.S_T, a.T, a.H,
                                                    a.dv, a.err);
    return cudaGetLastError();
}

}  // namespace

// Value-tile width: the widest tile that still gives every SM a CTA.
int fwd_tc_tile(int B, int H, int dv, int num_sms)
{
    for (int dvt = 64; dvt >= 16; dvt /= 2)
        if (dv % dvt == 0 && (long)B * H * (dv / dvt) >= num_sms) return dvt;
    return 16;
}

cudaError_t launch_fwd_tc(const FwdArgs &a)
{
    switch (fwd_tc_tile(a.B, a.H, a.dv, a.num_sms)) {
    case 64: return launch<128, 64>(a);
    case 32: return launch<128, 32>(a);
    default: return launch<128, 16>(a);
    }
}

}  // namespace gdn2
