// fwd_prep.cu -- the state-independent part of the chunkwise forward (bf16 inputs).
//
// One CTA per (batch, head, chunk) computes every quantity of the chunkwise WY
// form that does not depend on the state carried in from earlier chunks
// ("Gated DeltaNet-2", iplexlaw.co.kr, section "Procesamiento del token y
// entrenamiento paralelo"; gist.science, section 3: the cumulative per-channel
// decay is folded into asymmetric erase/key factors and a lower triangular
// system (I + T)^{-1} is solved per chunk).  With Gamma the chunk-local
// cumulative log-decay (fp32) and r the chunk midpoint:
//   Ehat = e^{Gamma-Gamma_r} b k    Qhat = e^{Gamma-Gamma_r} q
//   Khat = e^{Gamma_r-Gamma} k      Ktil = e^{Gamma_C-Gamma} k    Z = w v
//   A = strict_lower(Ehat Khat^T)   P = lower(Qhat Khat^T)   T = (I + A)^{-1}
//   W = T Ehat   U0 = T Z   Q' = Qhat - P W   PU0 = P T Z
//   G = Ktil^T W                    N = Ktil^T U0
// so that, with Sref = e^{Gamma_r} S for the incoming state S,
//   S_next = e^{Gamma_C} S + N - G Sref      O = PU0 + Q' Sref.
// G, N, Q', PU0 and the decays form the chunk's record in the workspace.
//
// Layout of the work on one SM: the CTA fits in half of the shared memory,
// tensor memory and register file, so two chunks are in flight per SM and one
// hides the other's load and UMMA latencies.  q, k, b and log_alpha arrive by
// TMA straight into the operand buffers and the factors are formed in place;
// v and w are read with plain vector loads.  Products are tcgen05 UMMAs with
// fp32 accumulators in tensor memory; the solve is fp32 (16x16 diagonal blocks
// by substitution on CUDA cores, then two levels of block merging whose small
// products run as warp-level tf32 MMAs).  Record pieces leave through bulk copies from freed buffers.
#include <cuda.h>

#include "launch.h"
#include "tc_common.cuh"

namespace gdn2 {
namespace {

using namespace sm100;

constexpr int kPrepThreads = 256;
constexpr int kDK = 128;

struct PrepLayout {
    static constexpr int EQ = 0;          // [Ehat;Qhat]; q and b arrive here; later [.;Q']
    static constexpr int KH = 32768;      // Khat -> fp32 T -> W operand -> G block 0
    static constexpr int KT = 49152;      // k arrives here -> Ktil -> G block 1
    static constexpr int PO = 65536;      // P
    static constexpr int TO = 73728;      // log_alpha (first half) -> fp32 A -> [T;PT] -> PU0 -> N block 1
    static constexpr int ZO = 90112;      // log_alpha (second half) -> Z -> U0 operand -> N block 0
    static constexpr int XS = 106496;     // solve scratch, 4 KB
    static constexpr int DEC = 110592;    // e^{Gamma_C}, e^{Gamma_r}
    static constexpr int TOT = 111616;    // quarter totals [4][128]
    static constexpr int BAR = 113664;
    static constexpr int SLOT = BAR + 16;
    static constexpr int BYTES = SLOT + 16 + 1024;
    static constexpr int TX = 3 * 16384 + 32768;  // q, k, b, log_alpha
    static constexpr uint32_t TM_G = 0, TM_PT = 64, TM_W = 0, TM_U = 128, TMEM_COLS = 256;
};
static_assert(PrepLayout::BYTES * 2 + 2048 <= 233472, "two CTAs per SM");

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&r)[32])
{
    float a[16], b[16];
    tmem_ld16(taddr, a);
    tmem_ld16(taddr + 16, b);
    tmem_ld_wait();
#pragma unroll
    for (int u = 0; u < 16; ++u) { r[u] = a[u]; r[16 + u] = b[u]; }
}

template <int DV>
__global__ void __launch_bounds__(kPrepThreads, 2)
prep_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
            const __grid_constant__ CUtensorMap tm_b, const __grid_constant__ CUtensorMap tm_la,
            const bf16 *__restrict__ vg, const bf16 *__restrict__ wg, uint8_t *__restrict__ ws, int Tlen, int H,
            int c0, int WC, unsigned int *err)
{
    using L = PrepLayout;
    using R = Record<DV>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int wq = warp & 3, wh = warp >> 2;  // TMEM lane quarter, column half
    const int cw = blockIdx.x, h = blockIdx.y, bi = blockIdx.z;
    const int t0 = (c0 + cw) * kChunk;
    const int Lc = min(kChunk, Tlen - t0);
    uint64_t *bar_tma = reinterpret_cast<uint64_t *>(sm + L::BAR);
    uint64_t *bar_mma = bar_tma + 1;
    uint32_t *slot = reinterpret_cast<uint32_t *>(sm + L::SLOT);
    float *la = reinterpret_cast<float *>(sm + L::TO);  // [64][128] fp32 over TO..ZO
    float *Af = reinterpret_cast<float *>(sm + L::TO);
    float *Tf = reinterpret_cast<float *>(sm + L::KH);
    float *Xs = reinterpret_cast<float *>(sm + L::XS);
    float *dec = reinterpret_cast<float *>(sm + L::DEC);
    float *tot = reinterpret_cast<float *>(sm + L::TOT);
    const uint32_t sbase = smem_u32(sm);
    uint8_t *rec = ws + (((long)bi * H + h) * WC + cw) * (long)R::BYTES;
    uint32_t mma_phase = 0;

    if (tid == 0) {
        mbar_init(bar_tma, 1);
        mbar_init(bar_mma, 1);
        fence_mbar_init();
        mbar_arrive_expect_tx(bar_tma, (uint32_t)L::TX);
        for (int kb = 0; kb < 2; ++kb) {
            tma_load_4d(sm + L::EQ + kb * 16384 + 8192, &tm_q, bar_tma, kb * 64, h, t0, bi);
            tma_load_4d(sm + L::EQ + kb * 16384, &tm_b, bar_tma, kb * 64, h, t0, bi);
            tma_load_4d(sm + L::KT + kb * 8192, &tm_k, bar_tma, kb * 64, h, t0, bi);
        }
        tma_load_4d(sm + L::TO, &tm_la, bar_tma, 0, h, t0, bi);
    }
    if (warp == 0) {
        tmem_alloc(slot, L::TMEM_COLS);
        tmem_relinquish();
    }
    // v and w for Z = w v: plain vector loads, issued before anything waits
    constexpr int ZV = 64 * DV / 8 / kPrepThreads;  // 16-byte vectors per thread
    uint4 vv[ZV], wv[ZV];
#pragma unroll
    for (int m = 0; m < ZV; ++m) {
        const int idx = tid + m * kPrepThreads;
        const int t = idx / (DV / 8), j = (idx % (DV / 8)) * 8;
        vv[m] = make_uint4(0, 0, 0, 0);
        wv[m] = make_uint4(0, 0, 0, 0);
        if (t < Lc) {
            const long off = (((long)bi * Tlen + t0 + t) * H + h) * DV + j;
            vv[m] = __ldg(reinterpret_cast<const uint4 *>(vg + off));
            wv[m] = __ldg(reinterpret_cast<const uint4 *>(wg + off));
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *slot;
    const uint32_t lane_base = (uint32_t)(wq * 32) << 16;

    // One thread polls each barrier; the others park on the CTA barrier, which
    // leaves the issue slots to the co-resident CTA.  tcgen05.fence::after
    // orders the tensor-memory reads after that barrier.
    auto mma_done = [&]() {
        const bool mine = (tid == 0) ? mbar_wait(bar_mma, mma_phase, err) : true;
        mma_phase ^= 1;
        const bool all = __syncthreads_and(mine) != 0;
        tc_fence_after();
        return all;
    };
    bool ok = __syncthreads_and((tid == 0) ? mbar_wait(bar_tma, 0, err) : true) != 0;

    if (ok) {
        // ---------------------------------------------------------- Gamma and factors (in place)
        const int p = tid & 63, qr = tid >> 6;           // channel pair, token quarter
        const int kb = p >> 5, cb = (p & 31) * 4;
        float2 lv[16];
#pragma unroll
        for (int u = 0; u < 16; ++u) lv[u] = *reinterpret_cast<const float2 *>(la + (qr * 16 + u) * kDK + 2 * p);
        float g0 = 0.f, g1 = 0.f;
#pragma unroll
        for (int u = 0; u < 16; ++u) {
            g0 += lv[u].x; g1 += lv[u].y;
            lv[u] = make_float2(g0, g1);
        }
        tot[qr * kDK + 2 * p] = g0;
        tot[qr * kDK + 2 * p + 1] = g1;
        __syncthreads();
        float pre0 = 0.f, pre1 = 0.f, gc0 = 0.f, gc1 = 0.f;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float a0 = tot[q * kDK + 2 * p], a1 = tot[q * kDK + 2 * p + 1];
            if (q < qr) { pre0 += a0; pre1 += a1; }
            gc0 += a0; gc1 += a1;
        }
        // midpoint reference: Gamma after 32 tokens (tokens past T carry log_alpha = 0)
        const float gr0 = tot[2 * p] + tot[kDK + 2 * p], gr1 = tot[2 * p + 1] + tot[kDK + 2 * p + 1];
        if (qr == 0) {
            dec[2 * p] = expf(gc0);
            dec[2 * p + 1] = expf(gc1);
            dec[kDK + 2 * p] = expf(gr0);
            dec[kDK + 2 * p + 1] = expf(gr1);
        }
        const float ecr0 = ex2_approx((gc0 - gr0) * kLog2e), ecr1 = ex2_approx((gc1 - gr1) * kLog2e);
        uint8_t *eq = sm + L::EQ + kb * 16384, *kh = sm + L::KH + kb * 8192, *kt = sm + L::KT + kb * 8192;
        unsigned int bad = 0;
        const float sh0 = pre0 - gr0, sh1 = pre1 - gr1;
#pragma unroll
        for (int u = 0; u < 16; ++u) {
            const int t = qr * 16 + u;
            const float x0 = lv[u].x + sh0, x1 = lv[u].y + sh1;
            bad |= (fabsf(x0) > kMaxHalfChunkLogDecay) | (fabsf(x1) > kMaxHalfChunkLogDecay);
            const float up0 = ex2_approx(x0 * kLog2e), up1 = ex2_approx(x1 * kLog2e);
            const float dn0 = ex2_approx(-x0 * kLog2e), dn1 = ex2_approx(-x1 * kLog2e);
            const uint32_t off = swz_off(t, cb, 128);
            const float2 kv = ld_bf16x2(kt + off), bv = ld_bf16x2(eq + off), qv = ld_bf16x2(eq + 8192 + off);
            st_bf16x2(eq + off, up0 * bv.x * kv.x, up1 * bv.y * kv.y);
            st_bf16x2(eq + 8192 + off, up0 * qv.x, up1 * qv.y);
            st_bf16x2(kh + off, dn0 * kv.x, dn1 * kv.y);
            st_bf16x2(kt + off, ecr0 * dn0 * kv.x, ecr1 * dn1 * kv.y);
        }
        if (bad) atomicOr(err, kErrRange);
        fence_proxy_async_smem();
        __syncthreads();

        // ---------------------------------------------------------- Gram: [Ehat;Qhat] Khat^T
        if (tid == 0) {
            tc_fence_after();
            const uint32_t id = idesc_bf16(128, 64, 0, 0);
#pragma unroll
            for (int ks = 0; ks < kDK / 16; ++ks) {
                const uint32_t kofs = (ks & 3) * 32;
                umma_bf16(tmem + L::TM_G, smem_desc(sbase + L::EQ + (ks >> 2) * 16384 + kofs, 16, 1024, kSw128),
                          smem_desc(sbase + L::KH + (ks >> 2) * 8192 + kofs, 16, 1024, kSw128), id, ks > 0);
            }
            umma_commit(bar_mma);
        }
        // Z = w v while the Gram runs (log_alpha in ZO is no longer needed)
#pragma unroll
        for (int m = 0; m < ZV; ++m) {
            const int idx = tid + m * kPrepThreads;
            const int t = idx / (DV / 8), j = (idx % (DV / 8)) * 8;
            float fv[8], fw[8], fz[8];
            unpack8(vv[m], fv);
            unpack8(wv[m], fw);
#pragma unroll
            for (int u = 0; u < 8; ++u) fz[u] = fv[u] * fw[u];
            *reinterpret_cast<uint4 *>(sm + L::ZO + (j >> 6) * 8192 + swz_off(t, (j & 63) * 2, 128)) = pack8(fz);
        }
        fence_proxy_async_smem();
        ok = mma_done();
    }

    if (ok) {
        // ---------------------------------------------------------- A (fp32) and P (bf16)
        {
            const int r = wq * 32 + lane;
            float v[32];
            tmem_ld32(tmem + lane_base + L::TM_G + wh * 32, v);
            if (r < 64) {
                const int t = r;
#pragma unroll
                for (int s4 = 0; s4 < 32; s4 += 4) {
                    const int s = wh * 32 + s4;
                    float4 a4;
                    a4.x = (s + 0 < t) ? v[s4 + 0] : 0.f;
                    a4.y = (s + 1 < t) ? v[s4 + 1] : 0.f;
                    a4.z = (s + 2 < t) ? v[s4 + 2] : 0.f;
                    a4.w = (s + 3 < t) ? v[s4 + 3] : 0.f;
                    *reinterpret_cast<float4 *>(Af + af_off(t, s)) = a4;
                }
            } else {
                const int t = r - 64;
#pragma unroll
                for (int s8 = 0; s8 < 32; s8 += 8) {
                    float f[8];
#pragma unroll
                    for (int u = 0; u < 8; ++u) f[u] = (wh * 32 + s8 + u <= t) ? v[s8 + u] : 0.f;
                    *reinterpret_cast<uint4 *>(sm + L::PO + swz_off(t, (wh * 32 + s8) * 2, 128)) = pack8(f);
                }
            }
            // T starts as zero; Khat (Gram operand, now consumed) gives its room to T
#pragma unroll
            for (int m = 0; m < 4; ++m)
                reinterpret_cast<float4 *>(Tf)[tid + m * kPrepThreads] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
        tc_fence_before();
        __syncthreads();

        // ---------------------------------------------------------- T = (I + A)^{-1}
        // (a) diagonal 16x16 blocks: one column per thread, rows of A read as float4
        if (tid < 64) {
            const int b0 = (tid >> 4) * 16, j = tid & 15;
            float x[16];
#pragma unroll
            for (int t = 0; t < 16; ++t) {
                float a[16];
#pragma unroll
                for (int s4 = 0; s4 < 16; s4 += 4) {
                    const float4 a4 = *reinterpret_cast<const float4 *>(Af + af_off(b0 + t, b0 + s4));
                    a[s4] = a4.x; a[s4 + 1] = a4.y; a[s4 + 2] = a4.z; a[s4 + 3] = a4.w;
                }
                float acc0 = (t == j) ? 1.f : 0.f, acc1 = 0.f;
#pragma unroll
                for (int s = 0; s < t; ++s) {
                    if (s & 1) acc1 -= a[s] * x[s];
                    else acc0 -= a[s] * x[s];
                }
                x[t] = acc0 + acc1;
                Tf[af_off(b0 + t, b0 + j)] = x[t];
            }
        }
        __syncthreads();
        // (b), (c): the merges are small products inside a dependency chain; they
        // run as warp-level tf32 MMAs (m16n8k8) on the fp32 blocks.  g, c: fragment
        // coordinates of this lane.
        const int fg = lane >> 2, fc = lane & 3;
        // (b) T_{b+1,b} = -D_{b+1} (A_{b+1,b} D_b) for the pairs (0,1), (2,3).
        //     Warp w < 4: pair w >> 1, 8-column tile w & 1 of the 16x16 block.
        if (warp < 4) {
            const int which = warp >> 1, n0 = (warp & 1) * 8;
            const int R0 = 16 + 32 * which, C0 = 32 * which;
            float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int k0 = 0; k0 < 16; k0 += 8) {
                mma_tf32(d, to_tf32(Af[af_off(R0 + fg, C0 + k0 + fc)]), to_tf32(Af[af_off(R0 + fg + 8, C0 + k0 + fc)]),
                         to_tf32(Af[af_off(R0 + fg, C0 + k0 + fc + 4)]), to_tf32(Af[af_off(R0 + fg + 8, C0 + k0 + fc + 4)]),
                         to_tf32(Tf[af_off(C0 + k0 + fc, C0 + n0 + fg)]), to_tf32(Tf[af_off(C0 + k0 + fc + 4, C0 + n0 + fg)]));
            }
            float *x = Xs + which * 256;  // X[16][16]
            x[fg * 16 + n0 + 2 * fc] = d[0];
            x[fg * 16 + n0 + 2 * fc + 1] = d[1];
            x[(fg + 8) * 16 + n0 + 2 * fc] = d[2];
            x[(fg + 8) * 16 + n0 + 2 * fc + 1] = d[3];
        }
        __syncthreads();
        if (warp < 4) {
            const int which = warp >> 1, n0 = (warp & 1) * 8;
            const int R0 = 16 + 32 * which, C0 = 32 * which;
            const float *x = Xs + which * 256;
            float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int k0 = 0; k0 < 16; k0 += 8) {
                mma_tf32(d, to_tf32(Tf[af_off(R0 + fg, R0 + k0 + fc)]), to_tf32(Tf[af_off(R0 + fg + 8, R0 + k0 + fc)]),
                         to_tf32(Tf[af_off(R0 + fg, R0 + k0 + fc + 4)]), to_tf32(Tf[af_off(R0 + fg + 8, R0 + k0 + fc + 4)]),
                         to_tf32(x[(k0 + fc) * 16 + n0 + fg]), to_tf32(x[(k0 + fc + 4) * 16 + n0 + fg]));
            }
            Tf[af_off(R0 + fg, C0 + n0 + 2 * fc)] = -d[0];
            Tf[af_off(R0 + fg, C0 + n0 + 2 * fc + 1)] = -d[1];
            Tf[af_off(R0 + fg + 8, C0 + n0 + 2 * fc)] = -d[2];
            Tf[af_off(R0 + fg + 8, C0 + n0 + 2 * fc + 1)] = -d[3];
        }
        __syncthreads();
        // (c) T[32:64, 0:32] = -T_BB (A[32:64, 0:32] T_AA).  Warp w: 16-row tile w >> 2,
        //     8-column tile w & 3 of the 32x32 block; T_AA and T_BB are lower triangular.
        {
            const int m0 = (warp >> 2) * 16, n0 = (warp & 3) * 8;
            float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int k0 = 0; k0 < 32; k0 += 8) {
                if (k0 + 8 <= n0) continue;  // rows k of T_AA above column n0 are zero
                mma_tf32(d, to_tf32(Af[af_off(32 + m0 + fg, k0 + fc)]), to_tf32(Af[af_off(32 + m0 + fg + 8, k0 + fc)]),
                         to_tf32(Af[af_off(32 + m0 + fg, k0 + fc + 4)]), to_tf32(Af[af_off(32 + m0 + fg + 8, k0 + fc + 4)]),
                         to_tf32(Tf[af_off(k0 + fc, n0 + fg)]), to_tf32(Tf[af_off(k0 + fc + 4, n0 + fg)]));
            }
            Xs[(m0 + fg) * 32 + n0 + 2 * fc] = d[0];
            Xs[(m0 + fg) * 32 + n0 + 2 * fc + 1] = d[1];
            Xs[(m0 + fg + 8) * 32 + n0 + 2 * fc] = d[2];
            Xs[(m0 + fg + 8) * 32 + n0 + 2 * fc + 1] = d[3];
        }
        __syncthreads();
        {
            const int m0 = (warp >> 2) * 16, n0 = (warp & 3) * 8;
            float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int k0 = 0; k0 < 32; k0 += 8) {
                if (k0 >= m0 + 16) continue;  // columns k of T_BB right of row m0 + 15 are zero
                mma_tf32(d, to_tf32(Tf[af_off(32 + m0 + fg, 32 + k0 + fc)]),
                         to_tf32(Tf[af_off(32 + m0 + fg + 8, 32 + k0 + fc)]),
                         to_tf32(Tf[af_off(32 + m0 + fg, 32 + k0 + fc + 4)]),
                         to_tf32(Tf[af_off(32 + m0 + fg + 8, 32 + k0 + fc + 4)]),
                         to_tf32(Xs[(k0 + fc) * 32 + n0 + fg]), to_tf32(Xs[(k0 + fc + 4) * 32 + n0 + fg]));
            }
            Tf[af_off(32 + m0 + fg, n0 + 2 * fc)] = -d[0];
            Tf[af_off(32 + m0 + fg, n0 + 2 * fc + 1)] = -d[1];
            Tf[af_off(32 + m0 + fg + 8, n0 + 2 * fc)] = -d[2];
            Tf[af_off(32 + m0 + fg + 8, n0 + 2 * fc + 1)] = -d[3];
        }
        __syncthreads();
        // (d) T -> bf16 operand rows 0..63 of [T;PT] (A has served its purpose)
        {
            const int t = tid >> 2, g = (tid & 3) * 16;
            float f[16];
#pragma unroll
            for (int u = 0; u < 16; u += 4) {
                const float4 v4 = *reinterpret_cast<const float4 *>(Tf + af_off(t, g + u));
                f[u] = v4.x; f[u + 1] = v4.y; f[u + 2] = v4.z; f[u + 3] = v4.w;
            }
            *reinterpret_cast<uint4 *>(sm + L::TO + swz_off(t, g * 2, 128)) = pack8(f);
            *reinterpret_cast<uint4 *>(sm + L::TO + swz_off(t, g * 2 + 16, 128)) = pack8(f + 8);
        }
        fence_proxy_async_smem();
        __syncthreads();

        // ---------------------------------------------------------- PT = P T   (M = 64)
        if (tid == 0) {
            tc_fence_after();
            const uint32_t id = idesc_bf16(64, 64, 0, 1);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                umma_bf16(tmem + L::TM_PT, smem_desc(sbase + L::PO + ks * 32, 16, 1024, kSw128),
                          smem_desc(sbase + L::TO + ks * 2048, 8192, 1024, kSw128), id, ks > 0);
            umma_commit(bar_mma);
        }
        ok = mma_done();
    }

    if (ok) {
        {   // M = 64 accumulator: row 16*wq + l sits in TMEM lane 32*wq + l (l < 16)
            float v[32];
            tmem_ld32(tmem + lane_base + L::TM_PT + wh * 32, v);
            if (lane < 16) {
                const int row = 64 + wq * 16 + lane;
#pragma unroll
                for (int s8 = 0; s8 < 32; s8 += 8)
                    *reinterpret_cast<uint4 *>(sm + L::TO + swz_off(row, (wh * 32 + s8) * 2, 128)) = pack8(v + s8);
            }
        }
        tc_fence_before();
        fence_proxy_async_smem();
        __syncthreads();

        // ---------------------------------------------------------- [W;PW] = [T;PT] Ehat,  [U0;PU0] = [T;PT] Z
        if (tid == 0) {
            tc_fence_after();
            const uint32_t idw = idesc_bf16(128, kDK, 0, 1), idz = idesc_bf16(128, DV, 0, 1);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                const uint64_t ad = smem_desc(sbase + L::TO + ks * 32, 16, 1024, kSw128);
                umma_bf16(tmem + L::TM_W, ad, smem_desc(sbase + L::EQ + ks * 2048, 16384, 1024, kSw128), idw, ks > 0);
                umma_bf16(tmem + L::TM_U, ad, smem_desc(sbase + L::ZO + ks * 2048, 8192, 1024, kSw128), idz, ks > 0);
            }
            umma_commit(bar_mma);
        }
        ok = mma_done();
    }

    if (ok) {
        {
            const int r = wq * 32 + lane;
            const int t = r & 63;
            // W rows -> W operand (KH); PW rows -> Q' = Qhat - PW, in place over Qhat
#pragma unroll
            for (int part = 0; part < 64; part += 32) {
                float v[32];
                tmem_ld32(tmem + lane_base + L::TM_W + wh * 64 + part, v);
#pragma unroll
                for (int s8 = 0; s8 < 32; s8 += 8) {
                    const uint32_t off = swz_off(t, (part + s8) * 2, 128);
                    if (r < 64) {
                        *reinterpret_cast<uint4 *>(sm + L::KH + wh * 8192 + off) = pack8(v + s8);
                    } else {
                        uint4 *qp = reinterpret_cast<uint4 *>(sm + L::EQ + wh * 16384 + 8192 + off);
                        float qh[8], f[8];
                        unpack8(*qp, qh);
#pragma unroll
                        for (int u = 0; u < 8; ++u) f[u] = qh[u] - v[s8 + u];
                        *qp = pack8(f);
                    }
                }
            }
            // U0 rows -> U0 operand (ZO); PU0 rows -> PU0 (TO, the record's block layout)
            constexpr int HALF = DV / 2;
#pragma unroll
            for (int part = 0; part < HALF; part += 32) {
                float v[32];
                tmem_ld32(tmem + lane_base + L::TM_U + wh * HALF + part, v);
#pragma unroll
                for (int s8 = 0; s8 < 32; s8 += 8) {
                    const int col = wh * HALF + part + s8;
                    const uint32_t off = (col >> 6) * 8192 + swz_off(t, (col & 63) * 2, 128);
                    *reinterpret_cast<uint4 *>(sm + (r < 64 ? L::ZO : L::TO) + off) = pack8(v + s8);
                }
            }
        }
        tc_fence_before();
        fence_proxy_async_smem();
        __syncthreads();

        // ---------------------------------------------------------- G = Ktil^T W,  N = Ktil^T U0
        if (tid == 0) {
            tc_fence_after();
            bulk_store(rec + R::QP, sm + L::EQ + 8192, 8192);          // Q' (two 8 KB blocks)
            bulk_store(rec + R::QP + 8192, sm + L::EQ + 24576, 8192);
            bulk_store(rec + R::PU, sm + L::TO, 64 * DV * 2);          // PU0
            bulk_commit();
            const uint32_t idg = idesc_bf16(128, kDK, 1, 1), idn = idesc_bf16(128, DV, 1, 1);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                const uint64_t ad = smem_desc(sbase + L::KT + ks * 2048, 8192, 1024, kSw128);
                umma_bf16(tmem + L::TM_W, ad, smem_desc(sbase + L::KH + ks * 2048, 8192, 1024, kSw128), idg, ks > 0);
                umma_bf16(tmem + L::TM_U, ad, smem_desc(sbase + L::ZO + ks * 2048, 8192, 1024, kSw128), idn, ks > 0);
            }
            umma_commit(bar_mma);
        }
        bool mine = true;
        if (tid == 0) {
            mine = mbar_wait(bar_mma, mma_phase, err);
            bulk_wait_read_all();  // PU0 has left TO before N is staged there
        }
        mma_phase ^= 1;
        ok = __syncthreads_and(mine) != 0;
        tc_fence_after();
    }

    if (ok) {
        {   // G rows -> KH (block 0) / KT (block 1);  N rows -> ZO (block 0) / TO (block 1)
            const int i = wq * 32 + lane;  // key channel
#pragma unroll
            for (int part = 0; part < 64; part += 32) {
                float v[32];
                tmem_ld32(tmem + lane_base + L::TM_W + wh * 64 + part, v);
#pragma unroll
                for (int s8 = 0; s8 < 32; s8 += 8)
                    *reinterpret_cast<uint4 *>(sm + (wh ? L::KT : L::KH) + swz_off(i, (part + s8) * 2, 128)) =
                        pack8(v + s8);
            }
            constexpr int HALF = DV / 2;
#pragma unroll
            for (int part = 0; part < HALF; part += 32) {
                float v[32];
                tmem_ld32(tmem + lane_base + L::TM_U + wh * HALF + part, v);
#pragma unroll
                for (int s8 = 0; s8 < 32; s8 += 8) {
                    const int col = wh * HALF + part + s8;
                    *reinterpret_cast<uint4 *>(sm + ((col >> 6) ? L::TO : L::ZO) + swz_off(i, (col & 63) * 2, 128)) =
                        pack8(v + s8);
                }
            }
        }
        fence_proxy_async_smem();
        __syncthreads();
        if (tid == 0) {
            bulk_store(rec + R::GC, sm + L::KH, 16384);
            bulk_store(rec + R::GC + 16384, sm + L::KT, 16384);
            bulk_store(rec + R::NC, sm + L::ZO, 16384);
            if (DV > 64) bulk_store(rec + R::NC + 16384, sm + L::TO, 16384);
            bulk_store(rec + R::DEC, sm + L::DEC, 1024);
            bulk_commit();
            bulk_wait_read_all();
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

template <int DV>
cudaError_t launch_prep_impl(const FwdArgs &a, const CUtensorMap *maps, uint8_t *ws, int c0, int ncw, int WC)
{
    using L = PrepLayout;
    auto kern = prep_kernel<DV>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::BYTES);
    if (e != cudaSuccess) return e;
    dim3 grid(ncw, a.H, a.B);
    kern<<<grid, kPrepThreads, L::BYTES, a.stream>>>(maps[0], maps[1], maps[2], maps[3], (const bf16 *)a.v,
                                                     (const bf16 *)a.w, ws, a.T, a.H, c0, WC, a.err);
    return cudaGetLastError();
}

cudaError_t launch_prep(const FwdArgs &a, const CUtensorMap *maps, uint8_t *ws, int c0, int ncw, int WC)
{
    return a.dv == 128 ? launch_prep_impl<128>(a, maps, ws, c0, ncw, WC) : launch_prep_impl<64>(a, maps, ws, c0, ncw, WC);
}

}  // namespace gdn2
