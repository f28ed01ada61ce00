// bwd_tc.cu -- the bf16 tensor-core backward of the chunkwise forward (dk = 128).
//
// "Gated DeltaNet-2", iplexlaw.co.kr, section "Procesamiento del token y
// entrenamiento paralelo" (and gist.science, section 3): training uses the
// chunkwise WY form, and its backward keeps the per-channel gates b and w inside
// the gradients of the auxiliaries.  For one chunk of C = 64 tokens, with the
// state S entering it, the decayed factors Ebar = e^{Gamma} b k, Qbar = e^{Gamma} q,
// Ktil = e^{Gamma_C - Gamma} k, A = strict_lower(e k^T decayed), P = lower(q k^T
// decayed), T = (I + A)^{-1} and Z = w v, the forward is
//   X = Z - Ebar S,  U = T X,  O = Qbar S + P U,  S' = e^{Gamma_C} S + Ktil^T U.
// Given dO and the gradient dS' of the state leaving the chunk:
//   gU = Ktil dS' + P^T dO          dX = T^T gU          dv = dX w, dw = dX v
//   dQbar = dO S^T   dEbar = -dX S^T   dKtil = U dS'^T   dP = dO U^T   dA = -dX U^T
// and dA, dP reach e, q, k through the pairwise decays e^{Gamma_t - Gamma_s}.
// dS, the gradient of the state entering the chunk, is the transpose of the
// chunk's map applied to dS' and dO (the adjoint chain, chain_body.cuh ADJ).
//
// Steps (one stream, no host synchronisation):
//   1. prep of every chunk (prep_body.cuh), keeping T and P beside the records
//      (and T - bf16(T), with a flag in the record, where T is far from the identity);
//   2. in one launch, on separate CTAs, the forward chain over every chunk (bf16
//      images of each chunk's entry state) and the adjoint chain over the chunks
//      in reverse (images of each chunk's dS', and dS0): the adjoint chain needs
//      the records and dO, not the forward's states;
//   3. grad_kernel: one CTA per (chunk, head, batch), all in parallel, the
//      products above as tcgen05 UMMAs with fp32 accumulators in tensor memory;
//      a flagged chunk then runs again with T and X as bf16 pairs.
//
// In grad_kernel the decays split at the chunk midpoint r like the forward's
// prep (Ehat = e^{Gamma - Gamma_r} e, Qhat, Khat = e^{Gamma_r - Gamma} k), the
// state images scaled by rows, S_r = Diag(e^{Gamma_r}) S and
// dS_c = Diag(e^{Gamma_C - Gamma_r}) dS', so that
//   dq = e^{Gamma - Gamma_r} (dO S_r^T + dP Khat)
//   de = e^{Gamma - Gamma_r} (-dX S_r^T + dA Khat)
//   dk_write = e^{Gamma_r - Gamma} (U dS_c^T + dP^T Qhat + dA^T Ehat)
// accumulate in tensor memory.  A chunk whose decay is too strong for the split
// (the forward prep's test) uses Ebar, Qbar, Ktil and unscaled images instead,
// and forms the pairwise terms by walks over running products of alpha.  Then
//   dk = dk_write + de b,  db = de k,  dGamma_t = q dq + e de - k dk_write,
// and dlog_alpha_u = sum_{t >= u} dGamma_t + dGamma_C (Gamma_C = Gamma at the
// chunk end).  Written that way, dlog_alpha is a small difference of large
// terms when the decay is strong, so the sum is regrouped to cancel exactly:
//   * the diagonal of P (P_tt does not depend on Gamma) adds dP_tt k_t to dq_t
//     and dP_tt q_t to dk_t but nothing to dGamma;
//   * Ktil's share, K_t = k_t e^{Gamma_C - Gamma_t} (U dS'^T)_t, enters dGamma_t
//     with a minus sign and dGamma_C with a plus sign, so it adds
//     sum_{t < u} K_t to dlog_alpha_u;
//   * what remains of dGamma_C is rowsum(dS' o e^{Gamma_C} S).
#include <cuda.h>

#include "chain_body.cuh"
#include "launch.h"

namespace gdn2 {
namespace bwdtc {

using namespace sm100;

constexpr int kGT = 256;   // grad_kernel threads
constexpr int kDK = 128;
constexpr int kBar = 1;    // the named barrier of grad_kernel's threads

// Shared memory of grad_kernel (byte offsets from a 1024-aligned base).  Every
// tile is sized for dv = 128; dv = 64 uses the first half of the value tiles.
struct GradLayout {
    static constexpr int EQ = 0;          // per 64-key half: [E rows 0-63 | Q rows 64-127], 128-byte swizzle
    static constexpr int KT = 32768;      // per 64-key half: K rows 0-63
    static constexpr int SR = 49152;      // state image S -> S_r (no swizzle, [128][dv] MN-major)
    static constexpr int DSC = 81920;     // image of dS' -> dS_c
    static constexpr int G = 114688;      // per 64-value block: [dO rows 0-63 | -dX rows 64-127]
    static constexpr int U = 147456;      // per 64-value block: gU, then U (rows = tokens)
    static constexpr int XG = 163840;     // per 64-value block: X
    static constexpr int TT = 180224;     // T [64][64]
    static constexpr int PP = 188416;     // P [64][64]
    static constexpr int DPA = 196608;    // [dP rows 0-63 | dA rows 64-127], 64 token columns
    static constexpr int MISC = 212992;
    static constexpr int SIG_S = MISC;            // [128] row scale of S
    static constexpr int SIG_D = MISC + 512;      // [128] row scale of dS'
    static constexpr int GRV = MISC + 1024;       // [128] Gamma_r (0 in the bounded form)
    static constexpr int GCV = MISC + 1536;       // [128] Gamma_C
    static constexpr int QTOT = MISC + 2048;      // [4][128] quarter sums
    static constexpr int QPROD = MISC + 4096;     // [4][128] quarter products of alpha (bounded form)
    static constexpr int DGC = MISC + 6144;       // [2][128] halves of rowsum(dS' o e^{Gamma_C} S)
    static constexpr int DIAG = MISC + 7168;      // [64] dP_tt
    static constexpr int BAR = MISC + 7424;       // bar_ld, bar_mma, bar_raw
    static constexpr int SLOT = BAR + 32;         // tensor-memory address
    static constexpr int DATA = SLOT + 16;
    static constexpr int BYTES = DATA + 1024;
    // reused by the epilogue, once the products that read them have completed
    static constexpr int XST = SR;                // x = Gamma - Gamma_r, fp32 [64][128] (fo layout)
    static constexpr int KST = DSC;               // K_t, fp32 [64][128]
    static constexpr int DGS = G;                 // dGamma without K and the diagonal, fp32 [64][128]
    static constexpr int ALPHA = U;               // bounded: alpha, fp32 [64][128] (U and XG)
    static constexpr int RQ = EQ, RB = EQ + 16384, RK = KT;  // bounded: raw q, b, k, bf16 [64][128]
    // midpoint: raw q, b, k again by TMA for the epilogue (128-byte swizzle, 64-channel halves)
    static constexpr int TQ = U, TB = XG, TK = TT;
    // tensor-memory columns
    static constexpr uint32_t TM_DX0 = 0, TM_GU = 128, TM_U = 256, TM_DX = 384;  // Ebar S, gU, U, dX
    // dk' holds U dS_c^T, dk2 the pairwise part (dP^T Qhat + dA^T Ehat) once [dP; dA] is read
    static constexpr uint32_t TM_DPA = 0, TM_DQ = 128, TM_DE = 256, TM_DK = 384, TM_DK2 = 0;
    static constexpr uint32_t TMEM_COLS = 512;
};
static_assert(GradLayout::BYTES <= 232448, "shared memory");

// fp32 [64][128] tile in shared memory, 16-byte chunks XORed with the row: row
// reads of 16 rows by 16 lanes and column-pair reads by 32 lanes stay spread.
__device__ __forceinline__ int fo(int t, int j) { return t * 128 + ((((j >> 2) ^ (t & 7)) << 2) | (j & 3)); }

struct GradArgs {
    const bf16 *q, *k, *b, *v, *w;
    const float *la;
    const uint8_t *sx;      // [pairs][n] images of the state entering each chunk
    const uint8_t *dsx;     // [pairs][n] images of dS' (the gradient of the state leaving each chunk)
    const uint8_t *tp;      // [pairs][n] T, P and, for ill-conditioned chunks, T - bf16(T) (kTpBytes each)
    const uint8_t *recs;    // [pairs][n] prep records (the ill-conditioned flag)
    float *gq, *gk, *gb, *gla, *gv, *gw;
    int T, H, n;
    unsigned int *err;
};

// The gradients of chunk c of (batch bi, head h): one CTA of kGT threads, `sm`
// the 1024-byte aligned shared memory.  ILL: the chunk's T is far from the
// identity (the prep's flag), and T and X enter U = T X and dX = T^T gU as bf16
// pairs (hi + lo): U = T X_hi + T X_lo + T_lo X_hi, dX = T^T gU + T_lo^T gU, for
// U and dX are then alternating sums whose cancellation would amplify the
// roundings of bf16 T and X.  Returns false when a wait timed out (in-flight
// copies may then still land).
template <int DV, bool ILL>
__device__ __forceinline__ bool grad_chunk(const CUtensorMap &tm_q, const CUtensorMap &tm_k, const CUtensorMap &tm_b,
                                           const CUtensorMap &tm_do, const GradArgs &g, uint8_t *sm, int c, int h,
                                           int bi)
{
    using L = GradLayout;
    constexpr int NBV = DV / 64;           // 64-value blocks
    constexpr int SXB = 128 * DV * 2;      // bytes of a state image
    constexpr int HC = DV / 2;             // value columns per warp half in the M = 64 readouts
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int t0 = c * kChunk, Lc = min(kChunk, g.T - t0);
    const long pair = (long)bi * g.H + h, idx = pair * g.n + c;
    uint64_t *bar_ld = reinterpret_cast<uint64_t *>(sm + L::BAR), *bar_mma = bar_ld + 1, *bar_raw = bar_ld + 2;
    uint32_t *slot = reinterpret_cast<uint32_t *>(sm + L::SLOT);
    float *sig_s = reinterpret_cast<float *>(sm + L::SIG_S), *sig_d = reinterpret_cast<float *>(sm + L::SIG_D);
    float *grv = reinterpret_cast<float *>(sm + L::GRV), *gcv = reinterpret_cast<float *>(sm + L::GCV);
    float *qtot = reinterpret_cast<float *>(sm + L::QTOT), *qprod = reinterpret_cast<float *>(sm + L::QPROD);
    float *dgc = reinterpret_cast<float *>(sm + L::DGC), *diag = reinterpret_cast<float *>(sm + L::DIAG);
    const uint32_t sbase = smem_u32(sm);
    auto tok = [&](int t) { return ((long)bi * g.T + t0 + t) * g.H + h; };

    if (tid == 0) {
        mbar_init(bar_ld, 1);
        mbar_init(bar_mma, 1);
        mbar_init(bar_raw, 1);
        fence_mbar_init();
        mbar_arrive_expect_tx(bar_ld, (uint32_t)(3 * 16384 + NBV * 8192 + 2 * SXB + 16384 + (ILL ? 8192 : 0)));
        for (int kb = 0; kb < 2; ++kb) {
            tma_load_4d(sm + L::EQ + kb * 16384, &tm_b, bar_ld, kb * 64, h, t0, bi);
            tma_load_4d(sm + L::EQ + kb * 16384 + 8192, &tm_q, bar_ld, kb * 64, h, t0, bi);
            tma_load_4d(sm + L::KT + kb * 8192, &tm_k, bar_ld, kb * 64, h, t0, bi);
        }
        for (int kb = 0; kb < NBV; ++kb) tma_load_4d(sm + L::G + kb * 16384, &tm_do, bar_ld, kb * 64, h, t0, bi);
        bulk_load(sm + L::SR, g.sx + idx * SXB, SXB, bar_ld);
        bulk_load(sm + L::DSC, g.dsx + idx * SXB, SXB, bar_ld);
        bulk_load(sm + L::TT, g.tp + idx * kTpBytes, 16384, bar_ld);  // T, then P
        // T - bf16(T) (free space until dP and dA are read out)
        if (ILL) bulk_load(sm + L::DPA, g.tp + idx * kTpBytes + 16384, 8192, bar_ld);
    }
    if (warp == 0) {
        // (no relinquish: a flagged chunk allocates again for its second pass)
        tmem_alloc(slot, L::TMEM_COLS);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *slot;
    uint32_t mph = 0;
    // M = 64 accumulators: row t = 16 wq + l sits in lane 32 wq + l (l < 16)
    const int wq = warp & 3, wh = warp >> 2;
    const int tr = 16 * wq + lane;
    const bool row_on = lane < 16;
    const bool row_live = row_on && tr < Lc;
    const uint32_t lbase = tmem + ((uint32_t)(32 * wq) << 16);
    // v and w of this thread's row and value columns [wh HC, +HC), fetched while the first
    // UMMAs run and kept for both readouts
    constexpr int NV = HC / 8;
    uint4 pv[NV], pw[NV];
    auto fetch_vw = [&]() {
#pragma unroll
        for (int i = 0; i < NV; ++i) {
            pv[i] = pw[i] = make_uint4(0, 0, 0, 0);
            if (row_live) {
                pv[i] = __ldg(reinterpret_cast<const uint4 *>(g.v + tok(tr) * DV + wh * HC + 8 * i));
                pw[i] = __ldg(reinterpret_cast<const uint4 *>(g.w + tok(tr) * DV + wh * HC + 8 * i));
            }
        }
    };
    auto mma_done = [&]() {
        const bool mine = (tid == 0) ? mbar_wait(bar_mma, mph, g.err) : true;
        mph ^= 1;
        const bool all = named_bar_and(kBar, kGT, mine) != 0;
        tc_fence_after();
        return all;
    };

    // ------------------------------------------------------------------ Gamma
    // thread (p, qr): key channels 2p, 2p+1 of tokens [16 qr, +16)
    const int p = tid & 63, qr = tid >> 6;
    float2 gam[16];  // Gamma (chunk-local, inclusive) of this thread's tokens
    float gr0, gr1;
    bool bounded;
    {
#pragma unroll
        for (int u = 0; u < 16; ++u) {
            const int t = qr * 16 + u;
            gam[u] = t < Lc ? __ldg(reinterpret_cast<const float2 *>(g.la + tok(t) * kDK + 2 * p)) : make_float2(0.f, 0.f);
        }
        float g0 = 0.f, g1 = 0.f;
#pragma unroll
        for (int u = 0; u < 16; ++u) {
            g0 += gam[u].x; g1 += gam[u].y;
            gam[u] = make_float2(g0, g1);
        }
        qtot[qr * kDK + 2 * p] = g0;
        qtot[qr * kDK + 2 * p + 1] = g1;
        // the forward prep's test: the midpoint split when every 16-token quarter
        // decays by at most e^{-40} (same sums, same order)
        bounded = !named_bar_and(kBar, kGT, (g0 >= -0.5f * kMidpointLogDecayRange) &&
                                                (g1 >= -0.5f * kMidpointLogDecayRange));
        float pre0 = 0.f, pre1 = 0.f, gc0 = 0.f, gc1 = 0.f;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float a0 = qtot[q * kDK + 2 * p], a1 = qtot[q * kDK + 2 * p + 1];
            if (q < qr) { pre0 += a0; pre1 += a1; }
            gc0 += a0; gc1 += a1;
        }
        gr0 = bounded ? 0.f : qtot[2 * p] + qtot[kDK + 2 * p];
        gr1 = bounded ? 0.f : qtot[2 * p + 1] + qtot[kDK + 2 * p + 1];
#pragma unroll
        for (int u = 0; u < 16; ++u) gam[u] = make_float2(gam[u].x + pre0, gam[u].y + pre1);
        if (qr == 0) {
            gcv[2 * p] = gc0; gcv[2 * p + 1] = gc1;
            grv[2 * p] = gr0; grv[2 * p + 1] = gr1;
            sig_s[2 * p] = bounded ? 1.f : expf(gr0);
            sig_s[2 * p + 1] = bounded ? 1.f : expf(gr1);
            sig_d[2 * p] = bounded ? 1.f : expf(gc0 - gr0);
            sig_d[2 * p + 1] = bounded ? 1.f : expf(gc1 - gr1);
        }
    }
    bool ok = named_bar_and(kBar, kGT, (tid == 0) ? mbar_wait(bar_ld, 0, g.err) : true) != 0;

    if (ok) {
        // -------------------------------------------- rowsum(dS' o e^{Gamma_C} S), then the row scalings
        // 16-byte pieces of the images: piece i holds row j = i % 128, columns 8 (i / 128) + [0, 8)
        const int j = tid & 127;
        float acc = 0.f;
#pragma unroll 4
        for (int m = 0; m < DV / 16; ++m) {
            const int i = tid + m * kGT;
            uint4 *dp = reinterpret_cast<uint4 *>(sm + L::DSC + i * 16);
            uint4 *sp = reinterpret_cast<uint4 *>(sm + L::SR + i * 16);
            float a[8], bq[8];
            unpack8(*dp, a);
            unpack8(*sp, bq);
#pragma unroll
            for (int u = 0; u < 8; ++u) acc = fmaf(a[u], bq[u], acc);
            if (!bounded) {
                const float ss = sig_s[j], sd = sig_d[j];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    a[u] *= sd;
                    bq[u] *= ss;
                }
                *dp = pack8(a);
                *sp = pack8(bq);
            }
        }
        dgc[(tid >> 7) * kDK + j] = acc * expf(gcv[j]);

        // -------------------------------------------- factors in place (two channels of 16 tokens a thread)
        const int hb = p >> 5, cbyte = (2 * p & 63) * 2;
        float2 sf[16], pf[16];  // the factor of E and Q, and that of K, per token
        if (!bounded) {
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                const float x0 = gam[u].x - gr0, x1 = gam[u].y - gr1;
                sf[u] = make_float2(ex2_approx(x0 * kLog2e), ex2_approx(x1 * kLog2e));
                pf[u] = make_float2(ex2_approx(-x0 * kLog2e), ex2_approx(-x1 * kLog2e));
            }
        } else {
            // running products of alpha: e^{Gamma_t} = prod_{u <= t} alpha_u and
            // e^{Gamma_C - Gamma_t} = prod_{u > t} alpha_u, never an inverse decay
            float2 al[16];
            float q0 = 1.f, q1 = 1.f;
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                const int t = qr * 16 + u;
                const float2 l = t < Lc ? __ldg(reinterpret_cast<const float2 *>(g.la + tok(t) * kDK + 2 * p))
                                        : make_float2(0.f, 0.f);
                al[u] = make_float2(ex2_approx(l.x * kLog2e), ex2_approx(l.y * kLog2e));
                q0 *= al[u].x; q1 *= al[u].y;
            }
            qprod[qr * kDK + 2 * p] = q0;
            qprod[qr * kDK + 2 * p + 1] = q1;
            named_bar(kBar, kGT);
            float pre0 = 1.f, pre1 = 1.f, post0 = 1.f, post1 = 1.f;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float a0 = qprod[q * kDK + 2 * p], a1 = qprod[q * kDK + 2 * p + 1];
                if (q < qr) { pre0 *= a0; pre1 *= a1; }
                if (q > qr) { post0 *= a0; post1 *= a1; }
            }
#pragma unroll
            for (int u = 15; u >= 0; --u) {
                pf[u] = make_float2(post0, post1);
                post0 *= al[u].x; post1 *= al[u].y;
            }
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                pre0 *= al[u].x; pre1 *= al[u].y;
                sf[u] = make_float2(pre0, pre1);
            }
        }
#pragma unroll
        for (int u = 0; u < 16; ++u) {
            const int t = qr * 16 + u;
            const uint32_t off = swz_off(t, cbyte, 128);
            __nv_bfloat162 *ep = reinterpret_cast<__nv_bfloat162 *>(sm + L::EQ + hb * 16384 + off);
            __nv_bfloat162 *qp = reinterpret_cast<__nv_bfloat162 *>(sm + L::EQ + hb * 16384 + 8192 + off);
            __nv_bfloat162 *kp = reinterpret_cast<__nv_bfloat162 *>(sm + L::KT + hb * 8192 + off);
            const float2 bv = __bfloat1622float2(*ep), qv = __bfloat1622float2(*qp), kv = __bfloat1622float2(*kp);
            *ep = __floats2bfloat162_rn(sf[u].x * bv.x * kv.x, sf[u].y * bv.y * kv.y);
            *qp = __floats2bfloat162_rn(sf[u].x * qv.x, sf[u].y * qv.y);
            *kp = __floats2bfloat162_rn(pf[u].x * kv.x, pf[u].y * kv.y);
        }
        fence_proxy_async_smem();
        named_bar(kBar, kGT);

        // -------------------------------------------- Ebar S (M = 64) and gU = Ktil dS' + P^T dO
        if (tid == 0) {
            tc_fence_after();
            const uint32_t id = idesc_bf16(64, DV, 0, 1), idp = idesc_bf16(64, DV, 1, 1);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
                umma_bf16(tmem + L::TM_DX0,
                          smem_desc(sbase + L::EQ + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024, kSw128),
                          smem_desc(sbase + L::SR + ks * 256, 128, 2048, kSwNone), id, ks > 0);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
                umma_bf16(tmem + L::TM_GU,
                          smem_desc(sbase + L::KT + (ks >> 2) * 8192 + (ks & 3) * 32, 16, 1024, kSw128),
                          smem_desc(sbase + L::DSC + ks * 256, 128, 2048, kSwNone), id, ks > 0);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                umma_bf16(tmem + L::TM_GU, smem_desc(sbase + L::PP + ks * 2048, 8192, 1024, kSw128),
                          smem_desc(sbase + L::G + ks * 2048, 16384, 1024, kSw128), idp, 1);
            umma_commit(bar_mma);
        }
        fetch_vw();
        ok = mma_done();
    }

    if (ok) {
        // -------------------------------------------- X = Z - Ebar S -> XG;  gU -> U (bf16, rows = tokens)
#pragma unroll
        for (int cc = 0; cc < HC; cc += 32) {
            const int col = wh * HC + cc;
            float d[32], gu[32];
            __syncwarp();
            tmem_ld32(lbase + L::TM_DX0 + col, d);
            tmem_ld32(lbase + L::TM_GU + col, gu);
            tmem_ld_wait();
            if (row_on) {
#pragma unroll
                for (int q8 = 0; q8 < 4; ++q8) {
                    const int cb = col + q8 * 8;
                    float z[8], fv[8], fw[8];
                    unpack8(pv[cc / 8 + q8], fv);
                    unpack8(pw[cc / 8 + q8], fw);
#pragma unroll
                    for (int u = 0; u < 8; ++u) z[u] = fv[u] * fw[u] - d[q8 * 8 + u];
                    const uint32_t sw = swz_off(tr, (cb & 63) * 2, 128);
                    const uint32_t off = (uint32_t)((cb >> 6) * 8192) + sw;
                    *reinterpret_cast<uint4 *>(sm + L::XG + off) = pack8(z);
                    *reinterpret_cast<uint4 *>(sm + L::U + off) = pack8(gu + q8 * 8);
                    if (ILL) {  // X - bf16(X) into the -dX half of G (free until dX is read out)
#pragma unroll
                        for (int u = 0; u < 8; ++u) z[u] -= __bfloat162float(__float2bfloat16_rn(z[u]));
                        *reinterpret_cast<uint4 *>(sm + L::G + (cb >> 6) * 16384 + 8192 + sw) = pack8(z);
                    }
                }
            }
        }
        tc_fence_before();
        fence_proxy_async_smem();
        named_bar(kBar, kGT);

        // -------------------------------------------- U = T X,  dX = T^T gU
        // In ill-conditioned chunks (the prep's flag) T and X are bf16 pairs (hi + lo):
        // U = T X_hi + T X_lo + T_lo X_hi and dX = T^T gU + T_lo^T gU, as U and dX
        // are alternating sums whose cancellation would amplify the roundings of
        // bf16 T and X.
        if (tid == 0) {
            tc_fence_after();
            const uint32_t id = idesc_bf16(64, DV, 0, 1), idt = idesc_bf16(64, DV, 1, 1);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                const uint64_t xh = smem_desc(sbase + L::XG + ks * 2048, 8192, 1024, kSw128);
                umma_bf16(tmem + L::TM_U, smem_desc(sbase + L::TT + ks * 32, 16, 1024, kSw128), xh, id, ks > 0);
                if (ILL) {
                    umma_bf16(tmem + L::TM_U, smem_desc(sbase + L::TT + ks * 32, 16, 1024, kSw128),
                              smem_desc(sbase + L::G + 8192 + ks * 2048, 16384, 1024, kSw128), id, 1);
                    umma_bf16(tmem + L::TM_U, smem_desc(sbase + L::DPA + ks * 32, 16, 1024, kSw128), xh, id, 1);
                }
            }
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                const uint64_t gu = smem_desc(sbase + L::U + ks * 2048, 8192, 1024, kSw128);
                umma_bf16(tmem + L::TM_DX, smem_desc(sbase + L::TT + ks * 2048, 8192, 1024, kSw128), gu, idt, ks > 0);
                if (ILL)
                    umma_bf16(tmem + L::TM_DX, smem_desc(sbase + L::DPA + ks * 2048, 8192, 1024, kSw128), gu, idt, 1);
            }
            umma_commit(bar_mma);
        }
        ok = mma_done();
    }

    if (ok) {
        // -------------------------------------------- U -> U;  dv, dw (v and w still in registers);  -dX -> G
#pragma unroll
        for (int cc = 0; cc < HC; cc += 32) {
            const int col = wh * HC + cc;
            float uu[32], dx[32];
            __syncwarp();
            tmem_ld32(lbase + L::TM_U + col, uu);
            tmem_ld32(lbase + L::TM_DX + col, dx);
            tmem_ld_wait();
            if (row_on) {
#pragma unroll
                for (int q8 = 0; q8 < 4; ++q8) {
                    const int cb = col + q8 * 8;
                    const uint32_t sw = swz_off(tr, (cb & 63) * 2, 128);
                    *reinterpret_cast<uint4 *>(sm + L::U + (cb >> 6) * 8192 + sw) = pack8(uu + q8 * 8);
                    float nd[8];
#pragma unroll
                    for (int u = 0; u < 8; ++u) nd[u] = -dx[q8 * 8 + u];
                    *reinterpret_cast<uint4 *>(sm + L::G + (cb >> 6) * 16384 + 8192 + sw) = pack8(nd);
                    if (row_live) {
                        float fv[8], fw[8];
                        unpack8(pv[cc / 8 + q8], fv);
                        unpack8(pw[cc / 8 + q8], fw);
                        float4 *ov = reinterpret_cast<float4 *>(g.gv + tok(tr) * DV + cb);
                        float4 *ow = reinterpret_cast<float4 *>(g.gw + tok(tr) * DV + cb);
                        const float *x = dx + q8 * 8;
                        ov[0] = make_float4(x[0] * fw[0], x[1] * fw[1], x[2] * fw[2], x[3] * fw[3]);
                        ov[1] = make_float4(x[4] * fw[4], x[5] * fw[5], x[6] * fw[6], x[7] * fw[7]);
                        ow[0] = make_float4(x[0] * fv[0], x[1] * fv[1], x[2] * fv[2], x[3] * fv[3]);
                        ow[1] = make_float4(x[4] * fv[4], x[5] * fv[5], x[6] * fv[6], x[7] * fv[7]);
                    }
                }
            }
        }
        tc_fence_before();
        fence_proxy_async_smem();
        named_bar(kBar, kGT);

        // -------------------------------------------- [dP; dA] = [dO; -dX] U^T (M = 128),
        // dq' = dO S_r^T, de' = -dX S_r^T, dk' = U dS_c^T (M = 64)
        if (tid == 0) {
            tc_fence_after();
            const uint32_t id5 = idesc_bf16(128, 64, 0, 0), id6 = idesc_bf16(64, kDK, 0, 0);
#pragma unroll
            for (int ks = 0; ks < DV / 16; ++ks)
                umma_bf16(tmem + L::TM_DPA,
                          smem_desc(sbase + L::G + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024, kSw128),
                          smem_desc(sbase + L::U + (ks >> 2) * 8192 + (ks & 3) * 32, 16, 1024, kSw128), id5, ks > 0);
            // S_r^T, dS_c^T: the images read K-major (8-value K chunks of 2 KB, 8-row groups of 128 bytes)
#pragma unroll
            for (int ks = 0; ks < DV / 16; ++ks) {
                const uint64_t bs = smem_desc(sbase + L::SR + ks * 4096, 2048, 128, kSwNone);
                const uint32_t ga = L::G + (ks >> 2) * 16384 + (ks & 3) * 32;
                umma_bf16(tmem + L::TM_DQ, smem_desc(sbase + ga, 16, 1024, kSw128), bs, id6, ks > 0);
                umma_bf16(tmem + L::TM_DE, smem_desc(sbase + ga + 8192, 16, 1024, kSw128), bs, id6, ks > 0);
                umma_bf16(tmem + L::TM_DK,
                          smem_desc(sbase + L::U + (ks >> 2) * 8192 + (ks & 3) * 32, 16, 1024, kSw128),
                          smem_desc(sbase + L::DSC + ks * 4096, 2048, 128, kSwNone), id6, ks > 0);
            }
            umma_commit(bar_mma);
        }
        ok = mma_done();
    }

    if (ok) {
        // raw q, b and k for the epilogue, into tiles whose products have completed
        if (tid == 0 && !bounded) {
            mbar_arrive_expect_tx(bar_raw, 3 * 16384);
            for (int kb = 0; kb < 2; ++kb) {
                tma_load_4d(sm + L::TQ + kb * 8192, &tm_q, bar_raw, kb * 64, h, t0, bi);
                tma_load_4d(sm + L::TB + kb * 8192, &tm_b, bar_raw, kb * 64, h, t0, bi);
                tma_load_4d(sm + L::TK + kb * 8192, &tm_k, bar_raw, kb * 64, h, t0, bi);
            }
        }
        // -------------------------------------------- [dP; dA] strictly lower -> DPA (bf16, rows t / 64 + t);
        // the diagonal of dP (fp32) -> diag
        {
            const int r = 32 * wq + lane, t = r & 63;
            float v[32];
            tmem_ld32(lbase + L::TM_DPA + wh * 32, v);
            tmem_ld_wait();
#pragma unroll
            for (int s8 = 0; s8 < 4; ++s8) {
                const int s0 = wh * 32 + s8 * 8;
                float f[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    f[u] = (s0 + u < t) ? v[s8 * 8 + u] : 0.f;
                    if (r < 64 && s0 + u == t) diag[t] = v[s8 * 8 + u];
                }
                *reinterpret_cast<uint4 *>(sm + L::DPA + swz_off(r, s0 * 2, 128)) = pack8(f);
            }
        }
        if (!bounded) {
            // x = Gamma - Gamma_r of every (token, channel), for the epilogue
            float *xs = reinterpret_cast<float *>(sm + L::XST);
#pragma unroll
            for (int u = 0; u < 16; ++u)
                *reinterpret_cast<float2 *>(xs + fo(qr * 16 + u, 2 * p)) =
                    make_float2(gam[u].x - gr0, gam[u].y - gr1);
        } else {
            // raw q, b, k (bf16 rows of 128 channels) and alpha, e^{Gamma}, e^{Gamma_C - Gamma}
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const int i = tid + m * kGT, t = i >> 4, c8 = (i & 15) * 8;
                uint4 rq = make_uint4(0, 0, 0, 0), rb = rq, rk = rq;
                if (t < Lc) {
                    rq = __ldg(reinterpret_cast<const uint4 *>(g.q + tok(t) * kDK + c8));
                    rb = __ldg(reinterpret_cast<const uint4 *>(g.b + tok(t) * kDK + c8));
                    rk = __ldg(reinterpret_cast<const uint4 *>(g.k + tok(t) * kDK + c8));
                }
                *reinterpret_cast<uint4 *>(sm + L::RQ + t * 256 + c8 * 2) = rq;
                *reinterpret_cast<uint4 *>(sm + L::RB + t * 256 + c8 * 2) = rb;
                *reinterpret_cast<uint4 *>(sm + L::RK + t * 256 + c8 * 2) = rk;
            }
            float *alp = reinterpret_cast<float *>(sm + L::ALPHA);
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                const int t = qr * 16 + u;
                const float2 l = t < Lc ? __ldg(reinterpret_cast<const float2 *>(g.la + tok(t) * kDK + 2 * p))
                                        : make_float2(0.f, 0.f);
                *reinterpret_cast<float2 *>(alp + fo(t, 2 * p)) =
                    make_float2(ex2_approx(l.x * kLog2e), ex2_approx(l.y * kLog2e));
            }
        }
        tc_fence_before();
        fence_proxy_async_smem();
        named_bar(kBar, kGT);

        // -------------------------------------------- dq' += dP Khat, de' += dA Khat, dk2 = dP^T Qhat + dA^T Ehat
        if (tid == 0) {
            tc_fence_after();
            if (!bounded) {
                const uint32_t id = idesc_bf16(64, kDK, 0, 1), idt = idesc_bf16(64, kDK, 1, 1);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {
                    const uint64_t kh = smem_desc(sbase + L::KT + ks * 2048, 8192, 1024, kSw128);
                    umma_bf16(tmem + L::TM_DQ, smem_desc(sbase + L::DPA + ks * 32, 16, 1024, kSw128), kh, id, 1);
                    umma_bf16(tmem + L::TM_DE, smem_desc(sbase + L::DPA + 8192 + ks * 32, 16, 1024, kSw128), kh,
                              id, 1);
                }
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {
                    umma_bf16(tmem + L::TM_DK2, smem_desc(sbase + L::DPA + ks * 2048, 8192, 1024, kSw128),
                              smem_desc(sbase + L::EQ + 8192 + ks * 2048, 16384, 1024, kSw128), idt, ks > 0);
                    umma_bf16(tmem + L::TM_DK2, smem_desc(sbase + L::DPA + 8192 + ks * 2048, 8192, 1024, kSw128),
                              smem_desc(sbase + L::EQ + ks * 2048, 16384, 1024, kSw128), idt, 1);
                }
            }
            umma_commit(bar_mma);
        }
        ok = mma_done();
    }

    if (ok) {
        // -------------------------------------------- per (token, channel): dq, dk, db, dGamma and K
        const float *xs = reinterpret_cast<const float *>(sm + L::XST);
        const float *alp = reinterpret_cast<const float *>(sm + L::ALPHA);
        float *dgs = reinterpret_cast<float *>(sm + L::DGS), *kst = reinterpret_cast<float *>(sm + L::KST);
        if (!bounded) ok = named_bar_and(kBar, kGT, (tid == 0) ? mbar_wait(bar_raw, 0, g.err) : true) != 0;
#pragma unroll 1
        for (int pass = 0; pass < 4 && ok; ++pass) {
            const int j0 = wh * 64 + pass * 16;
            float aq[16], ae[16], ak[16], ap[16];
            __syncwarp();
            tmem_ld16(lbase + L::TM_DQ + j0, aq);
            tmem_ld16(lbase + L::TM_DE + j0, ae);
            tmem_ld16(lbase + L::TM_DK + j0, ak);
            tmem_ld16(lbase + L::TM_DK2 + j0, ap);
            tmem_ld_wait();
            if (row_on) {
            const int t = tr;
            float qv[16], bv[16], kv[16], fq[16], fk[16];
            if (!bounded) {
                // (zero rows past the sequence end, from the TMA's fill)
#pragma unroll
                for (int h8 = 0; h8 < 16; h8 += 8) {
                    const uint32_t o = (uint32_t)((j0 >> 6) * 8192) + swz_off(t, ((j0 & 63) + h8) * 2, 128);
                    unpack8(*reinterpret_cast<const uint4 *>(sm + L::TQ + o), qv + h8);
                    unpack8(*reinterpret_cast<const uint4 *>(sm + L::TB + o), bv + h8);
                    unpack8(*reinterpret_cast<const uint4 *>(sm + L::TK + o), kv + h8);
                }
#pragma unroll
                for (int u4 = 0; u4 < 16; u4 += 4) {
                    const float4 x = *reinterpret_cast<const float4 *>(xs + fo(t, j0 + u4));
                    const float xv[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        fq[u4 + u] = ex2_approx(xv[u] * kLog2e);
                        fk[u4 + u] = ex2_approx(-xv[u] * kLog2e);
                    }
                }
#pragma unroll
                for (int u = 0; u < 16; ++u) {
                    aq[u] *= fq[u];
                    ae[u] *= fq[u];
                    ap[u] *= fk[u];
                }
            } else {
#pragma unroll
                for (int h8 = 0; h8 < 16; h8 += 8) {
                    unpack8(*reinterpret_cast<const uint4 *>(sm + L::RQ + t * 256 + (j0 + h8) * 2), qv + h8);
                    unpack8(*reinterpret_cast<const uint4 *>(sm + L::RB + t * 256 + (j0 + h8) * 2), bv + h8);
                    unpack8(*reinterpret_cast<const uint4 *>(sm + L::RK + t * 256 + (j0 + h8) * 2), kv + h8);
                }
                // pairwise terms with decays prod_{s < u <= t} alpha_u (running products),
                // strictly off the diagonal:
                //   dq_t += sum_{s < t} dP_ts k_s f_ts,  de_t += sum_{s < t} dA_ts k_s f_ts
                //   dk_t += sum_{t' > t} (dP_t't q_t' + dA_t't e_t') f_t't
                // the first walk ends with f = e^{Gamma_t}, the second with e^{Gamma_C - Gamma_t}
                float wq[16], we[16], f[16];
#pragma unroll
                for (int u = 0; u < 16; ++u) {
                    wq[u] = we[u] = ap[u] = 0.f;
                    f[u] = 1.f;
                }
#pragma unroll 1
                for (int s = t; s >= 0; --s) {
                    const float dp = __bfloat162float(*reinterpret_cast<const bf16 *>(sm + L::DPA + swz_off(t, 2 * s, 128)));
                    const float da = __bfloat162float(*reinterpret_cast<const bf16 *>(sm + L::DPA + swz_off(64 + t, 2 * s, 128)));
                    float ks_[16];
                    unpack8(*reinterpret_cast<const uint4 *>(sm + L::RK + s * 256 + j0 * 2), ks_);
                    unpack8(*reinterpret_cast<const uint4 *>(sm + L::RK + s * 256 + j0 * 2 + 16), ks_ + 8);
#pragma unroll
                    for (int u4 = 0; u4 < 16; u4 += 4) {
                        const float4 a = *reinterpret_cast<const float4 *>(alp + fo(s, j0 + u4));
                        const float av[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const float kf = ks_[u4 + u] * f[u4 + u];
                            wq[u4 + u] = fmaf(dp, kf, wq[u4 + u]);
                            we[u4 + u] = fmaf(da, kf, we[u4 + u]);
                            f[u4 + u] *= av[u];
                        }
                    }
                }
#pragma unroll
                for (int u = 0; u < 16; ++u) {
                    fq[u] = f[u];
                    aq[u] = fmaf(fq[u], aq[u], wq[u]);
                    ae[u] = fmaf(fq[u], ae[u], we[u]);
                    f[u] = 1.f;
                }
#pragma unroll 1
                for (int t2 = t; t2 < kChunk; ++t2) {
                    const float dp = __bfloat162float(*reinterpret_cast<const bf16 *>(sm + L::DPA + swz_off(t2, 2 * t, 128)));
                    const float da = __bfloat162float(*reinterpret_cast<const bf16 *>(sm + L::DPA + swz_off(64 + t2, 2 * t, 128)));
                    float q2[16], b2[16], k2[16];
                    unpack8(*reinterpret_cast<const uint4 *>(sm + L::RQ + t2 * 256 + j0 * 2), q2);
                    unpack8(*reinterpret_cast<const uint4 *>(sm + L::RQ + t2 * 256 + j0 * 2 + 16), q2 + 8);
                    unpack8(*reinterpret_cast<const uint4 *>(sm + L::RB + t2 * 256 + j0 * 2), b2);
                    unpack8(*reinterpret_cast<const uint4 *>(sm + L::RB + t2 * 256 + j0 * 2 + 16), b2 + 8);
                    unpack8(*reinterpret_cast<const uint4 *>(sm + L::RK + t2 * 256 + j0 * 2), k2);
                    unpack8(*reinterpret_cast<const uint4 *>(sm + L::RK + t2 * 256 + j0 * 2 + 16), k2 + 8);
#pragma unroll
                    for (int u = 0; u < 16; ++u) ap[u] = fmaf(fmaf(dp, q2[u], da * b2[u] * k2[u]), f[u], ap[u]);
                    if (t2 + 1 < kChunk) {
#pragma unroll
                        for (int u4 = 0; u4 < 16; u4 += 4) {
                            const float4 a = *reinterpret_cast<const float4 *>(alp + fo(t2 + 1, j0 + u4));
                            f[u4] *= a.x; f[u4 + 1] *= a.y; f[u4 + 2] *= a.z; f[u4 + 3] *= a.w;
                        }
                    }
                }
#pragma unroll
                for (int u = 0; u < 16; ++u) fk[u] = f[u];
            }
            // aq, ae: dq and de without the diagonal of P; ap: the pairwise part of
            // dk_write without it; kw = e^{Gamma_C - Gamma} (U dS'^T) Ktil's part:
            //   dq = aq + dP_tt k,  dk = kw + ap + dP_tt q + de b,  db = de k,
            //   dGamma (regrouped) = q aq + b k de - k ap,  K = k kw
            const float dpt = diag[t];
            const long ro = tok(t) * kDK + j0;
#pragma unroll
            for (int u4 = 0; u4 < 16; u4 += 4) {
                float gd[4], gk4[4], gb4[4], gq4[4], kk[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int x = u4 + u;
                    const float kw = fk[x] * ak[x];  // Ktil's part of dk_write
                    kk[u] = kv[x] * kw;
                    gq4[u] = fmaf(dpt, kv[x], aq[x]);
                    gb4[u] = ae[x] * kv[x];
                    gk4[u] = kw + ap[x] + fmaf(dpt, qv[x], ae[x] * bv[x]);
                    gd[u] = fmaf(qv[x], aq[x], fmaf(bv[x] * kv[x], ae[x], -kv[x] * ap[x]));
                    if (t == kChunk - 1) gd[u] += dgc[j0 + x] + dgc[kDK + j0 + x];
                }
                if (row_live) {
                    *reinterpret_cast<float4 *>(g.gq + ro + u4) = make_float4(gq4[0], gq4[1], gq4[2], gq4[3]);
                    *reinterpret_cast<float4 *>(g.gk + ro + u4) = make_float4(gk4[0], gk4[1], gk4[2], gk4[3]);
                    *reinterpret_cast<float4 *>(g.gb + ro + u4) = make_float4(gb4[0], gb4[1], gb4[2], gb4[3]);
                }
                *reinterpret_cast<float4 *>(dgs + fo(t, j0 + u4)) = make_float4(gd[0], gd[1], gd[2], gd[3]);
                *reinterpret_cast<float4 *>(kst + fo(t, j0 + u4)) = make_float4(kk[0], kk[1], kk[2], kk[3]);
            }
            }
        }
        named_bar(kBar, kGT);

        // -------------------------------------------- dlog_alpha_u = sum_{t >= u} dGamma_t + sum_{t < u} K_t
        {
            float2 dg[16], kp[16];
            float s0 = 0.f, s1 = 0.f, k0 = 0.f, k1 = 0.f;
#pragma unroll
            for (int u = 15; u >= 0; --u) {
                const float2 v = *reinterpret_cast<const float2 *>(dgs + fo(qr * 16 + u, 2 * p));
                s0 += v.x; s1 += v.y;
                dg[u] = make_float2(s0, s1);
            }
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                kp[u] = make_float2(k0, k1);
                const float2 v = *reinterpret_cast<const float2 *>(kst + fo(qr * 16 + u, 2 * p));
                k0 += v.x; k1 += v.y;
            }
            qtot[qr * kDK + 2 * p] = s0;
            qtot[qr * kDK + 2 * p + 1] = s1;
            qprod[qr * kDK + 2 * p] = k0;
            qprod[qr * kDK + 2 * p + 1] = k1;
            named_bar(kBar, kGT);
            float a0 = 0.f, a1 = 0.f;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                if (q > qr) { a0 += qtot[q * kDK + 2 * p]; a1 += qtot[q * kDK + 2 * p + 1]; }
                if (q < qr) { a0 += qprod[q * kDK + 2 * p]; a1 += qprod[q * kDK + 2 * p + 1]; }
            }
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                const int t = qr * 16 + u;
                if (t < Lc)
                    *reinterpret_cast<float2 *>(g.gla + tok(t) * kDK + 2 * p) =
                        make_float2(dg[u].x + kp[u].x + a0, dg[u].y + kp[u].y + a1);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, L::TMEM_COLS);
    }
    return ok;
}

// The bf16-pair pass, out of line: the plain pass keeps its schedule.
template <int DV>
__device__ __noinline__ void grad_chunk_pairs(const CUtensorMap &tm_q, const CUtensorMap &tm_k, const CUtensorMap &tm_b,
                                              const CUtensorMap &tm_do, const GradArgs &g, uint8_t *sm, int c, int h,
                                              int bi)
{
    grad_chunk<DV, true>(tm_q, tm_k, tm_b, tm_do, g, sm, c, h, bi);
}

// One CTA per (chunk, head, batch).  A chunk the prep flagged (T far from the
// identity) is computed twice: the plain pass, then the bf16-pair pass over its
// gradients.
template <int DV>
__global__ void __launch_bounds__(kGT, 1)
grad_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
            const __grid_constant__ CUtensorMap tm_b, const __grid_constant__ CUtensorMap tm_do,
            const __grid_constant__ GradArgs g)
{
    using L = GradLayout;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, c = blockIdx.x, h = blockIdx.y, bi = blockIdx.z;
    // the prep's flag, issued now and first used after the plain pass
    uint32_t flag = 0;
    if (tid == 0)
        flag = ld_nc_u32(g.recs + (((long)bi * g.H + h) * g.n + c) * (long)Record<DV>::BYTES + Record<DV>::DEC + 512);
    const bool ok = grad_chunk<DV, false>(tm_q, tm_k, tm_b, tm_do, g, sm, c, h, bi);
    // (the second pass's copies land where the first pass's threads wrote)
    fence_proxy_async_smem();
    if (__syncthreads_or(flag != 0) && ok) {
        if (tid == 0) {
            uint64_t *bar = reinterpret_cast<uint64_t *>(sm + L::BAR);
            mbar_inval(bar);
            mbar_inval(bar + 1);
            mbar_inval(bar + 2);
        }
        grad_chunk_pairs<DV>(tm_q, tm_k, tm_b, tm_do, g, sm, c, h, bi);
    }
}

// Both chains of the backward: CTAs x < DV / DVT run the forward chain of value
// tile x of one (batch, head), the others the adjoint chain of tile x - DV / DVT.
template <int DV, int DVT>
__global__ void __launch_bounds__(chain::kChainThreads, 1)
chains_kernel(const __grid_constant__ CUtensorMap tm_do, const uint8_t *__restrict__ recs, uint8_t *__restrict__ sx,
              uint8_t *__restrict__ dsx, const float *S0, const float *dS_T, float *dS0, int H, int n,
              unsigned int *err)
{
    using CL = chain::ChainLayout<DV, DVT>;
    constexpr int NT = DV / DVT;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5;
    const bool adj = (int)blockIdx.x >= NT;
    const int tile = adj ? (int)blockIdx.x - NT : (int)blockIdx.x, h = blockIdx.y, bi = blockIdx.z;
    uint32_t *slot = reinterpret_cast<uint32_t *>(sm + CL::SLOT);
    const long pair = (long)bi * H + h;
    if (tid == 0) chain::chain_init<DV, DVT>(sm);
    if (warp == 0) {
        tmem_alloc(slot, CL::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *slot;
    const uint8_t *r = recs + pair * n * (long)Record<DV>::BYTES;
    if (adj) {
        const chain::ReverseFlow<DV> f{r, dsx + pair * n * (long)SxSlot<DV>::BYTES, &tm_do, n, h, bi};
        chain::chain_run<DV, DVT, chain::ReverseFlow<DV>, true>(sm, tmem, tid, f, dS_T, dS0, pair, tile, n, err);
    } else {
        const chain::WindowFlow<DV> f{r, sx + pair * n * (long)SxSlot<DV>::BYTES};
        chain::chain_run<DV, DVT>(sm, tmem, tid, f, S0, nullptr, pair, tile, n, err);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, CL::TMEM_COLS);
    }
}

struct Plan {
    long pairs;
    int n;            // chunks
    size_t rec, tp, sx, dsx, total;
};

Plan plan(int B, int T, int H, int dv)
{
    Plan p{};
    p.pairs = (long)B * H;
    p.n = (T + kChunk - 1) / kChunk;
    const size_t rb = dv == 128 ? Record<128>::BYTES : Record<64>::BYTES;
    const size_t xb = dv == 128 ? SxSlot<128>::BYTES : SxSlot<64>::BYTES;
    const size_t per = (size_t)p.pairs * p.n;
    size_t off = 0;
    p.rec = off; off += per * rb;
    p.tp = off; off += per * kTpBytes;
    p.sx = off; off += per * xb;
    p.dsx = off; off += per * xb;
    p.total = off;
    return p;
}

template <int DV, int DVT>
cudaError_t launch_chains(const CUtensorMap &tm_do, const uint8_t *recs, uint8_t *sx, uint8_t *dsx, const float *S0,
                          const float *dS_T, float *dS0, int B, int H, int n, cudaStream_t s, unsigned int *err)
{
    using CL = chain::ChainLayout<DV, DVT>;
    auto kern = chains_kernel<DV, DVT>;
    static std::atomic<unsigned long long> smem_set{0};
    cudaError_t e = ensure_smem_limit(kern, CL::BYTES, smem_set);
    if (e != cudaSuccess) return e;
    kern<<<dim3(2 * (DV / DVT), H, B), chain::kChainThreads, CL::BYTES, s>>>(tm_do, recs, sx, dsx, S0, dS_T, dS0, H,
                                                                               n, err);
    return cudaGetLastError();
}

template <int DV>
cudaError_t launch_grad(const CUtensorMap *maps, const GradArgs &ga, int B, cudaStream_t s)
{
    auto kern = grad_kernel<DV>;
    static std::atomic<unsigned long long> smem_set{0};
    cudaError_t e = ensure_smem_limit(kern, GradLayout::BYTES, smem_set);
    if (e != cudaSuccess) return e;
    kern<<<dim3(ga.n, ga.H, B), kGT, GradLayout::BYTES, s>>>(maps[0], maps[1], maps[2], maps[3], ga);
    return cudaGetLastError();
}

}  // namespace bwdtc

size_t bwd_tc_workspace_bytes(int B, int T, int H, int dv) { return bwdtc::plan(B, T, H, dv).total; }

cudaError_t launch_bwd_tc(const BwdArgs &a, uint8_t *ws, unsigned int *err, int num_sms)
{
    using namespace bwdtc;
    const Plan pl = plan(a.B, a.T, a.H, a.dv);
    uint8_t *recs = ws + pl.rec, *tp = ws + pl.tp, *sx = ws + pl.sx, *dsx = ws + pl.dsx;

    FwdArgs f{};
    f.q = a.q; f.k = a.k; f.v = a.v; f.b = a.b; f.w = a.w; f.log_alpha = a.log_alpha;
    f.S0 = a.S0; f.o = nullptr; f.S_T = nullptr;
    f.B = a.B; f.T = a.T; f.H = a.H; f.dk = a.dk; f.dv = a.dv;
    f.bf16 = true; f.layout = 0; f.stream = a.stream; f.err = err; f.num_sms = num_sms;
    CUtensorMap fmaps[5];
    if (!make_input_maps(f, fmaps)) return cudaErrorInvalidValue;
    // maps of grad_kernel: q, k, b, dO
    CUtensorMap gmaps[4];
    gmaps[0] = fmaps[0];
    gmaps[1] = fmaps[1];
    gmaps[2] = fmaps[2];
    if (!make_token_map(&gmaps[3], a.dO, a.dv, a.H, a.T, a.B)) return cudaErrorInvalidValue;

    // value tiles of the chains: 64 wide while both chains' CTAs (four per pair) fit the SMs
    const int dvt = (a.dv == 64 || pl.pairs * 4 <= num_sms) ? 64 : 128;
    cudaError_t e = launch_prep(f, fmaps, recs, 0, pl.n, pl.n, false, tp);
    if (e == cudaSuccess) {
        if (a.dv == 64)
            e = launch_chains<64, 64>(gmaps[3], recs, sx, dsx, a.S0, a.dS_T, a.dS0, a.B, a.H, pl.n, a.stream, err);
        else if (dvt == 64)
            e = launch_chains<128, 64>(gmaps[3], recs, sx, dsx, a.S0, a.dS_T, a.dS0, a.B, a.H, pl.n, a.stream, err);
        else
            e = launch_chains<128, 128>(gmaps[3], recs, sx, dsx, a.S0, a.dS_T, a.dS0, a.B, a.H, pl.n, a.stream,
                                        err);
    }
    if (e == cudaSuccess) {
        GradArgs ga{};
        ga.q = (const bf16 *)a.q; ga.k = (const bf16 *)a.k; ga.b = (const bf16 *)a.b;
        ga.v = (const bf16 *)a.v; ga.w = (const bf16 *)a.w; ga.la = a.log_alpha;
        ga.sx = sx; ga.dsx = dsx; ga.tp = tp; ga.recs = recs;
        ga.gq = a.gq; ga.gk = a.gk; ga.gb = a.gb; ga.gla = a.gla; ga.gv = a.gv; ga.gw = a.gw;
        ga.T = a.T; ga.H = a.H; ga.n = pl.n; ga.err = err;
        e = a.dv == 128 ? launch_grad<128>(gmaps, ga, a.B, a.stream) : launch_grad<64>(gmaps, ga, a.B, a.stream);
    }
    return e;
}

}  // namespace gdn2
