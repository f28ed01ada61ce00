// bwd_simt.cu -- the chunkwise backward of the operator on the fp32 pipes.
//
// Gradients of L = sum(o * dO) + sum(S_T * dS_T) with respect to q, k, v, b,
// w, log_alpha and S0, chunkwise over 64-token chunks ("Gated DeltaNet-2",
// iplexlaw.co.kr, section "Procesamiento del token y entrenamiento paralelo":
// the WY form over 64-token blocks, whose backward must use the modulated keys
// and values -- the per-channel gates cannot be pulled out as a scalar beta).
//
// Per chunk, with S the state entering it, dS' = dL/dS at its end, Gamma the
// chunk-local cumulative log-decay, E = b (*) k the erase keys, A and P the
// strictly lower and lower Grams of the decayed erase keys and queries against
// the keys, T = (I + A)^{-1}, Ebar = e^{Gamma} (*) E and Ktil = e^{Gamma_C-Gamma} (*) k
// (derived from the token recurrence):
//   forward   U = T (Z - Ebar S),   S_next = e^{Gamma_C} (*) S + Ktil^T U
//   adjoint   dU = T^T (Ktil dS' + P^T dO)   (= dZ: dv = dU (*) w, dw = dU (*) v)
//             dS = e^{Gamma_C} (*) dS' + sum_t e^{Gamma_t} (*) (q_t dO_t^T - E_t dU_t^T)
//   dq_t = e^{Gamma_t} (*) (S dO_t) + sum_{s<=t} (dO_t . u_s) e^{Gamma_t-Gamma_s} (*) k_s
//   de_t = -e^{Gamma_t} (*) (S dU_t) - sum_{s<t} (dU_t . u_s) e^{Gamma_t-Gamma_s} (*) k_s
//   dk_t (write) = e^{Gamma_C-Gamma_t} (*) (dS' u_t) + sum_{s>=t} (dO_s . u_t) e^{Gamma_s-Gamma_t} (*) q_s
//                  - sum_{s>t} (dU_s . u_t) e^{Gamma_s-Gamma_t} (*) E_s
//   db_t = de_t (*) k_t,   dk_t = dk_t (write) + de_t (*) b_t
//   dGamma_t = q_t (*) dq_t + E_t (*) de_t - k_t (*) dk_t (write)   (+ rowsum(dS' (*) S_next)
//              at the chunk end); dlog_alpha is its reverse cumulative sum over the chunk.
// Every decay between two tokens is a running product of alpha (a decay, <= 1),
// so no factor can overflow and any log_alpha <= 0 (-inf included) is exact.
//
// Four kernels:
//   gram   (per chunk and head, all in parallel)  A and P by running products; T;
//          the decayed factors Ebar, Qbar, Ktil and e^{Gamma_C}
//   fwd    (per head and 8-column value tile, chunks in order)  the state entering
//          each chunk (checkpoint) and U
//   adj    (per head and value tile, chunks in reverse)  the adjoint at each chunk's
//          end, dU, dv, dw, dS0
//   grad   (per chunk and head, all in parallel, every value column)  dq, dk, db,
//          dlog_alpha; the sums over the value axis stay inside the CTA.
#include "common.cuh"
#include "launch.h"

namespace gdn2 {
namespace {

constexpr int kBwdThreads = 256;
constexpr int kChainDvTile = 8;  // value columns of a chain CTA (fwd, adj)
constexpr int C = kChunk;
constexpr int LDC = kChunk + 1;

// Workspace of one call, per (batch, head) pair and chunk, fp32.
struct BwdWs {
    float *T, *P;   // [pair][nch][C][C]
    float *ck;      // [pair][nch + 1][dk][dv]: the state entering each chunk, and S_T
    float *U, *dU;  // [pair][nch][C][dv]
    float *dS;      // [pair][nch][dk][dv]: dL/dS at the end of each chunk
    // decayed factors [pair][nch][C][dk]: Ebar = e^{Gamma} b k, Qbar = e^{Gamma} q,
    // Ktil = e^{Gamma_C - Gamma} k; and e^{Gamma_C} [pair][nch][dk]
    float *Eb, *Qb, *Kt, *gC;
};

// Chunk inputs into shared memory ([C][DK + 1] fp32; zero past the sequence end, alpha = 1 there).
template <typename T, int DK, int NT = kBwdThreads>
__device__ __forceinline__ void load_rows(float *dst, const T *src, int tid, long bi, int Tlen, int H, int h, int t0,
                                          int Lc)
{
    for (int idx = tid; idx < C * DK; idx += NT) {
        const int t = idx / DK, i = idx % DK;
        dst[t * (DK + 1) + i] = (t < Lc) ? to_f32(src[((bi * Tlen + t0 + t) * H + h) * (long)DK + i]) : 0.f;
    }
}
template <int DK, int NT = kBwdThreads>
__device__ __forceinline__ void load_alpha(float *dst, const float *la, int tid, long bi, int Tlen, int H, int h,
                                           int t0, int Lc)
{
    for (int idx = tid; idx < C * DK; idx += NT) {
        const int t = idx / DK, i = idx % DK;
        dst[t * (DK + 1) + i] = (t < Lc) ? expf(la[((bi * Tlen + t0 + t) * H + h) * (long)DK + i]) : 1.f;
    }
}

// ------------------------------------------------------------------ gram
template <int DK>
struct GramSmem {
    static constexpr int LDK = DK + 1;
    static constexpr size_t kBytes = sizeof(float) * (4 * C * LDK + 2 * C * LDC);
};

template <typename T, int DK>
__global__ void __launch_bounds__(kBwdThreads, 1)
bwd_gram_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ b,
                const float *__restrict__ log_alpha, BwdWs ws, int Tlen, int H)
{
    constexpr int LDK = DK + 1;
    extern __shared__ float smem[];
    float *sQ = smem, *sK = sQ + C * LDK, *sB = sK + C * LDK, *sAl = sB + C * LDK;
    float *sA = sAl + C * LDK, *sT = sA + C * LDC;
    const int tid = threadIdx.x, c = blockIdx.x, h = blockIdx.y;
    const long bi = blockIdx.z, pair = bi * H + h;
    const int nch = gridDim.x, t0 = c * C, Lc = min(C, Tlen - t0);
    float *Pg = ws.P + (pair * nch + c) * C * C, *Tg = ws.T + (pair * nch + c) * C * C;

    load_rows<T, DK>(sQ, q, tid, bi, Tlen, H, h, t0, Lc);
    load_rows<T, DK>(sK, k, tid, bi, Tlen, H, h, t0, Lc);
    load_rows<T, DK>(sB, b, tid, bi, Tlen, H, h, t0, Lc);
    load_alpha<DK>(sAl, log_alpha, tid, bi, Tlen, H, h, t0, Lc);
    __syncthreads();
    // A_ts = sum_i E_ti k_si f_tsi (s < t), P_ts = sum_i q_ti k_si f_tsi (s <= t),
    // f_tsi = prod_{s<u<=t} alpha_ui: thread (token t, channel quarter), 4 lanes per token
    {
        // (channel 4 j + cq for lane cq: the 4 lanes of a token hit 4 different banks)
        constexpr int CPT = DK / 4;
        const int t = tid >> 2, cq = tid & 3;
        const int tmax = (tid >> 5) * 8 + 7;  // the warp's largest token: every lane shuffles
        float qv[CPT], ev[CPT], f[CPT];
#pragma unroll
        for (int j = 0; j < CPT; ++j) {
            qv[j] = sQ[t * LDK + 4 * j + cq];
            ev[j] = sB[t * LDK + 4 * j + cq] * sK[t * LDK + 4 * j + cq];
            f[j] = 1.f;
        }
        for (int s = tmax; s >= 0; --s) {
            const bool on = s <= t;
            float pa = 0.f, aa = 0.f;
            if (on) {
#pragma unroll
                for (int j = 0; j < CPT; ++j) {
                    const float a = f[j] * sK[s * LDK + 4 * j + cq];
                    pa = fmaf(qv[j], a, pa);
                    aa = fmaf(ev[j], a, aa);
                    f[j] *= sAl[s * LDK + 4 * j + cq];
                }
            }
            pa += __shfl_xor_sync(0xffffffffu, pa, 1);
            aa += __shfl_xor_sync(0xffffffffu, aa, 1);
            pa += __shfl_xor_sync(0xffffffffu, pa, 2);
            aa += __shfl_xor_sync(0xffffffffu, aa, 2);
            if (cq == 0) {
                Pg[t * C + s] = on ? pa : 0.f;
                sA[t * LDC + s] = (s < t) ? aa : 0.f;
            }
        }
        if (cq == 0)
            for (int s = tmax + 1; s < C; ++s) {
                Pg[t * C + s] = 0.f;
                sA[t * LDC + s] = 0.f;
            }
    }
    // T = (I + A)^{-1}: (I + A) T = I by forward substitution, all columns at once
    for (int idx = tid; idx < C * C; idx += kBwdThreads) sT[(idx / C) * LDC + idx % C] = (idx / C == idx % C) ? 1.f : 0.f;
    __syncthreads();
    for (int s = 0; s < C - 1; ++s) {
        for (int idx = tid; idx < (C - 1 - s) * (s + 1); idx += kBwdThreads) {
            const int t = s + 1 + idx / (s + 1), j = idx % (s + 1);
            sT[t * LDC + j] -= sA[t * LDC + s] * sT[s * LDC + j];
        }
        __syncthreads();
    }
    for (int idx = tid; idx < C * C; idx += kBwdThreads) Tg[idx] = sT[(idx / C) * LDC + idx % C];
    // the decayed factors of the chain kernels (running products of alpha per channel)
    const long fo = (pair * nch + c) * (long)C * DK;
    if (tid < DK) {
        const int i = tid;
        float p = 1.f;
        for (int t = 0; t < C; ++t) {
            p *= sAl[t * LDK + i];
            ws.Eb[fo + t * DK + i] = p * sB[t * LDK + i] * sK[t * LDK + i];
            ws.Qb[fo + t * DK + i] = p * sQ[t * LDK + i];
        }
        ws.gC[(pair * nch + c) * DK + i] = p;
    } else if (tid < 2 * DK) {
        const int i = tid - DK;
        float sf = 1.f;
        for (int t = C - 1; t >= 0; --t) {
            ws.Kt[fo + t * DK + i] = sf * sK[t * LDK + i];
            sf *= sAl[t * LDK + i];
        }
    }
}

// Value-axis inputs of a chain kernel (zero past the sequence end).
template <typename T>
__device__ __forceinline__ float ld(const T *p, long off, bool on) { return on ? to_f32(p[off]) : 0.f; }

// ------------------------------------------------------------------ fwd (checkpoints and U)
template <int DK>
struct FwdSmem {
    static constexpr int LDK = DK + 1, DVT = kChainDvTile;
    static constexpr size_t kBytes = sizeof(float) * (2 * C * LDK + C * LDC + DK * DVT + 2 * C * DVT + DK);
};

template <typename T, int DK>
__global__ void __launch_bounds__(kBwdThreads, 2)
bwd_fwd_kernel(const T *__restrict__ k, const T *__restrict__ v, const T *__restrict__ b, const T *__restrict__ w,
               const float *__restrict__ log_alpha, const float *__restrict__ S0, BwdWs ws, int Tlen, int H, int DV)
{
    constexpr int LDK = DK + 1, DVT = kChainDvTile;
    extern __shared__ float smem[];
    float *sE = smem, *sKt = sE + C * LDK, *sT = sKt + C * LDK, *sS = sT + C * LDC, *sR = sS + DK * DVT;
    float *sU = sR + C * DVT, *sG = sU + C * DVT;
    const int tid = threadIdx.x, j0 = blockIdx.x * DVT, h = blockIdx.y;
    const long bi = blockIdx.z, pair = bi * H + h;
    const int nch = (Tlen + C - 1) / C;
    const long DD = (long)DK * DV;

    for (int idx = tid; idx < DK * DVT; idx += kBwdThreads) {
        const int i = idx / DVT, j = idx % DVT;
        sS[idx] = S0 ? S0[pair * DD + (long)i * DV + j0 + j] : 0.f;
    }
    for (int c = 0; c <= nch; ++c) {
        __syncthreads();  // the previous chunk is done with every buffer; S is final
        float *ck = ws.ck + (pair * (nch + 1) + c) * DD;
        for (int idx = tid; idx < DK * DVT; idx += kBwdThreads) ck[(long)(idx / DVT) * DV + j0 + idx % DVT] = sS[idx];
        if (c == nch) break;
        const int t0 = c * C, Lc = min(C, Tlen - t0);
        const float *Tg = ws.T + (pair * nch + c) * C * C;
        for (int idx = tid; idx < C * C; idx += kBwdThreads) sT[(idx / C) * LDC + idx % C] = Tg[idx];
        for (int idx = tid; idx < C * DVT; idx += kBwdThreads) {
            const int t = idx / DVT, j = idx % DVT;
            const long off = ((bi * Tlen + t0 + t) * H + h) * (long)DV + j0 + j;
            sR[idx] = ld(w, off, t < Lc) * ld(v, off, t < Lc);
        }
        // the chunk's decayed factors (from the gram kernel)
        {
            const long fo = (pair * nch + c) * (long)C * DK;
            for (int idx = tid; idx < C * DK; idx += kBwdThreads) {
                sE[(idx / DK) * LDK + idx % DK] = ws.Eb[fo + idx];
                sKt[(idx / DK) * LDK + idx % DK] = ws.Kt[fo + idx];
            }
            for (int i = tid; i < DK; i += kBwdThreads) sG[i] = ws.gC[(pair * nch + c) * DK + i];
        }
        __syncthreads();
        // the thread's outputs: column j of rows r0 + RS * m (independent sums, interleaved)
        constexpr int RS = kBwdThreads / DVT;    // rows apart
        constexpr int NO = C * DVT / kBwdThreads, NS = DK * DVT / kBwdThreads;
        const int r0 = tid / DVT, j = tid % DVT;
        // RHS = Z - Ebar S
        {
            float acc[NO];
#pragma unroll
            for (int m = 0; m < NO; ++m) acc[m] = 0.f;
            for (int i = 0; i < DK; ++i) {
                const float sv = sS[i * DVT + j];
#pragma unroll
                for (int m = 0; m < NO; ++m) acc[m] = fmaf(sE[(r0 + RS * m) * LDK + i], sv, acc[m]);
            }
#pragma unroll
            for (int m = 0; m < NO; ++m) sR[(r0 + RS * m) * DVT + j] -= acc[m];
        }
        __syncthreads();
        // U = T RHS (T lower triangular)
        {
            float *Ug = ws.U + (pair * nch + c) * (long)C * DV;
            float acc[NO];
#pragma unroll
            for (int m = 0; m < NO; ++m) acc[m] = 0.f;
            for (int s = 0; s < C; ++s) {
                const float rv = sR[s * DVT + j];
#pragma unroll
                for (int m = 0; m < NO; ++m) acc[m] = fmaf(sT[(r0 + RS * m) * LDC + s], rv, acc[m]);
            }
#pragma unroll
            for (int m = 0; m < NO; ++m) {
                const int t = r0 + RS * m;
                sU[t * DVT + j] = acc[m];
                Ug[(long)t * DV + j0 + j] = acc[m];
            }
        }
        __syncthreads();
        // S <- e^{Gamma_C} S + Ktil^T U
        {
            float acc[NS];
#pragma unroll
            for (int m = 0; m < NS; ++m) acc[m] = sG[r0 + RS * m] * sS[(r0 + RS * m) * DVT + j];
            for (int s = 0; s < C; ++s) {
                const float uv = sU[s * DVT + j];
#pragma unroll
                for (int m = 0; m < NS; ++m) acc[m] = fmaf(sKt[s * LDK + r0 + RS * m], uv, acc[m]);
            }
#pragma unroll
            for (int m = 0; m < NS; ++m) sS[(r0 + RS * m) * DVT + j] = acc[m];
        }
    }
}

// ------------------------------------------------------------------ adj (the adjoint chain)
template <int DK>
struct AdjSmem {
    static constexpr int LDK = DK + 1, DVT = kChainDvTile;
    static constexpr size_t kBytes = sizeof(float) * (3 * C * LDK + 2 * C * LDC + DK * DVT + 3 * C * DVT + DK);
};

template <typename T, int DK>
__global__ void __launch_bounds__(kBwdThreads, 2)
bwd_adj_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v, const T *__restrict__ b,
               const T *__restrict__ w, const float *__restrict__ log_alpha, const T *__restrict__ dO,
               const float *__restrict__ dS_T, BwdWs ws, float *__restrict__ gv, float *__restrict__ gw,
               float *__restrict__ dS0, int Tlen, int H, int DV)
{
    constexpr int LDK = DK + 1, DVT = kChainDvTile;
    extern __shared__ float smem[];
    float *sKt = smem, *sQb = sKt + C * LDK, *sEb = sQb + C * LDK, *sT = sEb + C * LDK, *sP = sT + C * LDC;
    float *sD = sP + C * LDC, *sO = sD + DK * DVT, *sR = sO + C * DVT, *sU = sR + C * DVT, *sG = sU + C * DVT;
    const int tid = threadIdx.x, j0 = blockIdx.x * DVT, h = blockIdx.y;
    const long bi = blockIdx.z, pair = bi * H + h;
    const int nch = (Tlen + C - 1) / C;
    const long DD = (long)DK * DV;

    for (int idx = tid; idx < DK * DVT; idx += kBwdThreads) {
        const int i = idx / DVT, j = idx % DVT;
        sD[idx] = dS_T ? dS_T[pair * DD + (long)i * DV + j0 + j] : 0.f;
    }
    for (int c = nch - 1; c >= 0; --c) {
        const int t0 = c * C, Lc = min(C, Tlen - t0);
        __syncthreads();  // the later chunk is done with every buffer; dS' is final
        float *dsg = ws.dS + (pair * nch + c) * DD;
        for (int idx = tid; idx < DK * DVT; idx += kBwdThreads) dsg[(long)(idx / DVT) * DV + j0 + idx % DVT] = sD[idx];
        const float *Tg = ws.T + (pair * nch + c) * C * C, *Pg = ws.P + (pair * nch + c) * C * C;
        for (int idx = tid; idx < C * C; idx += kBwdThreads) {
            sT[(idx / C) * LDC + idx % C] = Tg[idx];
            sP[(idx / C) * LDC + idx % C] = Pg[idx];
        }
        for (int idx = tid; idx < C * DVT; idx += kBwdThreads) {
            const int t = idx / DVT, j = idx % DVT;
            sO[idx] = ld(dO, ((bi * Tlen + t0 + t) * H + h) * (long)DV + j0 + j, t < Lc);
        }
        // the chunk's decayed factors (from the gram kernel)
        {
            const long fo = (pair * nch + c) * (long)C * DK;
            for (int idx = tid; idx < C * DK; idx += kBwdThreads) {
                const int r = (idx / DK) * LDK + idx % DK;
                sKt[r] = ws.Kt[fo + idx];
                sQb[r] = ws.Qb[fo + idx];
                sEb[r] = ws.Eb[fo + idx];
            }
            for (int i = tid; i < DK; i += kBwdThreads) sG[i] = ws.gC[(pair * nch + c) * DK + i];
        }
        __syncthreads();
        // the thread's outputs: column j of rows r0 + RS * m (independent sums, interleaved)
        constexpr int RS = kBwdThreads / DVT, NO = C * DVT / kBwdThreads;
        const int r0 = tid / DVT, j = tid % DVT;
        // RHS2 = Ktil dS' + P^T dO  (P lower: P_ts = 0 for t < s)
        {
            float acc[NO];
#pragma unroll
            for (int m = 0; m < NO; ++m) acc[m] = 0.f;
            for (int i = 0; i < DK; ++i) {
                const float dv = sD[i * DVT + j];
#pragma unroll
                for (int m = 0; m < NO; ++m) acc[m] = fmaf(sKt[(r0 + RS * m) * LDK + i], dv, acc[m]);
            }
            for (int t = 0; t < C; ++t) {
                const float ov = sO[t * DVT + j];
#pragma unroll
                for (int m = 0; m < NO; ++m) acc[m] = fmaf(sP[t * LDC + r0 + RS * m], ov, acc[m]);
            }
#pragma unroll
            for (int m = 0; m < NO; ++m) sR[(r0 + RS * m) * DVT + j] = acc[m];
        }
        __syncthreads();
        // dU = T^T RHS2 (T lower: T_ts = 0 for t < s); dv = dU (*) w, dw = dU (*) v
        {
            float *dUg = ws.dU + (pair * nch + c) * (long)C * DV;
            float acc[NO];
#pragma unroll
            for (int m = 0; m < NO; ++m) acc[m] = 0.f;
            for (int t = 0; t < C; ++t) {
                const float rv = sR[t * DVT + j];
#pragma unroll
                for (int m = 0; m < NO; ++m) acc[m] = fmaf(sT[t * LDC + r0 + RS * m], rv, acc[m]);
            }
#pragma unroll
            for (int m = 0; m < NO; ++m) {
                const int s = r0 + RS * m;
                sU[s * DVT + j] = acc[m];
                dUg[(long)s * DV + j0 + j] = acc[m];
                if (s < Lc) {
                    const long off = ((bi * Tlen + t0 + s) * H + h) * (long)DV + j0 + j;
                    gv[off] = acc[m] * to_f32(w[off]);
                    gw[off] = acc[m] * to_f32(v[off]);
                }
            }
        }
        __syncthreads();
        // dS = e^{Gamma_C} dS' + sum_t e^{Gamma_t} (q_t dO_t^T - E_t dU_t^T)
        {
            constexpr int JPT = DVT * DK / kBwdThreads;  // columns per thread
            const int i = tid % DK, jb = (tid / DK) * JPT;
            float acc[JPT];
#pragma unroll
            for (int j = 0; j < JPT; ++j) acc[j] = 0.f;
            for (int t = 0; t < C; ++t) {
                const float qp = sQb[t * LDK + i], ep = sEb[t * LDK + i];
#pragma unroll
                for (int j = 0; j < JPT; ++j) acc[j] += qp * sO[t * DVT + jb + j] - ep * sU[t * DVT + jb + j];
            }
            const float g = sG[i];
#pragma unroll
            for (int j = 0; j < JPT; ++j) sD[i * DVT + jb + j] = g * sD[i * DVT + jb + j] + acc[j];
        }
    }
    __syncthreads();
    if (dS0)
        for (int idx = tid; idx < DK * DVT; idx += kBwdThreads)
            dS0[pair * DD + (long)(idx / DVT) * DV + j0 + idx % DVT] = sD[idx];
}

// ------------------------------------------------------------------ grad (key-axis gradients)
constexpr int kGradCols = 16;     // value columns staged at a time
constexpr int kGradThreads = 512;  // 16 (token, channel) pairs per thread at dk = 128
template <int DK>
struct GradSmem {
    static constexpr int LDK = DK + 1;
    static constexpr size_t kBytes =
        sizeof(float) * (4 * C * LDK + 2 * C * LDC + 3 * C * kGradCols + 3 * DK * (kGradCols + 1) + DK);
};

template <typename T, int DK>
__global__ void __launch_bounds__(kGradThreads, 1)
bwd_grad_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ b,
                const float *__restrict__ log_alpha, const T *__restrict__ dO, BwdWs ws, float *__restrict__ gq,
                float *__restrict__ gk, float *__restrict__ gb, float *__restrict__ gla, int Tlen, int H, int DV)
{
    constexpr int LDK = DK + 1, NC = kGradCols;
    constexpr int TPT = C * DK / kGradThreads;  // tokens per thread
    constexpr int WPT = C * C / kGradThreads;   // W1/W2 entries per thread
    extern __shared__ float smem[];
    float *sQ = smem, *sK = sQ + C * LDK, *sB = sK + C * LDK, *sAl = sB + C * LDK;
    float *sW1 = sAl + C * LDK, *sW2 = sW1 + C * LDC;  // W1[t][s] = dO_t . u_s, W2[t][s] = dU_t . u_s
    float *sUc = sW2 + C * LDC, *sdUc = sUc + C * NC, *sOc = sdUc + C * NC;
    // the block's columns of S (entering), dS' and S (leaving): rows padded to NC + 1
    float *sSc = sOc + C * NC, *sDc = sSc + DK * (NC + 1), *sNc = sDc + DK * (NC + 1), *sRow = sNc + DK * (NC + 1);
    const int tid = threadIdx.x, c = blockIdx.x, h = blockIdx.y;
    const long bi = blockIdx.z, pair = bi * H + h;
    const int nch = gridDim.x, t0 = c * C, Lc = min(C, Tlen - t0);
    const long DD = (long)DK * DV;
    const float *Sc = ws.ck + (pair * (nch + 1) + c) * DD, *Sn = Sc + DD;  // entering and leaving the chunk
    const float *dSc = ws.dS + (pair * nch + c) * DD;                         // dS' at the chunk end
    const float *Ug = ws.U + (pair * nch + c) * (long)C * DV, *dUg = ws.dU + (pair * nch + c) * (long)C * DV;

    load_rows<T, DK, kGradThreads>(sQ, q, tid, bi, Tlen, H, h, t0, Lc);
    load_rows<T, DK, kGradThreads>(sK, k, tid, bi, Tlen, H, h, t0, Lc);
    load_rows<T, DK, kGradThreads>(sB, b, tid, bi, Tlen, H, h, t0, Lc);
    load_alpha<DK, kGradThreads>(sAl, log_alpha, tid, bi, Tlen, H, h, t0, Lc);

    // this thread: channel i of tokens tb + ts * m, and WPT entries (t, s) of W1, W2
    const int i = tid % DK, tb = tid / DK, ts = kGradThreads / DK;
    float so[TPT], su[TPT], du[TPT];
#pragma unroll
    for (int m = 0; m < TPT; ++m) so[m] = su[m] = du[m] = 0.f;
    float w1[WPT], w2[WPT];
#pragma unroll
    for (int m = 0; m < WPT; ++m) w1[m] = w2[m] = 0.f;
    float row = 0.f;
    for (int jc = 0; jc < DV; jc += NC) {
        __syncthreads();  // the previous columns are read
        for (int idx = tid; idx < C * NC; idx += kGradThreads) {
            const int t = idx / NC, j = idx % NC;
            sUc[idx] = Ug[(long)t * DV + jc + j];
            sdUc[idx] = dUg[(long)t * DV + jc + j];
            sOc[idx] = (t < Lc) ? to_f32(dO[((bi * Tlen + t0 + t) * H + h) * (long)DV + jc + j]) : 0.f;
        }
        for (int idx = tid; idx < DK * NC; idx += kGradThreads) {
            const int r = idx / NC, j = idx % NC;
            sSc[r * (NC + 1) + j] = Sc[(long)r * DV + jc + j];
            sDc[r * (NC + 1) + j] = dSc[(long)r * DV + jc + j];
            sNc[r * (NC + 1) + j] = Sn[(long)r * DV + jc + j];
        }
        __syncthreads();
#pragma unroll
        for (int m = 0; m < WPT; ++m) {
            const int e = tid + m * kGradThreads, t = e / C, s = e % C;
#pragma unroll 8
            for (int j = 0; j < NC; ++j) {
                w1[m] = fmaf(sOc[t * NC + j], sUc[s * NC + j], w1[m]);
                w2[m] = fmaf(sdUc[t * NC + j], sUc[s * NC + j], w2[m]);
            }
        }
        // (S dO_t)_i, (S dU_t)_i, (dS' u_t)_i and rowsum(dS' (*) S_next)_i over these columns
        const float *si = sSc + i * (NC + 1), *di = sDc + i * (NC + 1), *ni = sNc + i * (NC + 1);
#pragma unroll 4
        for (int j = 0; j < NC; ++j) {
            const float sij = si[j], dij = di[j];
            if (tb == 0) row = fmaf(dij, ni[j], row);
#pragma unroll
            for (int m = 0; m < TPT; ++m) {
                const int t = tb + ts * m;
                so[m] = fmaf(sij, sOc[t * NC + j], so[m]);
                su[m] = fmaf(sij, sdUc[t * NC + j], su[m]);
                du[m] = fmaf(dij, sUc[t * NC + j], du[m]);
            }
        }
    }
#pragma unroll
    for (int m = 0; m < WPT; ++m) {
        const int e = tid + m * kGradThreads;
        sW1[(e / C) * LDC + e % C] = w1[m];
        sW2[(e / C) * LDC + e % C] = w2[m];
    }
    if (tb == 0) sRow[i] = row;
    __syncthreads();
    // per (token, channel): dq, de, dk (write) by running products of alpha down (s <= t)
    // and up (s >= t) from t (unrolled: the accumulators above stay in registers)
#pragma unroll
    for (int m = 0; m < TPT; ++m) {
        const int t = tb + ts * m;
        float f = 1.f, aq = 0.f, ae = 0.f;
        for (int s = t; s >= 0; --s) {
            const float ks = sK[s * LDK + i];
            aq = fmaf(sW1[t * LDC + s] * f, ks, aq);
            if (s < t) ae = fmaf(sW2[t * LDC + s] * f, ks, ae);
            f *= sAl[s * LDK + i];
        }
        const float pre = f;  // e^{Gamma_t}
        float g = 1.f, akw = 0.f;
        for (int s = t; s < C; ++s) {
            if (s > t) g *= sAl[s * LDK + i];
            akw = fmaf(sW1[s * LDC + t] * g, sQ[s * LDK + i], akw);
            if (s > t) akw = fmaf(-sW2[s * LDC + t] * g, sB[s * LDK + i] * sK[s * LDK + i], akw);
        }
        const float suf = g;  // e^{Gamma_C - Gamma_t}
        const float dq = pre * so[m] + aq;
        const float de = -(pre * su[m] + ae);
        const float dkw = suf * du[m] + akw;
        const float qi = sQ[t * LDK + i], ki = sK[t * LDK + i], bv = sB[t * LDK + i];
        if (t < Lc) {
            const long off = ((bi * Tlen + t0 + t) * H + h) * (long)DK + i;
            gq[off] = dq;
            gk[off] = dkw + de * bv;
            gb[off] = de * ki;
            gla[off] = qi * dq + bv * ki * de - ki * dkw;  // dGamma_t, summed below
        }
    }
    __syncthreads();  // every dGamma of the chunk is written
    // dlog_alpha: reverse cumulative sum of dGamma over the chunk's tokens, with the chunk-end term
    for (int ii = tid; ii < DK; ii += kGradThreads) {
        float acc = sRow[ii];
        for (int t = Lc - 1; t >= 0; --t) {
            float *p = gla + ((bi * Tlen + t0 + t) * H + h) * (long)DK + ii;
            acc += *p;
            *p = acc;
        }
    }
}

template <typename T, int DK>
cudaError_t launch(const BwdArgs &a)
{
    static std::atomic<unsigned long long> s0{0}, s1{0}, s2{0}, s3{0};
    auto kg = bwd_gram_kernel<T, DK>;
    auto kf = bwd_fwd_kernel<T, DK>;
    auto ka = bwd_adj_kernel<T, DK>;
    auto kd = bwd_grad_kernel<T, DK>;
    cudaError_t e = ensure_smem_limit(kg, (int)GramSmem<DK>::kBytes, s0);
    if (e == cudaSuccess) e = ensure_smem_limit(kf, (int)FwdSmem<DK>::kBytes, s1);
    if (e == cudaSuccess) e = ensure_smem_limit(ka, (int)AdjSmem<DK>::kBytes, s2);
    if (e == cudaSuccess) e = ensure_smem_limit(kd, (int)GradSmem<DK>::kBytes, s3);
    if (e != cudaSuccess) return e;
    const int nch = (a.T + C - 1) / C;
    const long pairs = (long)a.B * a.H;
    BwdWs ws;
    float *p = a.ws;
    ws.T = p; p += pairs * nch * C * C;
    ws.P = p; p += pairs * nch * C * C;
    ws.ck = p; p += pairs * (nch + 1) * (long)a.dk * a.dv;
    ws.U = p; p += pairs * nch * (long)C * a.dv;
    ws.dU = p; p += pairs * nch * (long)C * a.dv;
    ws.dS = p; p += pairs * nch * (long)a.dk * a.dv;
    ws.Eb = p; p += pairs * nch * (long)C * a.dk;
    ws.Qb = p; p += pairs * nch * (long)C * a.dk;
    ws.Kt = p; p += pairs * nch * (long)C * a.dk;
    ws.gC = p;
    const dim3 chunks(nch, a.H, a.B), tiles(a.dv / kChainDvTile, a.H, a.B);
    kg<<<chunks, kBwdThreads, GramSmem<DK>::kBytes, a.stream>>>((const T *)a.q, (const T *)a.k, (const T *)a.b,
                                                                 a.log_alpha, ws, a.T, a.H);
    kf<<<tiles, kBwdThreads, FwdSmem<DK>::kBytes, a.stream>>>((const T *)a.k, (const T *)a.v, (const T *)a.b,
                                                               (const T *)a.w, a.log_alpha, a.S0, ws, a.T, a.H, a.dv);
    ka<<<tiles, kBwdThreads, AdjSmem<DK>::kBytes, a.stream>>>((const T *)a.q, (const T *)a.k, (const T *)a.v,
                                                               (const T *)a.b, (const T *)a.w, a.log_alpha,
                                                               (const T *)a.dO, a.dS_T, ws, a.gv, a.gw, a.dS0, a.T,
                                                               a.H, a.dv);
    kd<<<chunks, kGradThreads, GradSmem<DK>::kBytes, a.stream>>>((const T *)a.q, (const T *)a.k, (const T *)a.b,
                                                                 a.log_alpha, (const T *)a.dO, ws, a.gq, a.gk, a.gb,
                                                                 a.gla, a.T, a.H, a.dv);
    return cudaGetLastError();
}

}  // namespace

size_t bwd_workspace_floats(int B, int T, int H, int dk, int dv)
{
    const long nch = (T + C - 1) / C, pairs = (long)B * H;
    return (size_t)pairs * (2 * nch * C * C + (nch + 1) * (long)dk * dv + 2 * nch * (long)C * dv +
                            nch * (long)dk * dv + 3 * nch * (long)C * dk + nch * (long)dk);
}

cudaError_t launch_bwd_simt(const BwdArgs &a)
{
    if (a.bf16) return a.dk == 128 ? launch<__nv_bfloat16, 128>(a) : launch<__nv_bfloat16, 64>(a);
    return a.dk == 128 ? launch<float, 128>(a) : launch<float, 64>(a);
}

}  // namespace gdn2
