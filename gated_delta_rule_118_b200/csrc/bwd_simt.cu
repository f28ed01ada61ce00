// bwd_simt.cu -- the chunkwise backward of the operator on the fp32 pipes.
//
// Gradients of L = sum(o * dO) + sum(S_T * dS_T) with respect to q, k, v, b,
// w, log_alpha and S0, chunk by chunk in reverse ("Gated DeltaNet-2",
// iplexlaw.co.kr, section "Procesamiento del token y entrenamiento paralelo":
// the WY form over 64-token blocks, whose backward must use the modulated keys
// and values -- the per-channel gates cannot be pulled out as a scalar beta).
//
// Per chunk, with S the state entering it (a checkpoint from the forward), dS'
// = dL/dS at its end (carried from the chunk after), Gamma the chunk-local
// cumulative log-decay, E = b (*) k the erase keys, A and P the strictly lower
// and lower Grams of the decayed erase keys and queries against the keys, and
// T = (I + A)^{-1} (derived from the token recurrence; the forward's
// U = T (Z - Ebar S) are the chunk's write residuals u_t):
//   dU   = T^T (Ktil dS' + P^T dO)          (= dZ: dv = dU (*) w, dw = dU (*) v)
//   dq_t = e^{Gamma_t} (*) (S dO_t) + sum_{s<=t} (dO_t . u_s) e^{Gamma_t-Gamma_s} (*) k_s
//   de_t = -e^{Gamma_t} (*) (S dU_t) - sum_{s<t} (dU_t . u_s) e^{Gamma_t-Gamma_s} (*) k_s
//   dk_t (write) = e^{Gamma_C-Gamma_t} (*) (dS' u_t) + sum_{s>=t} (dO_s . u_t) e^{Gamma_s-Gamma_t} (*) q_s
//                  - sum_{s>t} (dU_s . u_t) e^{Gamma_s-Gamma_t} (*) E_s
//   db_t = de_t (*) k_t,   dk_t = dk_t (write) + de_t (*) b_t
//   dGamma_t = q_t (*) dq_t + E_t (*) de_t - k_t (*) dk_t (write)  (+ rowsum(dS' (*) S_end) at the
//              chunk end), and dlog_alpha is its reverse cumulative sum over the chunk
//   dS (entering) = e^{Gamma_C} (*) dS' + sum_t e^{Gamma_t} (*) (q_t dO_t^T - E_t dU_t^T)
// Every decay between two tokens is a running product of alpha (a decay, <= 1),
// so no factor can overflow and any log_alpha <= 0 (-inf included) is exact.
//
// One CTA owns one (batch, head, 16-column value tile) and walks the chunks from
// the last; the value-axis gradients of its columns are its own, the key-axis
// ones (dq, dk, db, dlog_alpha) are sums over the value columns, added across
// the tiles with fp32 atomics into buffers the host zeroed.
#include "common.cuh"
#include "launch.h"

namespace gdn2 {
namespace {

constexpr int kBwdThreads = 256;
constexpr int kBwdDvTile = 16;

template <int DK>
struct BwdSmem {
    static constexpr int C = kChunk, LDK = DK + 1, LDC = kChunk + 1, DVT = kBwdDvTile;
    static constexpr int kFloats = 5 * C * LDK      // q, k, b, alpha, scratch X
                                   + 2 * C * LDC    // A | W1, P | W2
                                   + 2 * DK * DVT   // S (entering), dS' (carried)
                                   + 3 * C * DVT    // U, dU, dO
                                   + DK;            // row sums
    static constexpr size_t kBytes = sizeof(float) * kFloats;
};

template <typename T, int DK>
__global__ void __launch_bounds__(kBwdThreads, 1)
bwd_simt_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                const T *__restrict__ b, const T *__restrict__ w, const float *__restrict__ log_alpha,
                const T *__restrict__ dO, const float *__restrict__ dS_T, const float *__restrict__ ckpt,
                float *__restrict__ gq, float *__restrict__ gk, float *__restrict__ gv, float *__restrict__ gb,
                float *__restrict__ gw, float *__restrict__ gla, float *__restrict__ dS0, int Tlen, int H, int DV)
{
    using L = BwdSmem<DK>;
    constexpr int C = kChunk, LDK = L::LDK, LDC = L::LDC, DVT = L::DVT;
    extern __shared__ float smem[];
    float *sQ = smem;               // q            [C][LDK]
    float *sK = sQ + C * LDK;       // k
    float *sB = sK + C * LDK;       // b
    float *sAl = sB + C * LDK;      // alpha = exp(log_alpha)
    float *sX = sAl + C * LDK;      // scratch: Ebar, then Ktil, then dGamma
    float *sA = sX + C * LDK;       // A (strict lower), then W1[t][s] = dO_t . u_s   [C][LDC]
    float *sP = sA + C * LDC;       // P (lower), then W2[t][s] = dU_t . u_s
    float *sS = sP + C * LDC;       // S entering the chunk, this tile   [DK][DVT]
    float *sD = sS + DK * DVT;      // dS' at the chunk end (carried)
    float *sU = sD + DK * DVT;      // Z -> U   [C][DVT]
    float *sdU = sU + C * DVT;      // RHS -> dU
    float *sO = sdU + C * DVT;      // dO
    float *sRow = sO + C * DVT;     // rowsum(dS' (*) S_end) of this tile [DK]

    const int tid = threadIdx.x;
    const int j0 = blockIdx.x * DVT;
    const int h = blockIdx.y;
    const long bi = blockIdx.z;
    const long pair = bi * H + h;
    const int nch = (Tlen + C - 1) / C;
    const long DD = (long)DK * DV;
    const float *ck = ckpt + pair * (long)(nch + 1) * DD;

    for (int idx = tid; idx < DK * DVT; idx += kBwdThreads) {
        const int i = idx / DVT, j = idx % DVT;
        sD[idx] = dS_T ? dS_T[pair * DD + (long)i * DV + j0 + j] : 0.f;
    }

    for (int c = nch - 1; c >= 0; --c) {
        const int t0 = c * C, Lc = min(C, Tlen - t0);
        __syncthreads();  // the previous (later) chunk is done with every buffer
        // ---- loads: inputs (zero past the sequence end, alpha = 1 there), the
        //      state entering the chunk, dO, Z; rowsum(dS' (*) S_end)
        for (int idx = tid; idx < C * DK; idx += kBwdThreads) {
            const int t = idx / DK, i = idx % DK;
            float qv = 0.f, kv = 0.f, bv = 0.f, al = 1.f;
            if (t < Lc) {
                const long off = ((bi * Tlen + t0 + t) * H + h) * (long)DK + i;
                qv = to_f32(q[off]); kv = to_f32(k[off]); bv = to_f32(b[off]); al = expf(log_alpha[off]);
            }
            sQ[t * LDK + i] = qv; sK[t * LDK + i] = kv; sB[t * LDK + i] = bv; sAl[t * LDK + i] = al;
        }
        for (int idx = tid; idx < DK * DVT; idx += kBwdThreads) {
            const int i = idx / DVT, j = idx % DVT;
            sS[idx] = ck[(long)c * DD + (long)i * DV + j0 + j];
        }
        for (int idx = tid; idx < C * DVT; idx += kBwdThreads) {
            const int t = idx / DVT, j = idx % DVT;
            float z = 0.f, g = 0.f;
            if (t < Lc) {
                const long off = ((bi * Tlen + t0 + t) * H + h) * (long)DV + j0 + j;
                z = to_f32(w[off]) * to_f32(v[off]);
                g = to_f32(dO[off]);
            }
            sU[idx] = z;
            sO[idx] = g;
        }
        for (int i = tid; i < DK; i += kBwdThreads) {
            const float *se = ck + (long)(c + 1) * DD + (long)i * DV + j0;
            float acc = 0.f;
            for (int j = 0; j < DVT; ++j) acc += sD[i * DVT + j] * se[j];
            sRow[i] = acc;
        }
        __syncthreads();

        // ---- A_ts = sum_i E_ti k_si f_tsi (s < t), P_ts = sum_i q_ti k_si f_tsi (s <= t),
        //      f_tsi = prod_{s<u<=t} alpha_ui: thread (token t, channel quarter), 4 lanes per token
        {
            constexpr int CPT = DK / 4;
            const int t = tid >> 2, cq = tid & 3, i0 = cq * CPT;
            const int tmax = (tid >> 5) * 8 + 7;  // the warp's largest token: every lane shuffles
            float qv[CPT], ev[CPT], f[CPT];
#pragma unroll
            for (int j = 0; j < CPT; ++j) {
                qv[j] = sQ[t * LDK + i0 + j];
                ev[j] = sB[t * LDK + i0 + j] * sK[t * LDK + i0 + j];
                f[j] = 1.f;
            }
            for (int s = tmax; s >= 0; --s) {
                const bool on = s <= t;
                float pa = 0.f, aa = 0.f;
                if (on) {
#pragma unroll
                    for (int j = 0; j < CPT; ++j) {
                        const float a = f[j] * sK[s * LDK + i0 + j];
                        pa = fmaf(qv[j], a, pa);
                        aa = fmaf(ev[j], a, aa);
                        f[j] *= sAl[s * LDK + i0 + j];
                    }
                }
                pa += __shfl_xor_sync(0xffffffffu, pa, 1);
                aa += __shfl_xor_sync(0xffffffffu, aa, 1);
                pa += __shfl_xor_sync(0xffffffffu, pa, 2);
                aa += __shfl_xor_sync(0xffffffffu, aa, 2);
                if (cq == 0) {
                    sP[t * LDC + s] = on ? pa : 0.f;
                    sA[t * LDC + s] = (s < t) ? aa : 0.f;
                }
            }
            if (cq == 0)
                for (int s = tmax + 1; s < C; ++s) {
                    sP[t * LDC + s] = 0.f;
                    sA[t * LDC + s] = 0.f;
                }
        }
        // ---- X = Ebar = e^{Gamma} (*) b (*) k (channel walks over the tokens)
        for (int i = tid; i < DK; i += kBwdThreads) {
            float p = 1.f;
            for (int t = 0; t < C; ++t) {
                p *= sAl[t * LDK + i];
                sX[t * LDK + i] = p * sB[t * LDK + i] * sK[t * LDK + i];
            }
        }
        __syncthreads();
        // ---- U: (I + A) U = Z - Ebar S
        for (int idx = tid; idx < C * DVT; idx += kBwdThreads) {
            const int t = idx / DVT, j = idx % DVT;
            const float *e = sX + t * LDK;
            float acc = 0.f;
            for (int i = 0; i < DK; ++i) acc = fmaf(e[i], sS[i * DVT + j], acc);
            sU[idx] -= acc;
        }
        __syncthreads();
        for (int s = 0; s < C - 1; ++s) {
            for (int idx = tid; idx < (C - 1 - s) * DVT; idx += kBwdThreads) {
                const int t = s + 1 + idx / DVT, j = idx % DVT;
                sU[t * DVT + j] -= sA[t * LDC + s] * sU[s * DVT + j];
            }
            __syncthreads();
        }
        // ---- X = Ktil = e^{Gamma_C - Gamma} (*) k (channel walks from the chunk end)
        for (int i = tid; i < DK; i += kBwdThreads) {
            float sf = 1.f;
            for (int t = C - 1; t >= 0; --t) {
                sX[t * LDK + i] = sf * sK[t * LDK + i];
                sf *= sAl[t * LDK + i];
            }
        }
        __syncthreads();
        // ---- dU: (I + A^T) dU = Ktil dS' + P^T dO
        for (int idx = tid; idx < C * DVT; idx += kBwdThreads) {
            const int s = idx / DVT, j = idx % DVT;
            const float *kt = sX + s * LDK;
            float acc = 0.f;
            for (int i = 0; i < DK; ++i) acc = fmaf(kt[i], sD[i * DVT + j], acc);
            for (int t = s; t < C; ++t) acc = fmaf(sP[t * LDC + s], sO[t * DVT + j], acc);
            sdU[idx] = acc;
        }
        __syncthreads();
        for (int t = C - 1; t >= 1; --t) {
            for (int idx = tid; idx < t * DVT; idx += kBwdThreads) {
                const int s = idx / DVT, j = idx % DVT;
                sdU[s * DVT + j] -= sA[t * LDC + s] * sdU[t * DVT + j];
            }
            __syncthreads();
        }
        // ---- dv = dU (*) w, dw = dU (*) v for this tile's columns
        for (int idx = tid; idx < Lc * DVT; idx += kBwdThreads) {
            const int t = idx / DVT, j = idx % DVT;
            const long off = ((bi * Tlen + t0 + t) * H + h) * (long)DV + j0 + j;
            gv[off] = sdU[idx] * to_f32(w[off]);
            gw[off] = sdU[idx] * to_f32(v[off]);
        }
        // ---- W1[t][s] = dO_t . u_s,  W2[t][s] = dU_t . u_s  (this tile's columns)
        for (int idx = tid; idx < C * C; idx += kBwdThreads) {
            const int t = idx / C, s = idx % C;
            float a1 = 0.f, a2 = 0.f;
#pragma unroll
            for (int j = 0; j < DVT; ++j) {
                a1 = fmaf(sO[t * DVT + j], sU[s * DVT + j], a1);
                a2 = fmaf(sdU[t * DVT + j], sU[s * DVT + j], a2);
            }
            sA[t * LDC + s] = a1;
            sP[t * LDC + s] = a2;
        }
        __syncthreads();
        // ---- per (token, channel): dq, de, dk (write) by running products of alpha
        //      down (s <= t) and up (s >= t) from t; thread: channel i, tokens of one half
        {
            const int i = tid % DK, half = tid / DK;
            constexpr int TPT = C * DK / kBwdThreads;  // tokens per thread
            for (int m = 0; m < TPT; ++m) {
                const int t = (DK == 128) ? half + 2 * m : (tid / DK) + (kBwdThreads / DK) * m;
                // walk down: f = e^{Gamma_t - Gamma_s}
                float f = 1.f, aq = 0.f, ae = 0.f;
                for (int s = t; s >= 0; --s) {
                    const float ks = sK[s * LDK + i];
                    aq = fmaf(sA[t * LDC + s] * f, ks, aq);
                    if (s < t) ae = fmaf(sP[t * LDC + s] * f, ks, ae);
                    f *= sAl[s * LDK + i];
                }
                const float pre = f;  // e^{Gamma_t} (including token 0's decay)
                // walk up: g = e^{Gamma_s - Gamma_t}
                float g = 1.f, akw = 0.f;
                for (int s = t; s < C; ++s) {
                    if (s > t) g *= sAl[s * LDK + i];
                    akw = fmaf(sA[s * LDC + t] * g, sQ[s * LDK + i], akw);
                    if (s > t) akw = fmaf(-sP[s * LDC + t] * g, sB[s * LDK + i] * sK[s * LDK + i], akw);
                }
                const float suf = g;  // e^{Gamma_C - Gamma_t}
                // the state terms: (S dO_t)_i, (S dU_t)_i, (dS' u_t)_i over this tile's columns
                float so = 0.f, su = 0.f, du = 0.f;
#pragma unroll
                for (int j = 0; j < DVT; ++j) {
                    const float sij = sS[i * DVT + j];
                    so = fmaf(sij, sO[t * DVT + j], so);
                    su = fmaf(sij, sdU[t * DVT + j], su);
                    du = fmaf(sD[i * DVT + j], sU[t * DVT + j], du);
                }
                const float dq = pre * so + aq;
                const float de = -(pre * su + ae);
                const float dkw = suf * du + akw;
                const float qi = sQ[t * LDK + i], ki = sK[t * LDK + i], bi_ = sB[t * LDK + i];
                sX[t * LDK + i] = qi * dq + bi_ * ki * de - ki * dkw;  // dGamma_t
                if (t < Lc) {
                    const long off = ((bi * Tlen + t0 + t) * H + h) * (long)DK + i;
                    atomicAdd(gq + off, dq);
                    atomicAdd(gk + off, dkw + de * bi_);
                    atomicAdd(gb + off, de * ki);
                }
            }
        }
        __syncthreads();
        // ---- dlog_alpha: reverse cumulative sum of dGamma (with the chunk-end term);
        //      dS entering the chunk = e^{Gamma_C} dS' + sum_t e^{Gamma_t} (q_t dO_t^T - E_t dU_t^T)
        for (int i = tid; i < DK; i += kBwdThreads) {
            float acc = sRow[i];
            for (int t = C - 1; t >= 0; --t) {
                acc += sX[t * LDK + i];
                if (t < Lc) atomicAdd(gla + ((bi * Tlen + t0 + t) * H + h) * (long)DK + i, acc);
            }
        }
        {
            constexpr int JPT = DVT * DK / kBwdThreads;  // columns per thread
            const int i = tid % DK, jb = (tid / DK) * JPT;
            float acc[JPT];
#pragma unroll
            for (int j = 0; j < JPT; ++j) acc[j] = 0.f;
            float p = 1.f;
            for (int t = 0; t < C; ++t) {
                p *= sAl[t * LDK + i];
                const float qp = p * sQ[t * LDK + i], ep = p * sB[t * LDK + i] * sK[t * LDK + i];
#pragma unroll
                for (int j = 0; j < JPT; ++j) acc[j] += qp * sO[t * DVT + jb + j] - ep * sdU[t * DVT + jb + j];
            }
            __syncthreads();  // every thread has read dS' (the row sums and the dkw terms read it)
#pragma unroll
            for (int j = 0; j < JPT; ++j) sD[i * DVT + jb + j] = p * sD[i * DVT + jb + j] + acc[j];
        }
    }
    __syncthreads();
    if (dS0) {
        for (int idx = tid; idx < DK * DVT; idx += kBwdThreads) {
            const int i = idx / DVT, j = idx % DVT;
            dS0[pair * DD + (long)i * DV + j0 + j] = sD[idx];
        }
    }
}

template <typename T, int DK>
cudaError_t launch(const BwdArgs &a)
{
    const size_t smem = BwdSmem<DK>::kBytes;
    auto kern = bwd_simt_kernel<T, DK>;
    static std::atomic<unsigned long long> smem_set{0};
    cudaError_t e = ensure_smem_limit(kern, (int)smem, smem_set);
    if (e != cudaSuccess) return e;
    dim3 grid(a.dv / kBwdDvTile, a.H, a.B);
    kern<<<grid, kBwdThreads, smem, a.stream>>>((const T *)a.q, (const T *)a.k, (const T *)a.v, (const T *)a.b,
                                                (const T *)a.w, a.log_alpha, (const T *)a.dO, a.dS_T, a.ckpt, a.gq,
                                                a.gk, a.gv, a.gb, a.gw, a.gla, a.dS0, a.T, a.H, a.dv);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bwd_simt(const BwdArgs &a)
{
    if (a.bf16) return a.dk == 128 ? launch<__nv_bfloat16, 128>(a) : launch<__nv_bfloat16, 64>(a);
    return a.dk == 128 ? launch<float, 128>(a) : launch<float, 64>(a);
}

}  // namespace gdn2
