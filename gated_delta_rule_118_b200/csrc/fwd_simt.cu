// fwd_simt.cu -- chunkwise forward on the fp32 FMA pipes.
//
// This is the fp32-input path of gdn2_fwd_chunked: every product runs in fp32
// on CUDA cores, so it meets the fp32 tolerance that tensor-core operands in
// bf16 cannot.  It follows the chunkwise (WY) form with chunks of 64 tokens
// ("Gated DeltaNet-2", iplexlaw.co.kr, section "Procesamiento del token y
// entrenamiento paralelo"; gist.science, section 3 "Efficient chunkwise
// parallel training"), with Gamma the chunk-local cumulative log-decay in fp32
// and r the chunk midpoint:
//   Ehat = e^{Gamma-Gamma_r} b k,  Qhat = e^{Gamma-Gamma_r} q,
//   Khat = e^{Gamma_r-Gamma} k,    Ktil = e^{Gamma_C-Gamma} k,
//   A = strict_lower(Ehat Khat^T), P = lower(Qhat Khat^T), Sref = e^{Gamma_r} S,
//   (I + A) U = Z - Ehat Sref,     O = Qhat Sref + P U,
//   S <- e^{Gamma_C} S + Ktil^T U.
// A chunk whose decay is too strong for the midpoint split (some
// |Gamma_t - Gamma_r| above kMidpointLogDecayRangeF32) uses the reference 0
// instead (Qbar = e^{Gamma} q, Ebar = e^{Gamma} b k, Sref = S) and forms A and P
// from running products of alpha, so that every factor is a decay (<= 1).
// One CTA owns one (batch, head, 32-column value tile); value columns of the
// state are independent because the erase and the decay act on key rows.
#include "common.cuh"
#include "gdn2.h"
#include "launch.h"

namespace gdn2 {
namespace {

constexpr int kSimtThreads = 256;
constexpr int kSimtDvTile = 32;

template <int DK, int DVT>
struct SimtSmem {
    static constexpr int LDK = DK + 1;     // padded rows: conflict-free column walks
    static constexpr int LDC = kChunk + 1;
    static constexpr int kFloats = 4 * kChunk * LDK   // Qhat, Khat, Ehat, Ktil
                                   + 2 * kChunk * LDC // A, P
                                   + 2 * DK * DVT     // S, Sref
                                   + kChunk * DVT     // Z -> U
                                   + 2 * DK;          // Gamma_r, Gamma_C
    static constexpr size_t kBytes = sizeof(float) * kFloats;
};

template <typename T, int DK, int DVT>
__global__ void __launch_bounds__(kSimtThreads)
fwd_simt_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                const T *__restrict__ b, const T *__restrict__ w,
                const float *__restrict__ log_alpha, const float *S0, T *__restrict__ o,
                float *S_T, int Tlen, int H, int DV, unsigned layout)
{
    using L = SimtSmem<DK, DVT>;
    constexpr int C = kChunk, LDK = L::LDK, LDC = L::LDC;
    extern __shared__ float smem[];
    float *sQ = smem;                 // q  -> Qhat        [C][LDK]
    float *sK = sQ + C * LDK;         // k  -> Khat
    float *sE = sK + C * LDK;         // b  -> Ehat
    float *sG = sE + C * LDK;         // log_alpha -> Gamma -> Ktil
    float *sA = sG + C * LDK;         // A  [C][LDC]
    float *sP = sA + C * LDC;         // P
    float *sS = sP + C * LDC;         // S  [DK][DVT]
    float *sR = sS + DK * DVT;        // Sref
    float *sU = sR + DK * DVT;        // Z -> U  [C][DVT]
    float *sGr = sU + C * DVT;        // Gamma_r [DK]
    float *sGc = sGr + DK;            // Gamma_C [DK]

    const int tid = threadIdx.x;
    const int j0 = blockIdx.x * DVT;  // first value column of this tile
    const int h = blockIdx.y;
    const long bi = blockIdx.z;
    const long pair = bi * H + h;
    // gate layouts: b, w or log_alpha may hold one value per (token, head)
    const bool b_scalar = layout & GDN2_ERASE_SCALAR, w_scalar = layout & GDN2_WRITE_SCALAR,
               a_scalar = layout & GDN2_DECAY_SCALAR;
    // the fused layer's raw inputs: q and k before their L2 norm, gate and decay logits
    const bool logits = layout & kLayerInputsBit;

    for (int idx = tid; idx < DK * DVT; idx += kSimtThreads) {
        const int i = idx / DVT, j = idx % DVT;
        sS[idx] = S0 ? S0[(pair * DK + i) * DV + j0 + j] : 0.f;
    }

    const int nchunks = (Tlen + C - 1) / C;
    for (int c = 0; c < nchunks; ++c) {
        const int t0 = c * C;
        const int Lc = min(C, Tlen - t0);
        __syncthreads();  // previous chunk done with every buffer

        // ---- load the chunk (rows past the sequence end are zero) ----
        for (int idx = tid; idx < C * DK; idx += kSimtThreads) {
            const int t = idx / DK, i = idx % DK;
            float qv = 0.f, kv = 0.f, bv = 0.f, la = 0.f;
            if (t < Lc) {
                const long tok = (bi * Tlen + t0 + t) * H + h, off = tok * DK + i;
                qv = to_f32(q[off]); kv = to_f32(k[off]);
                bv = to_f32(b[b_scalar ? tok : off]);
                la = log_alpha[a_scalar ? tok : off];
                if (logits) {
                    bv = 1.f / (1.f + expf(-bv));
                    la = fminf(la, 0.f) - log1pf(expf(-fabsf(la)));  // log sigmoid
                }
            }
            sQ[t * LDK + i] = qv; sK[t * LDK + i] = kv; sE[t * LDK + i] = bv; sG[t * LDK + i] = la;
        }
        for (int idx = tid; idx < C * DVT; idx += kSimtThreads) {
            const int t = idx / DVT, j = idx % DVT;
            float z = 0.f;
            if (t < Lc) {
                const long tok = (bi * Tlen + t0 + t) * H + h, off = tok * DV + j0 + j;
                const float wv = to_f32(w[w_scalar ? tok : off]);
                z = (logits ? 1.f / (1.f + expf(-wv)) : wv) * to_f32(v[off]);
            }
            sU[idx] = z;
        }
        __syncthreads();
        if (logits) {  // L2 norm of each q and k row (rows past the sequence end stay zero)
            for (int r = tid; r < 2 * C; r += kSimtThreads) {
                float *row = (r < C ? sQ : sK) + (r % C) * LDK;
                float ss = 0.f;
                for (int i = 0; i < DK; ++i) ss = fmaf(row[i], row[i], ss);
                const float inv = 1.f / sqrtf(ss + 1e-6f);
                for (int i = 0; i < DK; ++i) row[i] *= inv;
            }
            __syncthreads();
        }

        // ---- Gamma: inclusive cumulative log-decay per key channel, fp32 ----
        // The midpoint form is used while every |Gamma_t - Gamma_r| of the chunk
        // stays within kMidpointLogDecayRangeF32; otherwise (strong decay, or
        // log_alpha = -inf) the chunk takes the bounded form below.
        const int rmid = min(C / 2, Lc);  // reference token count (midpoint)
        bool far = false;
        for (int i = tid; i < DK; i += kSimtThreads) {
            float g = 0.f, gr = 0.f;
            for (int t = 0; t < C; ++t) {
                g += sG[t * LDK + i];
                if (t == rmid - 1) gr = g;
            }
            float h = 0.f;
            for (int t = 0; t < C; ++t) {
                h += sG[t * LDK + i];
                far |= !(fabsf(h - gr) <= kMidpointLogDecayRangeF32);
            }
            sGr[i] = gr;
            sGc[i] = g;
        }
        const bool exact = __syncthreads_or(far) != 0;

        if (!exact) {
            for (int i = tid; i < DK; i += kSimtThreads) {
                float g = 0.f;
                for (int t = 0; t < C; ++t) {
                    g += sG[t * LDK + i];
                    sG[t * LDK + i] = g;
                }
            }
            __syncthreads();
            // ---- decay-absorbed factors; Sref = e^{Gamma_r} S ----
            for (int idx = tid; idx < C * DK; idx += kSimtThreads) {
                const int t = idx / DK, i = idx % DK;
                const float g = sG[t * LDK + i];
                const float x = g - sGr[i];
                const float up = expf(x), dn = expf(-x), tl = expf(sGc[i] - g);
                const float kv = sK[t * LDK + i];
                sQ[t * LDK + i] *= up;
                sE[t * LDK + i] *= up * kv;
                sK[t * LDK + i] = dn * kv;
                sG[t * LDK + i] = tl * kv;
            }
            for (int idx = tid; idx < DK * DVT; idx += kSimtThreads)
                sR[idx] = expf(sGr[idx / DVT]) * sS[idx];
            __syncthreads();

            // ---- A = strict_lower(Ehat Khat^T), P = lower(Qhat Khat^T) ----
            for (int idx = tid; idx < C * C; idx += kSimtThreads) {
                const int t = idx / C, s = idx % C;
                float a = 0.f, p = 0.f;
                if (s <= t) {
                    const float *e = sE + t * LDK, *qq = sQ + t * LDK, *kk = sK + s * LDK;
#pragma unroll 8
                    for (int i = 0; i < DK; ++i) {
                        a += e[i] * kk[i];
                        p += qq[i] * kk[i];
                    }
                }
                sA[t * LDC + s] = (s < t) ? a : 0.f;
                sP[t * LDC + s] = p;
            }
        } else {
            // ---- bounded form: every factor is a decay over a stretch of the chunk ----
            //   A_ts = sum_i b_ti k_ti k_si f_tsi,  P_ts = sum_i q_ti k_si f_tsi,
            //   f_tsi = e^{Gamma_ti - Gamma_si} = prod_{s < u <= t} alpha_ui (running products),
            // then Qbar = e^{Gamma} q and Ebar = e^{Gamma} b k (decayed from the chunk
            // start, Sref = S) and Ktil = e^{Gamma_C - Gamma} k from suffix sums.
            for (int idx = tid; idx < DK * DVT; idx += kSimtThreads) sR[idx] = sS[idx];
            {
                constexpr int CPT = DK / 4;  // channels per thread; 4 lanes per token
                const int t = tid >> 2, cq = tid & 3, i0 = cq * CPT;
                const int tmax = (tid >> 5) * 8 + 7;  // the warp's largest token: every lane shuffles
                float qv[CPT], ev[CPT], f[CPT];
#pragma unroll
                for (int j = 0; j < CPT; ++j) {
                    qv[j] = sQ[t * LDK + i0 + j];
                    ev[j] = sE[t * LDK + i0 + j] * sK[t * LDK + i0 + j];
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
                            f[j] *= __expf(sG[s * LDK + i0 + j]);
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
            __syncthreads();
            for (int i = tid; i < DK; i += kSimtThreads) {
                float g = 0.f;
                for (int t = 0; t < C; ++t) {
                    g += sG[t * LDK + i];
                    const float e = expf(g);
                    sQ[t * LDK + i] *= e;
                    sE[t * LDK + i] *= e * sK[t * LDK + i];
                }
                float suf = 0.f;
                for (int t = C - 1; t >= 0; --t) {
                    const float l = sG[t * LDK + i];
                    sG[t * LDK + i] = expf(suf) * sK[t * LDK + i];
                    suf += l;
                }
            }
        }
        __syncthreads();
        // ---- right-hand side Z - Ehat Sref (in place in sU) ----
        for (int idx = tid; idx < C * DVT; idx += kSimtThreads) {
            const int t = idx / DVT, j = idx % DVT;
            const float *e = sE + t * LDK;
            float acc = 0.f;
#pragma unroll 8
            for (int i = 0; i < DK; ++i) acc += e[i] * sR[i * DVT + j];
            sU[idx] -= acc;
        }
        __syncthreads();

        // ---- forward substitution (I + A) U = RHS, column-oriented ----
        for (int s = 0; s < Lc - 1; ++s) {
            for (int idx = tid; idx < (C - 1 - s) * DVT; idx += kSimtThreads) {
                const int t = s + 1 + idx / DVT, j = idx % DVT;
                sU[t * DVT + j] -= sA[t * LDC + s] * sU[s * DVT + j];
            }
            __syncthreads();
        }

        // ---- O = Qhat Sref + P U ----
        for (int idx = tid; idx < Lc * DVT; idx += kSimtThreads) {
            const int t = idx / DVT, j = idx % DVT;
            const float *qq = sQ + t * LDK, *pp = sP + t * LDC;
            float acc = 0.f;
#pragma unroll 8
            for (int i = 0; i < DK; ++i) acc += qq[i] * sR[i * DVT + j];
            for (int s = 0; s <= t; ++s) acc += pp[s] * sU[s * DVT + j];
            o[((bi * Tlen + t0 + t) * H + h) * (long)DV + j0 + j] = from_f32<T>(acc);
        }
        // ---- S <- e^{Gamma_C} S + Ktil^T U ----
        for (int idx = tid; idx < DK * DVT; idx += kSimtThreads) {
            const int i = idx / DVT, j = idx % DVT;
            float acc = expf(sGc[i]) * sS[idx];
            for (int s = 0; s < Lc; ++s) acc += sG[s * LDK + i] * sU[s * DVT + j];
            sS[idx] = acc;
        }
    }
    __syncthreads();
    if (S_T) {
        for (int idx = tid; idx < DK * DVT; idx += kSimtThreads) {
            const int i = idx / DVT, j = idx % DVT;
            S_T[(pair * DK + i) * DV + j0 + j] = sS[idx];
        }
    }
}

template <typename T, int DK>
cudaError_t launch(const FwdArgs &a)
{
    constexpr int DVT = kSimtDvTile;
    const size_t smem = SimtSmem<DK, DVT>::kBytes;
    auto kern = fwd_simt_kernel<T, DK, DVT>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(a.dv / DVT, a.H, a.B);
    kern<<<grid, kSimtThreads, smem, a.stream>>>(
        (const T *)a.q, (const T *)a.k, (const T *)a.v, (const T *)a.b, (const T *)a.w,
        a.log_alpha, a.S0, (T *)a.o, a.S_T, a.T, a.H, a.dv, a.layout);
    return cudaGetLastError();
}

// The fused layer's output processing on the fp32-pipe path, whose CTAs each
// hold a 32-column slice of the outputs: one warp per (batch, token, head) row,
// in place: y = o / sqrt(mean(o^2) + eps) * weight * sigmoid(g)
// ("Gated DeltaNet-2", iplexlaw.co.kr, section "Procesamiento del token y
// entrenamiento paralelo": RMS normalisation and an output gate).
template <typename T, int DV>
__global__ void __launch_bounds__(256)
layer_epilogue_kernel(T *__restrict__ y, const T *__restrict__ g, const float *__restrict__ weight, float eps,
                      long rows)
{
    constexpr int PER = DV / 32;
    const long row = (long)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;  // whole warps
    T *yr = y + row * DV;
    const T *gr = g + row * DV;
    float x[PER];
    float ss = 0.f;
#pragma unroll
    for (int u = 0; u < PER; ++u) {
        x[u] = to_f32(yr[lane + 32 * u]);
        ss = fmaf(x[u], x[u], ss);
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float inv = rsqrtf(ss * (1.f / DV) + eps);
#pragma unroll
    for (int u = 0; u < PER; ++u) {
        const int j = lane + 32 * u;
        yr[j] = from_f32<T>(x[u] * inv * weight[j] / (1.f + expf(-to_f32(gr[j]))));
    }
}

template <typename T, int DV>
cudaError_t launch_epi(const FwdArgs &a)
{
    const long rows = (long)a.B * a.T * a.H;
    layer_epilogue_kernel<T, DV><<<(unsigned)((rows + 7) / 8), 256, 0, a.stream>>>((T *)a.o, (const T *)a.g,
                                                                                  a.norm_weight, a.eps, rows);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_layer_epilogue_rows(const FwdArgs &a)
{
    if (a.bf16) return a.dv == 128 ? launch_epi<__nv_bfloat16, 128>(a) : launch_epi<__nv_bfloat16, 64>(a);
    return a.dv == 128 ? launch_epi<float, 128>(a) : launch_epi<float, 64>(a);
}

cudaError_t launch_fwd_simt(const FwdArgs &a)
{
    if (a.bf16) return a.dk == 128 ? launch<__nv_bfloat16, 128>(a) : launch<__nv_bfloat16, 64>(a);
    return a.dk == 128 ? launch<float, 128>(a) : launch<float, 64>(a);
}

}  // namespace gdn2
