/*
 * gdn2_oracle.c -- fp64 CPU oracle for the Gated DeltaNet-2 operator.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU
 * baseline leg of the benchmark may load this file's library.  The CUDA
 * library never links, includes or calls anything here, and this file shares
 * no code with it.
 *
 * What it computes is the plain per-token definition of the gated delta rule
 * with decoupled erase and write gates, token by token, in double precision:
 *
 *   "Gated DeltaNet-2: Decoupling Erase and Write in Linear Attention"
 *   (iplexlaw.co.kr blog, section "Decisiones independientes en dos ejes"):
 *       e_t = b_t (*) k_t,   z_t = w_t (*) v_t,
 *       Sbar = D_t S_{t-1},  r_t = Sbar^T e_t,  S_t = Sbar + k_t (z_t - r_t)^T,
 *       and the query reads the updated state.
 *   (zubnet.ai news, update equation): D_t = Diag(alpha_t) is the per-key-
 *       channel decay, so it scales the key rows of the dk x dv state.
 *   (gist.science summary, section 1 "Gated Delta Rule-2"): b_t in [0,1]^dk
 *       acts on the key axis and w_t in [0,1]^dv on the value axis.
 *
 * Readings where the pages are silent: o_t = S_t^T q_t with no 1/sqrt(dk)
 * scale (no page scales q); alpha_t = exp(log_alpha_t) with log_alpha given
 * as input; gates are not clamped (an ablation on the iplexlaw page widens the
 * erase range to [0,2]); k is used as given (normalisation belongs to the
 * layer, not to the operator).
 *
 * There is no chunking, blocking or reordering: one (batch, head) pair at a
 * time, one token at a time, each sum in index order.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* Layouts (all row-major, contiguous):
 *   q, k, b, log_alpha : [B][T][H][dk]
 *   v, w, o            : [B][T][H][dv]
 *   S0, S_T            : [B][H][dk][dv]   (S0 may be NULL: zero state;
 *                                          S_T may be NULL: not written)
 * Returns 0 on success, -1 on bad sizes, -2 if scratch allocation fails. */
int gdn2_oracle_fwd(const double *q, const double *k, const double *v,
                    const double *b, const double *w, const double *log_alpha,
                    const double *S0, double *o, double *S_T,
                    int B, int T, int H, int dk, int dv, int nthreads)
{
    if (B < 0 || T < 0 || H < 0 || dk <= 0 || dv <= 0) return -1;
    const long npairs = (long)B * H;
    int failed = 0;
#ifdef _OPENMP
    if (nthreads <= 0) nthreads = omp_get_max_threads();
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads) reduction(| : failed)
#else
    (void)nthreads;
#endif
    for (long p = 0; p < npairs; ++p) {
        const long bi = p / H, hi = p % H;
        double *S = (double *)malloc(sizeof(double) * (size_t)dk * dv);
        double *e = (double *)malloc(sizeof(double) * (size_t)dk);
        double *z = (double *)malloc(sizeof(double) * (size_t)dv);
        double *r = (double *)malloc(sizeof(double) * (size_t)dv);
        double *alpha = (double *)malloc(sizeof(double) * (size_t)dk);
        if (!S || !e || !z || !r || !alpha) {
            failed = 1;
            free(S); free(e); free(z); free(r); free(alpha);
            continue;
        }
        const double *s0 = S0 ? S0 + p * (long)dk * dv : NULL;
        for (long i = 0; i < (long)dk * dv; ++i) S[i] = s0 ? s0[i] : 0.0;

        for (long t = 0; t < T; ++t) {
            const long rk = ((bi * T + t) * H + hi) * dk; /* row of a [B,T,H,dk] tensor */
            const long rv = ((bi * T + t) * H + hi) * dv; /* row of a [B,T,H,dv] tensor */

            /* decay, erase key and gated value */
            for (int i = 0; i < dk; ++i) {
                alpha[i] = exp(log_alpha[rk + i]);
                e[i] = b[rk + i] * k[rk + i];
            }
            for (int j = 0; j < dv; ++j) z[j] = w[rv + j] * v[rv + j];

            /* Sbar = Diag(alpha) S  (row i of the state is key channel i) */
            for (int i = 0; i < dk; ++i)
                for (int j = 0; j < dv; ++j) S[(long)i * dv + j] *= alpha[i];

            /* r = Sbar^T e : read of the decayed state along the erase key */
            for (int j = 0; j < dv; ++j) {
                double acc = 0.0;
                for (int i = 0; i < dk; ++i) acc += S[(long)i * dv + j] * e[i];
                r[j] = acc;
            }

            /* S = Sbar + k (z - r)^T */
            for (int i = 0; i < dk; ++i) {
                const double ki = k[rk + i];
                for (int j = 0; j < dv; ++j) S[(long)i * dv + j] += ki * (z[j] - r[j]);
            }

            /* o = S^T q, with the updated state */
            for (int j = 0; j < dv; ++j) {
                double acc = 0.0;
                for (int i = 0; i < dk; ++i) acc += S[(long)i * dv + j] * q[rk + i];
                o[rv + j] = acc;
            }
        }
        if (S_T) memcpy(S_T + p * (long)dk * dv, S, sizeof(double) * (size_t)dk * dv);
        free(S); free(e); free(z); free(r); free(alpha);
    }
    return failed ? -2 : 0;
}

/* Number of host threads the OpenMP runtime would use by default. */
int gdn2_oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
