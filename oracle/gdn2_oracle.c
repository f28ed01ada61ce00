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

/*
 * gdn2_oracle_bwd -- gradients of L = sum(o * dO) + sum(S_T * dS_T) with
 * respect to every input, by backpropagation through the recurrence above,
 * token by token in reverse, in double precision.
 *
 * The forward steps of one token, and the adjoint of each in reverse order
 * (dS is dL/dS_t from the later tokens; dS' adds the token's own output):
 *     o_t = S_t^T q_t               dS' = dS + q_t dO_t^T,   dq_t = S_t dO_t
 *     S_t = Sbar + k_t u_t^T        dk_t (write) = dS' u_t,  du_t = dS'^T k_t
 *     u_t = z_t - r_t               dz_t = du_t,             dr_t = -du_t
 *     z_t = w_t (*) v_t             dw_t = du_t (*) v_t,     dv_t = du_t (*) w_t
 *     r_t = Sbar^T e_t              dSbar = dS' + e_t dr_t^T, de_t = Sbar dr_t
 *     e_t = b_t (*) k_t             db_t = de_t (*) k_t,     dk_t += de_t (*) b_t
 *     Sbar = Diag(alpha_t) S_{t-1}  dS_{t-1} = Diag(alpha_t) dSbar,
 *     alpha_t = exp(log_alpha_t)    dlog_alpha_t = rowsum(dSbar (*) Sbar)
 * and dS_0 is the last dS.  The gates stay inside this aggregation: b and w
 * receive their own gradients, not one for a shared scalar ("Gated
 * DeltaNet-2", iplexlaw.co.kr, section "Procesamiento del token y
 * entrenamiento paralelo": the per-channel factors cannot be pulled out as a
 * scalar beta in backpropagation).
 *
 * The states of a stretch of 64 tokens are recomputed from a stored state at
 * its start (memory only: the arithmetic is the forward's, token by token).
 *
 * dO: [B][T][H][dv]; dS_T: [B][H][dk][dv] or NULL (zero); outputs dq, dk, db,
 * dlog_alpha: [B][T][H][dk]; dv, dw: [B][T][H][dv]; dS0: [B][H][dk][dv].
 */
int gdn2_oracle_bwd(const double *q, const double *k, const double *v,
                    const double *b, const double *w, const double *log_alpha,
                    const double *S0, const double *dO, const double *dS_T,
                    double *dq, double *dkey, double *dval, double *db, double *dw,
                    double *dla, double *dS0,
                    int B, int T, int H, int dk, int dv, int nthreads)
{
    if (B < 0 || T < 0 || H < 0 || dk <= 0 || dv <= 0) return -1;
    const long npairs = (long)B * H;
    const long DD = (long)dk * dv;
    const int SEG = 64;
    const long nseg = (T + SEG - 1) / SEG;
    int failed = 0;
#ifdef _OPENMP
    if (nthreads <= 0) nthreads = omp_get_max_threads();
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads) reduction(| : failed)
#else
    (void)nthreads;
#endif
    for (long p = 0; p < npairs; ++p) {
        const long bi = p / H, hi = p % H;
        double *ck = (double *)malloc(sizeof(double) * (size_t)(nseg + 1) * DD);  /* state at each stretch start */
        double *st = (double *)malloc(sizeof(double) * (size_t)(SEG + 1) * DD);   /* states of one stretch */
        double *S = (double *)malloc(sizeof(double) * (size_t)DD);
        double *dS = (double *)malloc(sizeof(double) * (size_t)DD);
        double *Sbar = (double *)malloc(sizeof(double) * (size_t)DD);
        double *vec = (double *)malloc(sizeof(double) * (size_t)(4 * dk + 4 * dv));
        if (!ck || !st || !S || !dS || !Sbar || !vec) {
            failed = 1;
            free(ck); free(st); free(S); free(dS); free(Sbar); free(vec);
            continue;
        }
        double *alpha = vec, *e = vec + dk, *dkv = vec + 2 * dk, *de = vec + 3 * dk;
        double *z = vec + 4 * dk, *r = z + dv, *u = r + dv, *du = u + dv;
        const double *s0 = S0 ? S0 + p * DD : NULL;

        /* forward: the state at the start of every stretch */
        for (long i = 0; i < DD; ++i) S[i] = s0 ? s0[i] : 0.0;
        for (long t = 0; t < T; ++t) {
            if (t % SEG == 0) memcpy(ck + (t / SEG) * DD, S, sizeof(double) * DD);
            const long rk = ((bi * T + t) * H + hi) * dk, rv = ((bi * T + t) * H + hi) * dv;
            for (int i = 0; i < dk; ++i) { alpha[i] = exp(log_alpha[rk + i]); e[i] = b[rk + i] * k[rk + i]; }
            for (int j = 0; j < dv; ++j) z[j] = w[rv + j] * v[rv + j];
            for (int i = 0; i < dk; ++i)
                for (int j = 0; j < dv; ++j) S[(long)i * dv + j] *= alpha[i];
            for (int j = 0; j < dv; ++j) {
                double acc = 0.0;
                for (int i = 0; i < dk; ++i) acc += S[(long)i * dv + j] * e[i];
                r[j] = acc;
            }
            for (int i = 0; i < dk; ++i)
                for (int j = 0; j < dv; ++j) S[(long)i * dv + j] += k[rk + i] * (z[j] - r[j]);
        }

        /* backward, stretch by stretch from the last */
        for (long i = 0; i < DD; ++i) dS[i] = dS_T ? dS_T[p * DD + i] : 0.0;
        for (long sg = nseg - 1; sg >= 0; --sg) {
            const long t0 = sg * SEG, t1 = (t0 + SEG < T) ? t0 + SEG : T;
            /* st[m] = state before token t0 + m (st[t1 - t0] = after the last) */
            memcpy(st, ck + sg * DD, sizeof(double) * DD);
            for (long t = t0; t < t1; ++t) {
                const long rk = ((bi * T + t) * H + hi) * dk, rv = ((bi * T + t) * H + hi) * dv;
                double *cur = st + (t - t0) * DD, *nxt = st + (t - t0 + 1) * DD;
                for (int i = 0; i < dk; ++i) { alpha[i] = exp(log_alpha[rk + i]); e[i] = b[rk + i] * k[rk + i]; }
                for (int j = 0; j < dv; ++j) z[j] = w[rv + j] * v[rv + j];
                for (int i = 0; i < dk; ++i)
                    for (int j = 0; j < dv; ++j) nxt[(long)i * dv + j] = alpha[i] * cur[(long)i * dv + j];
                for (int j = 0; j < dv; ++j) {
                    double acc = 0.0;
                    for (int i = 0; i < dk; ++i) acc += nxt[(long)i * dv + j] * e[i];
                    r[j] = acc;
                }
                for (int i = 0; i < dk; ++i)
                    for (int j = 0; j < dv; ++j) nxt[(long)i * dv + j] += k[rk + i] * (z[j] - r[j]);
            }
            for (long t = t1 - 1; t >= t0; --t) {
                const long rk = ((bi * T + t) * H + hi) * dk, rv = ((bi * T + t) * H + hi) * dv;
                const double *prev = st + (t - t0) * DD, *cur = st + (t - t0 + 1) * DD;  /* S_{t-1}, S_t */
                for (int i = 0; i < dk; ++i) { alpha[i] = exp(log_alpha[rk + i]); e[i] = b[rk + i] * k[rk + i]; }
                for (int j = 0; j < dv; ++j) z[j] = w[rv + j] * v[rv + j];
                /* Sbar, r and u of the forward step */
                for (int i = 0; i < dk; ++i)
                    for (int j = 0; j < dv; ++j) Sbar[(long)i * dv + j] = alpha[i] * prev[(long)i * dv + j];
                for (int j = 0; j < dv; ++j) {
                    double acc = 0.0;
                    for (int i = 0; i < dk; ++i) acc += Sbar[(long)i * dv + j] * e[i];
                    r[j] = acc;
                    u[j] = z[j] - acc;
                }
                /* o_t = S_t^T q_t */
                for (int i = 0; i < dk; ++i) {
                    double acc = 0.0;
                    for (int j = 0; j < dv; ++j) acc += cur[(long)i * dv + j] * dO[rv + j];
                    dq[rk + i] = acc;
                }
                for (int i = 0; i < dk; ++i)
                    for (int j = 0; j < dv; ++j) dS[(long)i * dv + j] += q[rk + i] * dO[rv + j];
                /* S_t = Sbar + k u^T */
                for (int i = 0; i < dk; ++i) {
                    double acc = 0.0;
                    for (int j = 0; j < dv; ++j) acc += dS[(long)i * dv + j] * u[j];
                    dkv[i] = acc;
                }
                for (int j = 0; j < dv; ++j) {
                    double acc = 0.0;
                    for (int i = 0; i < dk; ++i) acc += dS[(long)i * dv + j] * k[rk + i];
                    du[j] = acc;
                }
                /* z = w v */
                for (int j = 0; j < dv; ++j) { dw[rv + j] = du[j] * v[rv + j]; dval[rv + j] = du[j] * w[rv + j]; }
                /* r = Sbar^T e with dr = -du: dSbar = dS - e du^T, de = -Sbar du */
                for (int i = 0; i < dk; ++i) {
                    double acc = 0.0;
                    for (int j = 0; j < dv; ++j) {
                        dS[(long)i * dv + j] -= e[i] * du[j];
                        acc += Sbar[(long)i * dv + j] * du[j];
                    }
                    de[i] = -acc;
                }
                /* e = b k */
                for (int i = 0; i < dk; ++i) {
                    db[rk + i] = de[i] * k[rk + i];
                    dkey[rk + i] = dkv[i] + de[i] * b[rk + i];
                }
                /* Sbar = Diag(alpha) S_{t-1} */
                for (int i = 0; i < dk; ++i) {
                    double acc = 0.0;
                    for (int j = 0; j < dv; ++j) {
                        acc += dS[(long)i * dv + j] * Sbar[(long)i * dv + j];
                        dS[(long)i * dv + j] *= alpha[i];
                    }
                    dla[rk + i] = acc;
                }
            }
        }
        if (dS0) memcpy(dS0 + p * DD, dS, sizeof(double) * DD);
        free(ck); free(st); free(S); free(dS); free(Sbar); free(vec);
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
