"""fp64 model of the chunkwise (WY) backward that the tensor-core backward implements.

Test infrastructure, not the oracle: it restates the kernel's algebra in numpy
at full precision so that the algebra itself can be checked against the
oracle's gradients (the analytic backward of the token recurrence) on the CPU.

Training runs the chunkwise WY form, and its backward keeps the per-channel
gates b and w inside the gradients of the auxiliaries ("Gated DeltaNet-2",
iplexlaw.co.kr, section "Procesamiento del token y entrenamiento paralelo";
gist.science, section 3).  Per chunk of L <= C tokens, with S the state
entering it and Gamma the chunk-local cumulative log-decay (per key channel):
    e = b k,  Ebar = e^{Gamma} e,  Qbar = e^{Gamma} q,  Ktil = e^{Gamma_C - Gamma} k
    A_ts = sum_d e_t e^{Gamma_t - Gamma_s} k_s  (s < t),   P_ts likewise with q_t (s <= t)
    T = (I + A)^{-1},  X = w v - Ebar S,  U = T X
    O = Qbar S + P U,  S' = e^{Gamma_C} S + Ktil^T U
and, given dO and the gradient dS' of the state leaving the chunk,
    gU = Ktil dS' + P^T dO,  dX = T^T gU,  dv = dX w,  dw = dX v
    dQbar = dO S^T,  dEbar = -dX S^T,  dKtil = U dS'^T,  dP = dO U^T,  dA = -dX U^T
    dS = e^{Gamma_C} dS' + Qbar^T dO - Ebar^T dX            (the state entering)
and through the pairwise decays
    dq_t = e^{Gamma_t} dQbar_t + sum_s dP_ts e^{Gamma_t - Gamma_s} k_s
    de_t = e^{Gamma_t} dEbar_t + sum_s dA_ts e^{Gamma_t - Gamma_s} k_s
    dkw_s = e^{Gamma_C - Gamma_s} dKtil_s + sum_t (dP_ts q_t + dA_ts e_t) e^{Gamma_t - Gamma_s}
    dk = dkw + de b,  db = de k.
dlog_alpha_u is the sum over t >= u of dGamma_t = q dq + e de - k dkw, plus
dGamma_C.  `regrouped=True` forms it the way the kernel does, so that terms
which cancel do so exactly: P's diagonal enters dq and dk but not dGamma;
Ktil's share K_t = k_t e^{Gamma_C - Gamma_t} dKtil_t adds sum_{t < u} K_t; the
rest of dGamma_C is rowsum(dS' o e^{Gamma_C} S).

`rounding` (optional) is applied to the operands of U = T X and dX = T^T gU,
to study what their bf16 rounding costs; pairs=True takes T and X (not gU) as
bf16 pairs, hi + lo: U = T_hi X_hi + T_hi X_lo + T_lo X_hi and
dX = T_hi^T gU + T_lo^T gU, the products the kernel adds for flagged chunks.
"""
import numpy as np


def _pair_decay(G):
    """D[t, s, d] = e^{Gamma_t - Gamma_s} for s <= t, else 0."""
    L = G.shape[0]
    D = np.exp(G[:, None, :] - G[None, :, :])
    return D * np.tril(np.ones((L, L)))[:, :, None]


def _mm(a, b, rounding, pair_a, pair_b):
    """a @ b with both operands rounded; an operand marked as a pair also
    contributes its rounded remainder against the other's rounded part."""
    if rounding is None:
        return a @ b
    ah, bh = rounding(a), rounding(b)
    r = ah @ bh
    if pair_b:
        r = r + ah @ rounding(b - bh)
    if pair_a:
        r = r + rounding(a - ah) @ bh
    return r


def chunk_bwd(q, k, v, b, w, la, S, dO, dSn, *, regrouped=True, rounding=None, pairs=False):
    """Gradients of one chunk: returns (dq, dk, dv, db, dw, dla, dS)."""
    L = q.shape[0]
    G = np.cumsum(la, axis=0)
    GC = G[-1]
    e = b * k
    D = _pair_decay(G)
    strict = np.tril(np.ones((L, L)), -1)
    A = np.einsum("td,tsd,sd->ts", e, D, k) * strict
    P = np.einsum("td,tsd,sd->ts", q, D, k)
    T = np.linalg.inv(np.eye(L) + A)
    Eb, Qb, Kt = np.exp(G) * e, np.exp(G) * q, np.exp(GC - G) * k
    X = w * v - Eb @ S
    U = _mm(T, X, rounding, pairs, pairs)
    gU = Kt @ dSn + P.T @ dO
    dX = _mm(T.T, gU, rounding, pairs, False)
    dv, dw = dX * w, dX * v
    dQb, dEb, dKt = dO @ S.T, -dX @ S.T, U @ dSn.T
    dP = np.tril(dO @ U.T)
    dA = -(dX @ U.T) * strict
    dS = np.exp(GC)[:, None] * dSn + Qb.T @ dO - Eb.T @ dX
    if regrouped:
        dPs = dP * strict                       # P's diagonal: apart
        diag = np.diag(dP)[:, None]
    else:
        dPs, diag = dP, np.zeros((L, 1))
    dq = np.exp(G) * dQb + np.einsum("ts,tsd,sd->td", dPs, D, k)
    de = np.exp(G) * dEb + np.einsum("ts,tsd,sd->td", dA, D, k)
    dkw_pair = np.einsum("ts,tsd,td->sd", dPs, D, q) + np.einsum("ts,tsd,td->sd", dA, D, e)
    Ks = np.exp(GC - G) * dKt * k               # Ktil's share, per token and channel
    if regrouped:
        dG = q * dq + e * de - k * dkw_pair     # without P's diagonal and Ktil's share
        excl = np.cumsum(Ks, axis=0) - Ks       # sum over t < u
        dla = np.cumsum(dG[::-1], axis=0)[::-1] + excl + np.sum(dSn * (np.exp(GC)[:, None] * S), axis=1)
        dq = dq + diag * k
        dkw = dkw_pair + np.exp(GC - G) * dKt + diag * q
    else:
        dkw = dkw_pair + np.exp(GC - G) * dKt
        dG = q * dq + e * de - k * dkw
        dGC = np.sum(Ks, axis=0) + np.sum(dSn * (np.exp(GC)[:, None] * S), axis=1)
        dla = np.cumsum(dG[::-1], axis=0)[::-1] + dGC
    dk = dkw + de * b
    db = de * k
    return dq, dk, dv, db, dw, dla, dS


def _chunk_fwd(q, k, v, b, w, la, S):
    """State leaving one chunk (fp64, exact pairwise decays)."""
    L = q.shape[0]
    G = np.cumsum(la, axis=0)
    e = b * k
    A = np.einsum("td,tsd,sd->ts", e, _pair_decay(G), k) * np.tril(np.ones((L, L)), -1)
    U = np.linalg.solve(np.eye(L) + A, w * v - (np.exp(G) * e) @ S)
    return np.exp(G[-1])[:, None] * S + (np.exp(G[-1] - G) * k).T @ U


def wy_backward(q, k, v, b, w, log_alpha, S0, dO, dS_T, C=64, **kw):
    """Gradients of sum(o * dO) + sum(S_T * dS_T) over [B,T,H,d] inputs, chunk by
    chunk in reverse; returns a dict like the oracle's backward."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    out = {n: np.zeros(q.shape) for n in ("dq", "dk", "db", "dlog_alpha")}
    out.update({n: np.zeros(v.shape) for n in ("dv", "dw")})
    out["dS0"] = np.zeros((B, H, dk, dv))
    for bi in range(B):
        for h in range(H):
            S = np.zeros((dk, dv)) if S0 is None else S0[bi, h].copy()
            starts = list(range(0, T, C))
            entry = []
            for c0 in starts:
                sl = slice(c0, min(c0 + C, T))
                entry.append(S)
                S = _chunk_fwd(*(x[bi, sl, h] for x in (q, k, v, b, w, log_alpha)), S)
            dS = np.zeros((dk, dv)) if dS_T is None else dS_T[bi, h].copy()
            for c0, Sc in zip(reversed(starts), reversed(entry)):
                sl = slice(c0, min(c0 + C, T))
                g = chunk_bwd(*(x[bi, sl, h] for x in (q, k, v, b, w, log_alpha)), Sc, dO[bi, sl, h], dS, **kw)
                for n, x in zip(("dq", "dk", "dv", "db", "dw", "dlog_alpha"), g[:6]):
                    out[n][bi, sl, h] = x
                dS = g[6]
            out["dS0"][bi, h] = dS
    return out
