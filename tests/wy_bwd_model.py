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

The bf16 tensor-core backward's rounding points can be emulated one group at a
time (each option a rounding function, bf16 in the tests):
  * `rounding`: the operands of U = T X and dX = T^T gU; pairs=True takes T and
    X (not gU) as bf16 pairs, hi + lo: U = T_hi X_hi + T_hi X_lo + T_lo X_hi and
    dX = T_hi^T gU + T_lo^T gU, the products the kernel adds for flagged chunks;
  * `gram`: A and P from the Gram of bf16 midpoint factors (the prep);
  * `operands`: U, dX, dP, dA and the midpoint factors where the gradient
    products take them;
  * `images` (rounding, store): both chains over bf16 records, and bf16 images
    of every chunk's entry state and exit gradient.
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


def chunk_bwd(q, k, v, b, w, la, S, dO, dSn, *, regrouped=True, rounding=None, pairs=False, gram=None,
              operands=None):
    """Gradients of one chunk: returns (dq, dk, dv, db, dw, dla, dS).  `gram`
    (rounding): A and P from the Gram of bf16 midpoint factors, as the prep forms
    them on the tensor cores.  `operands` (rounding): the gradient products take
    bf16 U, dX, dP, dA and midpoint factors Qhat, Khat, Ehat, as the gradient
    kernel's UMMAs do (dP and dA against the factors; fp32 accumulation); only
    with regrouped=True and chunks within the midpoint split's range."""
    L = q.shape[0]
    G = np.cumsum(la, axis=0)
    GC = G[-1]
    e = b * k
    D = _pair_decay(G)
    strict = np.tril(np.ones((L, L)), -1)
    if gram is None:
        A = np.einsum("td,tsd,sd->ts", e, D, k) * strict
        P = np.einsum("td,tsd,sd->ts", q, D, k)
    else:
        r = min(32, L)
        Gr = G[r - 1]
        Eh, Qh, Kh = (gram(np.exp(G - Gr) * e), gram(np.exp(G - Gr) * q), gram(np.exp(Gr - G) * k))
        A = (Eh @ Kh.T) * strict
        P = np.tril(Qh @ Kh.T)
    T = np.linalg.inv(np.eye(L) + A)
    Eb, Qb, Kt = np.exp(G) * e, np.exp(G) * q, np.exp(GC - G) * k
    X = w * v - Eb @ S
    U = _mm(T, X, rounding, pairs, pairs)
    gU = Kt @ dSn + P.T @ dO
    dX = _mm(T.T, gU, rounding, pairs, False)
    dv, dw = dX * w, dX * v
    rq = operands or (lambda a: a)
    Uo, dXo = rq(U), rq(dX)
    dQb, dEb, dKt = dO @ S.T, -dXo @ S.T, Uo @ dSn.T
    dP = np.tril(dO @ Uo.T)
    dA = -(dXo @ Uo.T) * strict
    dS = np.exp(GC)[:, None] * dSn + Qb.T @ dO - Eb.T @ dX
    if regrouped:
        dPs = dP * strict                       # P's diagonal: apart
        diag = np.diag(dP)[:, None]
    else:
        dPs, diag = dP, np.zeros((L, 1))
    if operands is None:
        dq = np.exp(G) * dQb + np.einsum("ts,tsd,sd->td", dPs, D, k)
        de = np.exp(G) * dEb + np.einsum("ts,tsd,sd->td", dA, D, k)
        dkw_pair = np.einsum("ts,tsd,td->sd", dPs, D, q) + np.einsum("ts,tsd,td->sd", dA, D, e)
    else:  # through the midpoint split: e^{Gamma_t - Gamma_s} = e^{Gamma_t - Gamma_r} e^{Gamma_r - Gamma_s}
        r = min(32, L)
        up, dn = np.exp(G - G[r - 1]), np.exp(G[r - 1] - G)
        Kh, Qh, Eh = rq(dn * k), rq(up * q), rq(up * e)
        dPo, dAo = rq(dPs), rq(dA)
        dq = np.exp(G) * dQb + up * (dPo @ Kh)
        de = np.exp(G) * dEb + up * (dAo @ Kh)
        dkw_pair = dn * (dPo.T @ Qh + dAo.T @ Eh)
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


def _chains_rounded(x, S0, dO, dS_T, C, rd, st):
    """The two chains of the bf16 backward: the forward recompute over bf16 chunk
    records (NG, Y, Z) with the fp32 state read as a bf16 image, and the adjoint
    chain dS = e^{Gamma_C} dS' + NG^T bf16(dS') + QS^T dO over the same records.
    Returns the entry states and exit gradients of every chunk (fp32), for one
    (batch, head) given as [T, d] arrays."""
    from wy_model import chunk_record
    q, k, v, b, w, la = x
    T, dk = q.shape
    dv = v.shape[1]
    S = np.zeros((dk, dv)) if S0 is None else S0.copy()
    recs, entry = [], []
    for c0 in range(0, T, C):
        sl = slice(c0, min(c0 + C, T))
        gc, NG, QS, Y, _ = chunk_record(q[sl], k[sl], b[sl], la[sl], C)
        gc, NG, QS, Y = st(gc), rd(NG), rd(QS), rd(Y)
        recs.append((sl, gc, NG, QS))
        entry.append(S)
        S = st(gc[:, None] * S + NG @ rd(S) + Y @ rd(w[sl] * v[sl]))
    dS = np.zeros((dk, dv)) if dS_T is None else dS_T.copy()
    exit_ = [None] * len(recs)
    for i in reversed(range(len(recs))):
        sl, gc, NG, QS = recs[i]
        exit_[i] = dS
        dS = st(gc[:, None] * dS + NG.T @ rd(dS) + QS.T @ dO[sl])
    return entry, exit_, dS


def wy_backward(q, k, v, b, w, log_alpha, S0, dO, dS_T, C=64, images=None, **kw):
    """Gradients of sum(o * dO) + sum(S_T * dS_T) over [B,T,H,d] inputs, chunk by
    chunk in reverse; returns a dict like the oracle's backward.  `images`
    (rounding, store): the chains run over bf16 records and every chunk's
    gradients take the bf16 images of its entry state and exit gradient, as in
    the tensor-core backward; dS0 is then the adjoint chain's."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    out = {n: np.zeros(q.shape) for n in ("dq", "dk", "db", "dlog_alpha")}
    out.update({n: np.zeros(v.shape) for n in ("dv", "dw")})
    out["dS0"] = np.zeros((B, H, dk, dv))
    for bi in range(B):
        for h in range(H):
            if images is not None:
                rd, st = images
                xs = [a[bi, :, h] for a in (q, k, v, b, w, log_alpha)]
                entry, exit_, d0 = _chains_rounded(xs, None if S0 is None else S0[bi, h], dO[bi, :, h],
                                                   None if dS_T is None else dS_T[bi, h], C, rd, st)
                for i, c0 in enumerate(range(0, T, C)):
                    sl = slice(c0, min(c0 + C, T))
                    g = chunk_bwd(*(a[bi, sl, h] for a in (q, k, v, b, w, log_alpha)), rd(entry[i]),
                                  dO[bi, sl, h], rd(exit_[i]), **kw)
                    for n, x in zip(("dq", "dk", "dv", "db", "dw", "dlog_alpha"), g[:6]):
                        out[n][bi, sl, h] = x
                out["dS0"][bi, h] = d0
                continue
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
