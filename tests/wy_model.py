"""fp64 model of the chunkwise (WY) form of the gated delta rule.

This is the blocked algorithm the CUDA forward kernels implement, written in
numpy at full precision so that its algebra can be checked against the
token-by-token oracle before any kernel runs.  It is test infrastructure and
is not the oracle.

Per chunk of C tokens (the pages train with chunks of 64 tokens: iplexlaw.co.kr,
section "Procesamiento del token y entrenamiento paralelo"; zubnet.ai), with
Gamma_t the chunk-local cumulative log-decay (kept in fp32 on the GPU) and a
reference point r inside the chunk (its midpoint):
    Ehat_t = exp(Gamma_t - Gamma_r) (*) b_t (*) k_t      (decayed erase factor)
    Qhat_t = exp(Gamma_t - Gamma_r) (*) q_t
    Khat_s = exp(Gamma_r - Gamma_s) (*) k_s
    Ktil_s = exp(Gamma_C - Gamma_s) (*) k_s
    A = strictly-lower(Ehat Khat^T),   P = lower-inclusive(Qhat Khat^T)
    T = (I + A)^{-1},   Y = Ktil^T T,   PT = P T
    NG = -Y Ehat Diag(exp(Gamma_r)),   QS = (Qhat - PT Ehat) Diag(exp(Gamma_r))
and, with Z = w (*) v, the chunk maps the incoming state S to
    S_C = Diag(exp(Gamma_C)) S + NG S + Y Z,      O = QS S + PT Z.
(Equivalently U = T (Z - Ehat Diag(exp(Gamma_r)) S), O = Qhat Diag(exp(Gamma_r)) S
+ P U, S_C = Diag(exp(Gamma_C)) S + Ktil^T U.)  The decay is absorbed into
asymmetric erase/key factors and the lower triangular system (I + T)^{-1} is
solved per chunk, as the gist.science summary describes in section 3
("Efficient chunkwise parallel training").  Only Z depends on the values, so
every other part of the chunk's record is computed once for all value columns.
"""
import numpy as np


def chunk_record(q, k, b, la, C):
    """State-independent part of one chunk of L <= C tokens: (gc, NG, QS, Y, PT)."""
    L = q.shape[0]
    G = np.cumsum(la, axis=0)                       # Gamma_1..Gamma_L
    r = min(C // 2, L)
    Gr = G[r - 1] if r > 0 else np.zeros_like(G[0])
    up = np.exp(G - Gr)
    Eh = up * (b * k)
    Qh = up * q
    Kh = np.exp(Gr - G) * k
    Kt = np.exp(G[-1] - G) * k
    A = np.tril(Eh @ Kh.T, -1)
    P = np.tril(Qh @ Kh.T, 0)
    T = np.linalg.inv(np.eye(L) + A)
    Y = Kt.T @ T
    PT = P @ T
    er = np.exp(Gr)
    NG = -(Y @ Eh) * er[None, :]
    QS = (Qh - PT @ Eh) * er[None, :]
    return np.exp(G[-1]), NG, QS, Y, PT


def chunk_T(k, b, la, C):
    """T = (I + A)^{-1} of one chunk of L <= C tokens, A formed from the midpoint
    factors as in chunk_record."""
    L = k.shape[0]
    G = np.cumsum(la, axis=0)
    r = min(C // 2, L)
    Gr = G[r - 1] if r > 0 else np.zeros_like(G[0])
    A = np.tril((np.exp(G - Gr) * (b * k)) @ (np.exp(Gr - G) * k).T, -1)
    return np.linalg.inv(np.eye(L) + A)


def chunk_step(q, k, v, b, w, la, S, C):
    """One chunk of L <= C tokens for one (batch, head): returns (O, S_C)."""
    gc, NG, QS, Y, PT = chunk_record(q, k, b, la, C)
    Z = w * v
    O = QS @ S + PT @ Z
    S_new = gc[:, None] * S + NG @ S + Y @ Z
    return O, S_new


def wy_forward(q, k, v, b, w, log_alpha, S0=None, C=64):
    """[B,T,H,d] inputs (numpy, any float dtype) -> (o, S_T) in fp64."""
    q, k, v, b, w, la = (np.asarray(x, dtype=np.float64) for x in (q, k, v, b, w, log_alpha))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    o = np.zeros((B, T, H, dv))
    ST = np.zeros((B, H, dk, dv))
    for bi in range(B):
        for h in range(H):
            S = np.zeros((dk, dv)) if S0 is None else np.array(S0[bi, h], dtype=np.float64)
            for t0 in range(0, T, C):
                sl = slice(t0, min(T, t0 + C))
                O, S = chunk_step(q[bi, sl, h], k[bi, sl, h], v[bi, sl, h], b[bi, sl, h],
                                  w[bi, sl, h], la[bi, sl, h], S, C)
                o[bi, sl, h] = O
            ST[bi, h] = S
    return o, ST


def pair_record(r1, r2):
    """Two consecutive chunk records (gc, NG, QS, Y, PT) composed into one map of
    the state entering the first chunk.  With A = Diag(gc) + NG the transition of
    a chunk, S_1 = A_1 S + Y_1 Z_1 and S_2 = A_2 S_1 + Y_2 Z_2 give
        S_2 = Diag(gc_1 gc_2) S + NG' S + [Y_1' | Y_2] [Z_1; Z_2]
        NG' = Diag(gc_2) NG_1 + NG_2 Diag(gc_1) + NG_2 NG_1,   Y_1' = Diag(gc_2) Y_1 + NG_2 Y_1
    and the second chunk's outputs O_2 = QS_2 S_1 + PT_2 Z_2 become
        O_2 = QS_2' S + PT_21 Z_1 + PT_2 Z_2,   QS_2' = QS_2 Diag(gc_1) + QS_2 NG_1,   PT_21 = QS_2 Y_1.
    Returns (gc', NG', Y_1', QS_2', PT_21)."""
    g1, NG1, _, Y1, _ = r1
    g2, NG2, QS2, _, _ = r2
    NGp = g2[:, None] * NG1 + NG2 * g1[None, :] + NG2 @ NG1
    Y1p = g2[:, None] * Y1 + NG2 @ Y1
    QS2p = QS2 * g1[None, :] + QS2 @ NG1
    return g1 * g2, NGp, Y1p, QS2p, QS2 @ Y1


def wy_forward_pairs(q, k, v, b, w, log_alpha, S0=None, C=64):
    """wy_forward with the state carried over pairs of chunks (pair_record); an
    odd last chunk is a step of its own."""
    q, k, v, b, w, la = (np.asarray(x, dtype=np.float64) for x in (q, k, v, b, w, log_alpha))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    o = np.zeros((B, T, H, dv))
    ST = np.zeros((B, H, dk, dv))
    for bi in range(B):
        for h in range(H):
            S = np.zeros((dk, dv)) if S0 is None else np.array(S0[bi, h], dtype=np.float64)
            chunks = [slice(t0, min(T, t0 + C)) for t0 in range(0, T, C)]
            for i in range(0, len(chunks), 2):
                s1 = chunks[i]
                r1 = chunk_record(q[bi, s1, h], k[bi, s1, h], b[bi, s1, h], la[bi, s1, h], C)
                Z1 = w[bi, s1, h] * v[bi, s1, h]
                o[bi, s1, h] = r1[2] @ S + r1[4] @ Z1
                if i + 1 == len(chunks):
                    S = r1[0][:, None] * S + r1[1] @ S + r1[3] @ Z1
                    break
                s2 = chunks[i + 1]
                r2 = chunk_record(q[bi, s2, h], k[bi, s2, h], b[bi, s2, h], la[bi, s2, h], C)
                Z2 = w[bi, s2, h] * v[bi, s2, h]
                gp, NGp, Y1p, QS2p, PT21 = pair_record(r1, r2)
                o[bi, s2, h] = QS2p @ S + PT21 @ Z1 + r2[4] @ Z2
                S = gp[:, None] * S + NGp @ S + Y1p @ Z1 + r2[3] @ Z2
            ST[bi, h] = S
    return o, ST


def group_forward(q, k, v, b, w, log_alpha, S0=None, C=64, m=4, rounding=None, store=None, n_rounded=False):
    """wy_forward with the state carried over groups of m chunks: one step of the
    serial chain per group, with the group's composed map
        S_out = Diag(gp) S + NGp S + Np,   A_i = Diag(gc_i) + NG_i,
        Diag(gp) + NGp = A_m ... A_1,      Np = sum_j (A_m ... A_{j+1}) Y_j Z_j,
    and each chunk's entry state from the group's by the prefix of that product
    (state-independent work, off the serial path).  `rounding` (bf16) is applied
    to every tensor-core operand and `store` (fp32) to every stored accumulator,
    as the bf16 kernels do; `n_rounded` also rounds Np where it is read.  [B,T,H,d]
    inputs -> (o, S_T)."""
    rd = rounding or (lambda x: x)
    st = store or (lambda x: x)
    q, k, v, b, w, la = (np.asarray(x, dtype=np.float64) for x in (q, k, v, b, w, log_alpha))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    o = np.zeros((B, T, H, dv))
    ST = np.zeros((B, H, dk, dv))
    for bi in range(B):
        for h in range(H):
            S = np.zeros((dk, dv)) if S0 is None else np.array(S0[bi, h], dtype=np.float64)
            chunks = [slice(t0, min(T, t0 + C)) for t0 in range(0, T, C)]
            for g0 in range(0, len(chunks), m):
                Sx = rd(S)
                gp, NGp, Np = np.ones(dk), np.zeros((dk, dk)), np.zeros((dk, dv))
                for sl in chunks[g0:g0 + m]:
                    gc, NG, QS, Y, PT = chunk_record(q[bi, sl, h], k[bi, sl, h], b[bi, sl, h], la[bi, sl, h], C)
                    gc, NG, QS, Y, PT = st(gc), rd(NG), rd(QS), rd(Y), rd(PT)
                    Z = rd(w[bi, sl, h] * v[bi, sl, h])
                    Nr = rd(Np) if n_rounded else Np
                    Si = st(gp[:, None] * S + rd(NGp) @ Sx + Nr)           # this chunk's entry state
                    o[bi, sl, h] = rd(QS @ rd(Si) + PT @ Z) if rounding else QS @ Si + PT @ Z
                    NGp, Np = (st(gc[:, None] * NGp + NG * gp[None, :] + NG @ rd(NGp)),
                               st(gc[:, None] * Np + NG @ rd(Np) + Y @ Z))
                    gp = st(gc * gp)
                S = st(gp[:, None] * S + rd(NGp) @ Sx + (rd(Np) if n_rounded else Np))
            ST[bi, h] = S
    return o, ST


def group_adjoint(q, k, v, b, w, log_alpha, dO, dS_T=None, C=64, m=4):
    """The adjoint chain over groups of m chunks: dS, the gradient of
    sum(o * dO) + sum(S_T * dS_T) with respect to the state entering each chunk,
    stepping once per group.  With A_i = Diag(gc_i) + NG_i the chunk transition,
    the gradient entering a group is (A_m ... A_1)^T dS_out + sum_i (A_{i-1} ... A_1)^T
    QS_i^T dO_i, and the gradient leaving chunk i inside the group (what each
    chunk's gradients need) follows from dS_out by the suffix products.  The
    outputs O_i = QS_i S_i + PT_i Z_i only make the dO terms; Z does not enter.
    [B,T,H,d] inputs -> (dS0 [B,H,dk,dv], dS_out [B,H,nchunks,dk,dv])."""
    q, k, b, la, dO = (np.asarray(x, dtype=np.float64) for x in (q, k, b, log_alpha, dO))
    B, T, H, dk = q.shape
    dv = dO.shape[-1]
    chunks = [slice(t0, min(T, t0 + C)) for t0 in range(0, T, C)]
    dS0 = np.zeros((B, H, dk, dv))
    dS_out = np.zeros((B, H, len(chunks), dk, dv))
    for bi in range(B):
        for h in range(H):
            g = np.zeros((dk, dv)) if dS_T is None else np.array(dS_T[bi, h], dtype=np.float64)
            for g0 in reversed(range(0, len(chunks), m)):
                idx = list(range(g0, min(g0 + m, len(chunks))))
                A, QO = [], []
                for i in idx:
                    sl = chunks[i]
                    gc, NG, QS, _, _ = chunk_record(q[bi, sl, h], k[bi, sl, h], b[bi, sl, h], la[bi, sl, h], C)
                    A.append(np.diag(gc) + NG)
                    QO.append(QS.T @ dO[bi, sl, h])
                # gradient leaving each chunk of the group: suffix products from the group's exit
                for j, i in enumerate(idx):
                    d = g.copy()
                    for l in range(len(idx) - 1, j, -1):   # chunks after i, innermost last
                        d = A[l].T @ d + QO[l]
                    dS_out[bi, h, i] = d
                # gradient entering the group: the composed map and the prefix-weighted dO terms
                Ag = np.eye(dk)
                acc = np.zeros((dk, dv))
                for j in range(len(idx)):
                    acc += Ag.T @ QO[j]                    # (A_{j-1} ... A_1)^T QS_j^T dO_j
                    Ag = A[j] @ Ag
                g = Ag.T @ g + acc
            dS0[bi, h] = g
    return dS0, dS_out
