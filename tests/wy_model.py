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
