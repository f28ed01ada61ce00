"""Pins for the fp64 oracle: facts fixed by the pages and by the mathematics.

Each pin takes an oracle handle (``oracle.Oracle``) and raises AssertionError
when the oracle disagrees.  None of them re-types the oracle's own loop: they
use a hand-worked example, the published special cases (KDA, Gated DeltaNet,
DeltaNet) written in their own operator form, closed forms, a brute-force
product of explicit transition matrices, and structural invariants.  The
mutation test runs the same pins against deliberately broken copies of the
oracle and expects each copy to fail at least one of them.
"""
from __future__ import annotations

import json
from fractions import Fraction
from pathlib import Path

import numpy as np

GOLDEN = Path(__file__).resolve().parent / "golden"


def _rng(seed):
    return np.random.default_rng(seed)


def _unit(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def _inputs(T, dk, dv, seed, B=1, H=1, S0=True):
    r = _rng(seed)
    q = _unit(r.standard_normal((B, T, H, dk)))
    k = _unit(r.standard_normal((B, T, H, dk)))
    v = r.standard_normal((B, T, H, dv))
    b = r.uniform(0.0, 1.0, (B, T, H, dk))
    w = r.uniform(0.0, 1.0, (B, T, H, dv))
    la = -np.exp(r.uniform(-5.0, -0.5, (B, T, H, dk)))
    s0 = r.standard_normal((B, H, dk, dv)) * 0.3 if S0 else None
    return q, k, v, b, w, la, s0


def _close(a, b, tol, what):
    err = np.max(np.abs(np.asarray(a) - np.asarray(b)))
    scale = max(1.0, float(np.max(np.abs(b))))
    assert err <= tol * scale, f"{what}: max abs err {err:.3e} > {tol:.1e} * {scale:.3g}"


# ---------------------------------------------------------------------------
# 1. Hand-worked scalar example (tests/golden/scalar_hand_3tok.json).
def pin_scalar_hand(orc):
    g = json.loads((GOLDEN / "scalar_hand_3tok.json").read_text())

    def col(name):
        return np.array(g[name], dtype=np.float64).reshape(1, -1, 1, 1)
    o, st = orc.fwd(col("q"), col("k"), col("v"), col("b"), col("w"), np.log(col("alpha")),
                    S0=np.full((1, 1, 1, 1), g["s0"]))
    want_o = [float(Fraction(x)) for x in g["o"]]
    _close(o.ravel(), want_o, 1e-14, "scalar hand example o")
    _close(st.ravel(), [float(Fraction(g["s_T"]))], 1e-14, "scalar hand example S_T")


# ---------------------------------------------------------------------------
# 2-4. Published special cases, each in its own operator form.
def _kda_reference(q, k, v, beta, alpha, S0):
    """KDA: S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T, o_t = S_t^T q_t."""
    T, dk = k.shape
    S = S0.copy()
    o = np.zeros((T, v.shape[1]))
    for t in range(T):
        E = np.eye(dk) - beta[t] * np.outer(k[t], k[t])
        S = E @ np.diag(alpha[t]) @ S + beta[t] * np.outer(k[t], v[t])
        o[t] = S.T @ q[t]
    return o, S


def pin_reduces_to_kda(orc):
    """b = w = beta (one scalar per token) gives Kimi Delta Attention (iplexlaw
    page, 'Decisiones independientes en dos ejes'; gist.science section 1)."""
    T, dk, dv = 12, 5, 3
    q, k, v, _, _, la, s0 = _inputs(T, dk, dv, seed=11)
    beta = _rng(12).uniform(0.05, 1.0, T)
    b = np.broadcast_to(beta[None, :, None, None], (1, T, 1, dk)).copy()
    w = np.broadcast_to(beta[None, :, None, None], (1, T, 1, dv)).copy()
    o, st = orc.fwd(q, k, v, b, w, la, S0=s0)
    ro, rs = _kda_reference(q[0, :, 0], k[0, :, 0], v[0, :, 0], beta, np.exp(la[0, :, 0]), s0[0, 0])
    _close(o[0, :, 0], ro, 1e-12, "KDA reduction o")
    _close(st[0, 0], rs, 1e-12, "KDA reduction S_T")


def pin_reduces_to_gated_deltanet(orc):
    """b = w = beta and a scalar decay per token gives Gated DeltaNet:
    S_t = alpha_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T."""
    T, dk, dv = 10, 4, 6
    q, k, v, _, _, _, s0 = _inputs(T, dk, dv, seed=21)
    r = _rng(22)
    beta = r.uniform(0.05, 1.0, T)
    a = np.exp(-np.exp(r.uniform(-4, 0, T)))
    b = np.broadcast_to(beta[None, :, None, None], (1, T, 1, dk)).copy()
    w = np.broadcast_to(beta[None, :, None, None], (1, T, 1, dv)).copy()
    la = np.broadcast_to(np.log(a)[None, :, None, None], (1, T, 1, dk)).copy()
    o, st = orc.fwd(q, k, v, b, w, la, S0=s0)
    S = s0[0, 0].copy()
    for t in range(T):
        kt = k[0, t, 0]
        S = a[t] * (np.eye(dk) - beta[t] * np.outer(kt, kt)) @ S + beta[t] * np.outer(kt, v[0, t, 0])
        _close(o[0, t, 0], S.T @ q[0, t, 0], 1e-12, f"Gated DeltaNet reduction o[{t}]")
    _close(st[0, 0], S, 1e-12, "Gated DeltaNet reduction S_T")


def pin_reduces_to_deltanet(orc):
    """Additionally alpha = 1 gives DeltaNet: S_t = (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T."""
    T, dk, dv = 9, 3, 5
    q, k, v, _, _, _, s0 = _inputs(T, dk, dv, seed=31)
    beta = _rng(32).uniform(0.05, 1.0, T)
    b = np.broadcast_to(beta[None, :, None, None], (1, T, 1, dk)).copy()
    w = np.broadcast_to(beta[None, :, None, None], (1, T, 1, dv)).copy()
    o, st = orc.fwd(q, k, v, b, w, np.zeros((1, T, 1, dk)), S0=s0)
    S = s0[0, 0].copy()
    for t in range(T):
        kt = k[0, t, 0]
        S = S - beta[t] * np.outer(kt, kt @ S) + beta[t] * np.outer(kt, v[0, t, 0])
        _close(o[0, t, 0], S.T @ q[0, t, 0], 1e-12, f"DeltaNet reduction o[{t}]")
    _close(st[0, 0], S, 1e-12, "DeltaNet reduction S_T")


# ---------------------------------------------------------------------------
# 5. Exact recall: alpha = 1, b = w = 1, |k| = 1  =>  S_t^T k_t = v_t.
def pin_exact_recall(orc):
    T, dk, dv = 16, 8, 5
    q, k, v, _, _, _, s0 = _inputs(T, dk, dv, seed=41)
    ones_k = np.ones((1, T, 1, dk))
    o, _ = orc.fwd(k, k, v, ones_k, np.ones((1, T, 1, dv)), np.zeros((1, T, 1, dk)), S0=s0)
    _close(o, v, 1e-13, "exact recall S_t^T k_t = v_t")


# ---------------------------------------------------------------------------
# 6. Pure decay: b = w = 0  =>  S_t = Diag(prod alpha) S_0, o_t = S_t^T q_t.
def pin_pure_decay(orc):
    T, dk, dv = 20, 6, 4
    q, k, v, _, _, la, s0 = _inputs(T, dk, dv, seed=51)
    o, st = orc.fwd(q, k, v, np.zeros((1, T, 1, dk)), np.zeros((1, T, 1, dv)), la, S0=s0)
    cum = np.exp(np.cumsum(la[0, :, 0], axis=0))  # [T, dk]
    for t in range(T):
        St = cum[t][:, None] * s0[0, 0]
        _close(o[0, t, 0], St.T @ q[0, t, 0], 1e-13, f"pure decay o[{t}]")
    _close(st[0, 0], cum[-1][:, None] * s0[0, 0], 1e-13, "pure decay S_T")


# ---------------------------------------------------------------------------
# 7. Brute-force product form (zubnet.ai update equation; gist.science section 1):
#    S_t = M_t S_{t-1} + k_t z_t^T with M_t = (I - k_t e_t^T) D_t, unrolled.
def pin_product_form(orc):
    for (T, dk, dv, seed) in ((1, 3, 2, 61), (5, 4, 7, 62), (8, 8, 8, 63), (7, 6, 3, 64)):
        q, k, v, b, w, la, s0 = _inputs(T, dk, dv, seed=seed)
        b = b * 2.0  # the erase range [0, 2] of the ablation is not clamped
        o, st = orc.fwd(q, k, v, b, w, la, S0=s0)
        Ms, zs = [], []
        for t in range(T):
            kt, et = k[0, t, 0], b[0, t, 0] * k[0, t, 0]
            Ms.append((np.eye(dk) - np.outer(kt, et)) @ np.diag(np.exp(la[0, t, 0])))
            zs.append(np.outer(kt, w[0, t, 0] * v[0, t, 0]))
        for t in range(T):
            prod = np.eye(dk)
            for m in Ms[: t + 1]:
                prod = m @ prod
            St = prod @ s0[0, 0]
            for s in range(t + 1):
                tail = np.eye(dk)
                for m in Ms[s + 1: t + 1]:
                    tail = m @ tail
                St = St + tail @ zs[s]
            _close(o[0, t, 0], St.T @ q[0, t, 0], 1e-12, f"product form o[{t}] (T={T})")
            if t == T - 1:
                _close(st[0, 0], St, 1e-12, f"product form S_T (T={T})")


# ---------------------------------------------------------------------------
# 8. Linearity: o and S_T are linear in (S_0, v) jointly, and o is linear in q.
def pin_linearity(orc):
    T, dk, dv = 14, 5, 4
    q, k, v1, b, w, la, s1 = _inputs(T, dk, dv, seed=71)
    _, _, v2, _, _, _, s2 = _inputs(T, dk, dv, seed=72)
    q2 = _inputs(T, dk, dv, seed=73)[0]
    a, c = 0.7, -1.3
    o1, st1 = orc.fwd(q, k, v1, b, w, la, S0=s1)
    o2, st2 = orc.fwd(q, k, v2, b, w, la, S0=s2)
    o12, st12 = orc.fwd(q, k, a * v1 + c * v2, b, w, la, S0=a * s1 + c * s2)
    _close(o12, a * o1 + c * o2, 1e-12, "superposition o")
    _close(st12, a * st1 + c * st2, 1e-12, "superposition S_T")
    oq2, _ = orc.fwd(q2, k, v1, b, w, la, S0=s1)
    oq, _ = orc.fwd(a * q + c * q2, k, v1, b, w, la, S0=s1)
    _close(oq, a * o1 + c * oq2, 1e-12, "linearity in q")


# ---------------------------------------------------------------------------
# 9. Value columns are independent: the erase and the decay act on key rows.
def pin_column_permutation(orc):
    T, dk, dv = 11, 4, 6
    q, k, v, b, w, la, s0 = _inputs(T, dk, dv, seed=81)
    perm = _rng(82).permutation(dv)
    o, st = orc.fwd(q, k, v, b, w, la, S0=s0)
    op, stp = orc.fwd(q, k, v[..., perm], b, w[..., perm], la, S0=s0[..., perm])
    _close(op, o[..., perm], 1e-13, "column permutation o")
    _close(stp, st[..., perm], 1e-13, "column permutation S_T")
    oh, sth = orc.fwd(q, k, v[..., :3], b, w[..., :3], la, S0=s0[..., :3])
    _close(oh, o[..., :3], 1e-13, "column split o")
    _close(sth, st[..., :3], 1e-13, "column split S_T")


# ---------------------------------------------------------------------------
# 10. Splitting the sequence: fwd(0..T) == fwd(0..T1) then fwd(T1..T) from S_T1.
def pin_sequence_split(orc):
    T, T1, dk, dv = 23, 9, 5, 4
    q, k, v, b, w, la, s0 = _inputs(T, dk, dv, seed=91)
    o, st = orc.fwd(q, k, v, b, w, la, S0=s0)
    sl = slice(0, T1)
    oa, sa = orc.fwd(q[:, sl], k[:, sl], v[:, sl], b[:, sl], w[:, sl], la[:, sl], S0=s0)
    sl = slice(T1, T)
    ob, sb = orc.fwd(q[:, sl], k[:, sl], v[:, sl], b[:, sl], w[:, sl], la[:, sl], S0=sa)
    _close(np.concatenate([oa, ob], axis=1), o, 1e-13, "sequence split o")
    _close(sb, st, 1e-13, "sequence split S_T")


# ---------------------------------------------------------------------------
# 11. (batch, head) pairs are independent, and the layout puts each where it belongs.
def pin_batch_head_independence(orc):
    B, T, H, dk, dv = 2, 7, 3, 4, 5
    q, k, v, b, w, la, s0 = _inputs(T, dk, dv, seed=101, B=B, H=H)
    o, st = orc.fwd(q, k, v, b, w, la, S0=s0)
    for bi in range(B):
        for h in range(H):
            sl = (slice(bi, bi + 1), slice(None), slice(h, h + 1))
            oo, ss = orc.fwd(q[sl], k[sl], v[sl], b[sl], w[sl], la[sl], S0=s0[bi:bi + 1, h:h + 1])
            _close(o[sl], oo, 0.0, f"pair ({bi},{h}) o")
            _close(st[bi:bi + 1, h:h + 1], ss, 0.0, f"pair ({bi},{h}) S_T")


# ---------------------------------------------------------------------------
# 12. Orthonormal keys (alpha = 1, b = w = 1, S_0 = 0): each write lands in a
#     direction no earlier key reads, so nothing is erased; querying an earlier
#     key returns its value, a later key returns zero, and S_T = sum_i k_i v_i^T.
def pin_orthonormal_keys(orc):
    dk, dv = 6, 4
    r = _rng(121)
    K = np.linalg.qr(r.standard_normal((dk, dk)))[0].T          # rows: orthonormal keys
    v = r.standard_normal((1, dk, 1, dv))
    k = K.reshape(1, dk, 1, dk)
    q = np.empty_like(k)
    for t in range(dk):
        q[0, t, 0] = K[(t * 5 + 2) % dk]                         # a key written before, at t, or later
    one_k, one_v = np.ones((1, dk, 1, dk)), np.ones((1, dk, 1, dv))
    o, st = orc.fwd(q, k, v, one_k, one_v, np.zeros((1, dk, 1, dk)), S0=None)
    for t in range(dk):
        j = (t * 5 + 2) % dk
        _close(o[0, t, 0], v[0, j, 0] if j <= t else np.zeros(dv), 1e-13, f"orthonormal keys o[{t}]")
    _close(st[0, 0], K.T @ v[0, :, 0], 1e-13, "orthonormal keys S_T")


# ---------------------------------------------------------------------------
# 13. One basis key e_i, erase gate beta on channel i, write gate omega, decay
#     alpha_i: x_t = S_t^T e_i obeys x_t = alpha_i (1 - beta) x_{t-1} + omega v,
#     so x_t = omega v (1 - rho^t) / (1 - rho) with rho = alpha_i (1 - beta).  The
#     decay acts before the erase reads, the erase uses b and the write uses w.
def pin_gated_geometric(orc):
    T, dk, dv, i = 12, 5, 3, 2
    beta, omega, alpha = 0.3, 0.7, 0.9
    r = _rng(131)
    vv = r.standard_normal(dv)
    k = np.zeros((1, T, 1, dk)); k[..., i] = 1.0
    b = np.full((1, T, 1, dk), 0.55); b[..., i] = beta          # other channels' gates never act
    w = np.full((1, T, 1, dv), omega)
    la = np.full((1, T, 1, dk), np.log(0.5)); la[..., i] = np.log(alpha)
    v = np.broadcast_to(vv, (1, T, 1, dv)).copy()
    o, st = orc.fwd(k, k, v, b, w, la, S0=None)
    rho = alpha * (1.0 - beta)
    for t in range(T):
        _close(o[0, t, 0], omega * vv * (1.0 - rho ** (t + 1)) / (1.0 - rho), 1e-13, f"gated geometric o[{t}]")
    want = np.zeros((dk, dv)); want[i] = omega * vv * (1.0 - rho ** T) / (1.0 - rho)
    _close(st[0, 0], want, 1e-13, "gated geometric S_T")


ALL_PINS = [pin_scalar_hand, pin_reduces_to_kda, pin_reduces_to_gated_deltanet,
            pin_reduces_to_deltanet, pin_exact_recall, pin_pure_decay, pin_product_form,
            pin_linearity, pin_column_permutation, pin_sequence_split,
            pin_batch_head_independence, pin_orthonormal_keys, pin_gated_geometric]
