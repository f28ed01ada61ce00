"""Pins of the oracle's backward (gdn2_oracle_bwd): central finite differences
of the forward oracle, a closed form, the KDA reduction of the gate gradients,
and linearity in the incoming gradients (CPU only).

The backward the pages describe keeps the per-channel gates inside the
gradient aggregation ("Gated DeltaNet-2", iplexlaw.co.kr, section
"Procesamiento del token y entrenamiento paralelo"); each pin below checks a
consequence of the chain rule on the token recurrence, not a re-typed copy of
the oracle's loop.
"""
import numpy as np
import pytest

import oracle

NAMES = ("q", "k", "v", "b", "w", "log_alpha")


def _problem(T, dk, dv, seed, B=1, H=2, erase_max=2.0):
    r = np.random.default_rng(seed)
    d = dict(q=r.standard_normal((B, T, H, dk)), k=r.standard_normal((B, T, H, dk)) * 0.6,
             v=r.standard_normal((B, T, H, dv)), b=r.uniform(0.0, erase_max, (B, T, H, dk)),
             w=r.uniform(0.0, 1.0, (B, T, H, dv)), log_alpha=-np.exp(r.uniform(-4.0, 1.0, (B, T, H, dk))))
    S0 = 0.5 * r.standard_normal((B, H, dk, dv))
    dO = r.standard_normal((B, T, H, dv))
    dST = r.standard_normal((B, H, dk, dv))
    return d, S0, dO, dST


def _loss(d, S0, dO, dST):
    o, st = oracle.fwd(*(d[n] for n in NAMES), S0=S0)
    return float(np.sum(o * dO) + np.sum(st * dST))


@pytest.mark.parametrize("T", [1, 9, 70])
def test_every_gradient_matches_central_differences(T):
    """T = 70 crosses the 64-token stretch whose states the backward recomputes."""
    d, S0, dO, dST = _problem(T, 3, 2, seed=T)
    g = oracle.bwd(*(d[n] for n in NAMES), S0, dO, dST)
    h = 1e-6
    for name, gname in zip(NAMES + ("S0",), ("dq", "dk", "dv", "db", "dw", "dlog_alpha", "dS0")):
        x = S0 if name == "S0" else d[name]
        fd = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            keep = x[idx]
            x[idx] = keep + h
            lp = _loss(d, S0, dO, dST)
            x[idx] = keep - h
            lm = _loss(d, S0, dO, dST)
            x[idx] = keep
            fd[idx] = (lp - lm) / (2 * h)
        scale = max(np.abs(fd).max(), 1e-12)
        assert np.abs(g[gname] - fd).max() <= 2e-6 * scale + 1e-8, (name, np.abs(g[gname] - fd).max(), scale)


def test_pure_decay_closed_form():
    """b = w = 0: the state only decays (S_t = D_1..t S0) and the adjoint only
    decays back, so every gradient has a closed form in the decay products."""
    T, dk, dv = 7, 4, 3
    d, S0, dO, dST = _problem(T, dk, dv, seed=11, H=1)
    d["b"] = np.zeros_like(d["b"])
    d["w"] = np.zeros_like(d["w"])
    g = oracle.bwd(*(d[n] for n in NAMES), S0, dO, dST)
    a = np.exp(d["log_alpha"][0, :, 0])        # [T, dk]
    q, k, v = d["q"][0, :, 0], d["k"][0, :, 0], d["v"][0, :, 0]
    o_grad = dO[0, :, 0]
    s0, dst = S0[0, 0], dST[0, 0]
    pre = np.cumprod(a, axis=0)                # D_1..t
    # dS'_t = sum_{s >= t} D_{t+1..s} q_s dO_s^T + D_{t+1..T} dS_T
    dSp = []
    for t in range(T):
        acc = np.prod(a[t + 1:], axis=0)[:, None] * dst
        for s in range(t, T):
            acc = acc + (np.prod(a[t + 1:s + 1], axis=0) * q[s])[:, None] * o_grad[s][None, :]
        dSp.append(acc)
    for t in range(T):
        St = pre[t][:, None] * s0
        np.testing.assert_allclose(g["dq"][0, t, 0], St @ o_grad[t], rtol=1e-10, atol=1e-12)
        du = dSp[t].T @ k[t]
        np.testing.assert_allclose(g["dw"][0, t, 0], du * v[t], rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(g["dv"][0, t, 0], 0.0, atol=1e-15)
        np.testing.assert_allclose(g["dk"][0, t, 0], 0.0, atol=1e-12)
        np.testing.assert_allclose(g["db"][0, t, 0], -(St @ du) * k[t], rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(g["dlog_alpha"][0, t, 0], np.sum(dSp[t] * St, axis=1), rtol=1e-10, atol=1e-12)
    dS0 = a[0][:, None] * dSp[0]
    np.testing.assert_allclose(g["dS0"][0, 0], dS0, rtol=1e-10, atol=1e-12)


def test_kda_reduction_of_the_gate_gradients():
    """b = w = beta (a scalar per token, KDA): dL/dbeta_t = sum_i db_ti + sum_j dw_tj,
    checked against central differences in beta itself."""
    T, dk, dv = 6, 3, 4
    d, S0, dO, dST = _problem(T, dk, dv, seed=12, H=1)
    beta = np.random.default_rng(13).uniform(0.1, 0.9, (1, T, 1))

    def with_beta(bt):
        e = dict(d)
        e["b"] = np.repeat(bt[..., None], dk, axis=-1)
        e["w"] = np.repeat(bt[..., None], dv, axis=-1)
        return e

    g = oracle.bwd(*(with_beta(beta)[n] for n in NAMES), S0, dO, dST)
    agg = g["db"].sum(-1) + g["dw"].sum(-1)
    h = 1e-6
    for t in range(T):
        bp, bm = beta.copy(), beta.copy()
        bp[0, t, 0] += h
        bm[0, t, 0] -= h
        fd = (_loss(with_beta(bp), S0, dO, dST) - _loss(with_beta(bm), S0, dO, dST)) / (2 * h)
        assert abs(agg[0, t, 0] - fd) <= 1e-6 * max(1.0, abs(fd)), (t, agg[0, t, 0], fd)


def test_gradients_are_linear_in_the_incoming_gradients():
    d, S0, dO, dST = _problem(20, 4, 3, seed=14)
    r = np.random.default_rng(15)
    dO2, dST2 = r.standard_normal(dO.shape), r.standard_normal(dST.shape)
    g1 = oracle.bwd(*(d[n] for n in NAMES), S0, dO, dST)
    g2 = oracle.bwd(*(d[n] for n in NAMES), S0, dO2, dST2)
    g3 = oracle.bwd(*(d[n] for n in NAMES), S0, 2.0 * dO - 0.5 * dO2, 2.0 * dST - 0.5 * dST2)
    for n in g1:
        np.testing.assert_allclose(g3[n], 2.0 * g1[n] - 0.5 * g2[n], rtol=1e-10, atol=1e-10)
    gz = oracle.bwd(*(d[n] for n in NAMES), S0, np.zeros_like(dO), None)
    for n in gz:
        assert np.all(gz[n] == 0.0)
