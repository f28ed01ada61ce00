"""Pins of the layer oracle (oracle/layer.py): facts its definitions fix,
checked without re-typing them (CPU only).

"Gated DeltaNet-2", iplexlaw.co.kr, section "Procesamiento del token y
entrenamiento paralelo": L2-normalised queries and keys, sigmoid gates, RMS
normalisation of the output and an independent output gate.
"""
import numpy as np
import pytest

import oracle
from oracle import layer
from oracle_pins import _inputs

EPS = 1e-6


def _layer_inputs(T=7, dk=6, dv=5, seed=0, B=2, H=2):
    r = np.random.default_rng(seed)
    q = r.standard_normal((B, T, H, dk)) * 2.0
    k = r.standard_normal((B, T, H, dk)) * 1.5
    v = r.standard_normal((B, T, H, dv))
    bl = r.standard_normal((B, T, H, dk))
    wl = r.standard_normal((B, T, H, dv))
    al = 2.0 + r.standard_normal((B, T, H, dk))
    gl = r.standard_normal((B, T, H, dv))
    nw = 1.0 + 0.1 * r.standard_normal(dv)
    s0 = 0.3 * r.standard_normal((B, H, dk, dv))
    return q, k, v, bl, wl, al, gl, nw, s0


def test_query_and_key_scale_invariance():
    """Scaling each token's q or k by a positive factor changes nothing (L2 norm)."""
    q, k, v, bl, wl, al, gl, nw, s0 = _layer_inputs(seed=1)
    r = np.random.default_rng(2)
    cq = np.exp(r.uniform(-2, 2, q.shape[:-1] + (1,)))
    ck = np.exp(r.uniform(-2, 2, k.shape[:-1] + (1,)))
    y1, s1 = layer.layer_fwd(q, k, v, bl, wl, al, gl, nw, EPS, S0=s0)
    y2, s2 = layer.layer_fwd(q * cq, k * ck, v, bl, wl, al, gl, nw, EPS, S0=s0)
    # exact up to EPS_L2 / |x|^2 (about 1e-6 here)
    np.testing.assert_allclose(y1, y2, rtol=0, atol=1e-4 * np.abs(y1).max())
    np.testing.assert_allclose(s1, s2, rtol=0, atol=1e-4 * np.abs(s1).max())


def test_normalised_keys_have_unit_norm_and_recall_exactly():
    """With alpha = 1 (decay logit +inf), b = w = 1 (logits +inf) the operator on the
    normalised keys recalls the value just written: S_t^T k_hat_t = v_t, the
    closed form of the delta rule on a unit key."""
    q, k, v, bl, wl, al, gl, nw, s0 = _layer_inputs(seed=3)
    big = np.full_like(bl, 60.0)
    qh, kh, b, w, la = layer.prologue(q, k, big, np.full_like(wl, 60.0), np.full_like(al, 60.0))
    np.testing.assert_allclose(np.linalg.norm(kh, axis=-1), 1.0, atol=1e-5)
    for t in range(1, q.shape[1] + 1):
        _, st = oracle.fwd(kh[:, :t], kh[:, :t], v[:, :t], b[:, :t], w[:, :t], la[:, :t], S0=s0)
        recall = np.einsum("bhij,bhi->bhj", st, kh[:, t - 1])
        np.testing.assert_allclose(recall, v[:, t - 1], atol=1e-5)


def test_zero_logits_give_half_gates_and_half_decay():
    """sigmoid(0) = 1/2 exactly: zero logits are the operator with b = w = 1/2 and
    alpha = 1/2 on the normalised q, k, and the output gate halves the norm."""
    q, k, v, bl, wl, al, gl, nw, s0 = _layer_inputs(seed=4)
    z = np.zeros_like
    y, st = layer.layer_fwd(q, k, v, z(bl), z(wl), z(al), z(gl), np.ones_like(nw), EPS, S0=s0)
    qh, kh = layer.l2_normalise(q), layer.l2_normalise(k)
    o, st2 = oracle.fwd(qh, kh, v, np.full_like(bl, 0.5), np.full_like(wl, 0.5),
                        np.full_like(al, np.log(0.5)), S0=s0)
    np.testing.assert_allclose(st, st2, rtol=1e-12, atol=1e-14)
    rms = np.sqrt(np.mean(o * o, axis=-1, keepdims=True) + EPS)
    np.testing.assert_allclose(y, 0.5 * o / rms, rtol=1e-12, atol=1e-14)


def test_output_rows_have_unit_rms_before_weight_and_gate():
    """Open output gate (logit +inf) and unit weight: every output row has RMS 1
    (up to eps), whatever its scale before the norm."""
    q, k, v, bl, wl, al, gl, nw, s0 = _layer_inputs(seed=5)
    for scale in (1e-2, 1.0, 1e3):
        y, _ = layer.layer_fwd(q, k, scale * v, bl, wl, al, np.full_like(gl, 60.0), np.ones_like(nw),
                               1e-12, S0=scale * s0)
        np.testing.assert_allclose(np.sqrt(np.mean(y * y, axis=-1)), 1.0, rtol=1e-6)


def test_closed_output_gate_and_weight_scale():
    """A closed gate (logit -inf) zeroes the output; the weight scales each value
    channel linearly."""
    q, k, v, bl, wl, al, gl, nw, s0 = _layer_inputs(seed=6)
    y0, _ = layer.layer_fwd(q, k, v, bl, wl, al, np.full_like(gl, -800.0), nw, EPS, S0=s0)
    assert np.all(y0 == 0.0)
    y1, _ = layer.layer_fwd(q, k, v, bl, wl, al, gl, nw, EPS, S0=s0)
    y2, _ = layer.layer_fwd(q, k, v, bl, wl, al, gl, 3.0 * nw, EPS, S0=s0)
    np.testing.assert_allclose(y2, 3.0 * y1, rtol=1e-12, atol=1e-15)


def test_decay_is_the_sigmoid_of_its_logit():
    """Pure decay (b = w = 0 through logits -inf): the state after T tokens is
    prod_t sigmoid(decay_logit_t) times S0 on each key row (closed form)."""
    q, k, v, bl, wl, al, gl, nw, s0 = _layer_inputs(seed=7)
    neg = np.full_like
    _, st = layer.layer_fwd(q, k, v, neg(bl, -800.0), neg(wl, -800.0), al, gl, nw, EPS, S0=s0)
    decay = np.prod(1.0 / (1.0 + np.exp(-al)), axis=1)  # [B, H, dk]
    np.testing.assert_allclose(st, decay[..., None] * s0, rtol=1e-12)


def test_log_sigmoid_has_no_overflow():
    x = np.array([-1000.0, -30.0, 0.0, 30.0, 1000.0])
    ls = layer.log_sigmoid(x)
    assert np.all(np.isfinite(ls))
    np.testing.assert_allclose(ls[2], np.log(0.5))
    np.testing.assert_allclose(ls[0], -1000.0)
    assert ls[4] == 0.0 or abs(ls[4]) < 1e-300


def test_zero_alpha_forgets_everything_before():
    """log_alpha = -inf at token t (alpha = 0): the state after t is k_t (w_t v_t)^T,
    whatever came before (the decay empties the state, so the erase reads 0)."""
    q, k, v, b, w, la, s0 = _inputs(6, 5, 4, seed=8)
    la = la.copy()
    la[:, 3] = -np.inf
    _, st = oracle.fwd(q[:, :4], k[:, :4], v[:, :4], b[:, :4], w[:, :4], la[:, :4], S0=s0)
    expect = np.einsum("bhi,bhj->bhij", k[:, 3], w[:, 3] * v[:, 3])
    np.testing.assert_allclose(st, expect, rtol=1e-12, atol=1e-15)
