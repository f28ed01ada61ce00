"""The chunkwise backward's algebra (fp64 model of what the tensor-core backward
computes) equals the oracle's gradients, and the bf16-pair products for chunks
with T far from the identity remove the share of the error that the rounding
of T and X contributes (CPU)."""
import numpy as np
import pytest
import torch

import oracle
import synth
from oracle_pins import _inputs
from wy_bwd_model import wy_backward

GRADS = ("dq", "dk", "dv", "db", "dw", "dlog_alpha", "dS0")


def rel(got, ref):
    ref = np.asarray(ref)
    return float(np.abs(got - ref).max() / np.abs(ref).max())


def grads_case(T, dk, dv, seed, *, B=1, H=2, wide=False):
    q, k, v, b, w, la, s0 = _inputs(T, dk, dv, seed=seed, B=B, H=H)
    if wide:  # the long context's decay range and erase gates up to 2
        la = -np.exp(np.random.default_rng(seed).uniform(-9.0, 3.0, q.shape))
        b = 2 * b
    r = np.random.default_rng(seed + 1)
    return (q, k, v, b, w, la, s0), r.standard_normal(v.shape), r.standard_normal(s0.shape)


@pytest.mark.parametrize("regrouped", [True, False], ids=["regrouped", "plain"])
@pytest.mark.parametrize("C,T,wide", [(16, 150, False), (64, 200, False), (64, 64, True), (64, 200, True)])
def test_chunk_backward_matches_oracle(C, T, wide, regrouped):
    """Chunks of 16 and 64 with a ragged last chunk; decays down to -e^3 per token
    (a chunk's decay far beyond what a midpoint split holds) and erase gates in
    [0, 2]; dlog_alpha both regrouped (the kernel's form) and plain."""
    x, dO, dST = grads_case(T, 8, 6, seed=40 + T + C + wide, wide=wide)
    ref = oracle.bwd(*x, dO, dST)
    got = wy_backward(*x, dO, dST, C=C, regrouped=regrouped)
    errs = {n: rel(got[n], ref[n]) for n in GRADS}
    assert all(e <= 1e-11 for e in errs.values()), errs


def test_chunk_backward_without_initial_state_or_final_gradient():
    x, dO, _ = grads_case(100, 8, 8, seed=77)
    x = x[:-1] + (None,)
    ref = oracle.bwd(*x, dO, None)
    got = wy_backward(*x, dO, None, C=64)
    assert all(rel(got[n], ref[n]) <= 1e-11 for n in GRADS if n != "dS0")
    assert rel(got["dS0"], ref["dS0"]) <= 1e-11


def _bf16(x):
    return torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.bfloat16).double().numpy()


def _collinear_case(eps):
    d = synth.draw_fwd(1, 200, 2, 128, 128, seed=8300, dtype=torch.bfloat16, s0_sigma=0.05)
    if eps is not None:
        d = synth.collinear_keys(d, eps=eps, seed=8301)
    gen = torch.Generator().manual_seed(8301)
    dO = torch.randn(1, 200, 2, 128, generator=gen).to(torch.bfloat16).double().numpy()
    dST = torch.randn(1, 2, 128, 128, generator=gen).double().numpy()
    x = [d[n].double().numpy() for n in ("q", "k", "v", "b", "w", "log_alpha")] + [d["S0"].double().numpy()]
    return x, dO, dST


def test_pairs_remove_the_T_and_X_share_of_the_error():
    """Near-collinear keys (noise 0.02) and erase gates near 2: with bf16 T, X and
    gU in U = T X and dX = T^T gU (and everything else exact), dq's error is about
    6.6e-3; with T and X as bf16 pairs it falls to about 1.4e-5.  dv and dw keep
    the share of gU's rounding, which the pairs do not cover (about 9e-3)."""
    x, dO, dST = _collinear_case(0.02)
    ref = oracle.bwd(*x, dO, dST)
    plain = wy_backward(*x, dO, dST, rounding=_bf16, pairs=False)
    pairs = wy_backward(*x, dO, dST, rounding=_bf16, pairs=True)
    assert rel(plain["dq"], ref["dq"]) > 3e-3
    assert rel(pairs["dq"], ref["dq"]) < 1e-4
    for n in ("dk", "dlog_alpha", "dS0"):
        assert rel(pairs[n], ref[n]) < 0.5 * rel(plain[n], ref[n]), n
    assert rel(pairs["dv"], ref["dv"]) > 3e-3


def test_random_keys_need_no_pairs():
    """Random keys: bf16 T, X and gU alone stay far below the bf16 bar of 2e-2."""
    x, dO, dST = _collinear_case(None)
    ref = oracle.bwd(*x, dO, dST)
    plain = wy_backward(*x, dO, dST, rounding=_bf16, pairs=False)
    assert max(rel(plain[n], ref[n]) for n in GRADS) < 5e-3


@pytest.mark.parametrize("m,C,T", [(1, 64, 200), (2, 16, 150), (4, 16, 150), (3, 8, 100), (8, 4, 37)])
def test_grouped_adjoint_chain(m, C, T):
    """The adjoint chain stepping once per group of m composed chunk maps gives
    the oracle's dS0, and the gradient leaving every chunk (what each chunk's
    gradients take): the oracle's dS0 of the sequence's remainder after that
    chunk, started from the state the oracle reaches there."""
    from wy_model import group_adjoint
    x, dO, dST = grads_case(T, 8, 6, seed=500 + m * C)
    q, k, v, b, w, la, s0 = x
    ref = oracle.bwd(*x, dO, dST)
    dS0, dS_out = group_adjoint(q, k, v, b, w, la, dO, dST, C=C, m=m)
    assert rel(dS0, ref["dS0"]) <= 1e-11
    for i, t1 in enumerate(range(C, T, C)):
        _, s_mid = oracle.fwd(*(a[:, :t1] for a in (q, k, v, b, w, la)), S0=s0)
        tail = oracle.bwd(*(a[:, t1:] for a in (q, k, v, b, w, la)), np.asarray(s_mid), dO[:, t1:], dST)
        assert rel(dS_out[:, :, i], tail["dS0"]) <= 1e-11, i
    assert np.array_equal(dS_out[:, :, -1], dST)


def _f32(x):
    return np.asarray(x, dtype=np.float32).astype(np.float64)


FULL = dict(rounding=_bf16, gram=_bf16, operands=_bf16, images=(_bf16, _f32))


def test_midpoint_route_of_the_gradient_products_is_exact():
    x, dO, dST = _collinear_case(None)
    ref = oracle.bwd(*x, dO, dST)
    got = wy_backward(*x, dO, dST, operands=lambda a: a)
    assert max(rel(got[n], ref[n]) for n in GRADS) <= 1e-12


def test_emulated_bf16_backward_random_keys():
    """Every bf16 rounding point of the tensor-core backward emulated (the two
    chains' records and images, the prep's Gram, T, X, gU, and the gradient
    products' operands): within half the bf16 bar on random keys (about 6e-3 at
    most, db)."""
    x, dO, dST = _collinear_case(None)
    ref = oracle.bwd(*x, dO, dST)
    got = wy_backward(*x, dO, dST, pairs=True, **FULL)
    errs = {n: rel(got[n], ref[n]) for n in GRADS}
    assert max(errs.values()) <= 1e-2, errs


def test_emulated_bf16_backward_needs_the_pairs_on_collinear_keys():
    """Key noise 0.02, erase gates near 2: with T and X as pairs every gradient
    meets the bf16 bar (dq about 1.3e-2); without them dq reaches it (about
    2.1e-2).  The rest of dq's error is spread over the gradient products'
    operands (U and dX, the decayed factors, dP and dA: about 8e-3 each alone)."""
    x, dO, dST = _collinear_case(0.02)
    ref = oracle.bwd(*x, dO, dST)
    with_pairs = wy_backward(*x, dO, dST, pairs=True, **FULL)
    errs = {n: rel(with_pairs[n], ref[n]) for n in GRADS}
    assert max(errs.values()) <= 2e-2, errs
    without = wy_backward(*x, dO, dST, pairs=False, **FULL)
    assert rel(without["dq"], ref["dq"]) >= 1.8e-2


def _tf32(x):
    """Round to the tf32 format (10 explicit mantissa bits), to nearest even."""
    a = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    bits = a.view(np.uint32).astype(np.uint64)
    bits = (bits + 0x0FFF + ((bits >> 13) & 1)) & ~np.uint64(0x1FFF)
    return bits.astype(np.uint32).view(np.float32).astype(np.float64)


def test_tf32_rounding_helper():
    # 1 + 2^-10 is a tf32 number; 1 + 2^-11 (a tie) rounds to even (1); 1 + 3 * 2^-11 rounds up to 1 + 2^-9
    xs = np.array([1 + 2.0 ** -10, 1 + 2.0 ** -11, 1 + 3 * 2.0 ** -11, -3.0])
    assert np.array_equal(_tf32(xs), [1 + 2.0 ** -10, 1.0, 1 + 2.0 ** -9, -3.0])


def test_tf32_second_pass_would_reach_random_key_accuracy():
    """A flagged chunk's gradient products in tf32 instead of bf16 (the prep's Gram,
    the chains and the images staying bf16): every gradient within 5e-3 at key
    noise 0.02, against 1.3e-2 for dq with the bf16 pairs."""
    x, dO, dST = _collinear_case(0.02)
    ref = oracle.bwd(*x, dO, dST)
    got = wy_backward(*x, dO, dST, rounding=_tf32, gram=_bf16, operands=_tf32, images=(_bf16, _f32))
    errs = {n: rel(got[n], ref[n]) for n in GRADS}
    assert max(errs.values()) <= 5e-3, errs
