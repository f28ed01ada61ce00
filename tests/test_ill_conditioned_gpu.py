"""Chunks whose triangular system I + A is as ill-conditioned as the method
allows, against the fp64 oracle: near-collinear keys within each chunk and erase
gates near 2, so that every off-diagonal entry of A is close to 2 ("Gated
DeltaNet-2", iplexlaw.co.kr, section "Procesamiento del token y entrenamiento
paralelo": the per-chunk system (I + T)^{-1} of the WY form, which the pages
warn needs care in precision).  The forward in bf16 (tensor cores, the solve's
merges on tf32 warp MMAs) and fp32, and the backward in both.
"""
import pytest
import torch

import oracle
import synth
import gated_delta_rule_118_b200 as g
from parity import TOL_BF16, TOL_F32, rel_err, to_dev

pytestmark = pytest.mark.gpu
NAMES = ("q", "k", "v", "b", "w", "log_alpha")
GRADS = ("dq", "dk", "dv", "db", "dw", "dlog_alpha", "dS0")


def case(T, dtype, seed, eps):
    d = synth.draw_fwd(1, T, 2, 128, 128, seed=seed, dtype=dtype, s0_sigma=0.05)
    return synth.collinear_keys(d, eps=eps, seed=seed + 1)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32], ids=["bf16", "f32"])
@pytest.mark.parametrize("T", [200, 256])
@pytest.mark.parametrize("eps", [0.02, 0.2])
def test_forward_near_singular_chunks(T, dtype, eps):
    d = case(T, dtype, 8100 + T, eps)
    dd = to_dev(d)
    o, st = g.gdn2_fwd_chunked(*(dd[n] for n in NAMES), S0=dd["S0"])
    assert g.gdn2_check_device_error() == g.GDN2_OK
    o_ref, s_ref = oracle.fwd(*(d[n] for n in NAMES), S0=d["S0"])
    tol = TOL_F32 if dtype == torch.float32 else TOL_BF16
    eo, es = rel_err(o, o_ref), rel_err(st, s_ref)
    assert eo <= tol and es <= tol, (eo, es)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32], ids=["bf16", "f32"])
@pytest.mark.parametrize("eps", [0.02, 0.1, 0.3])
def test_backward_near_singular_chunks(dtype, eps):
    """Key noise 0.02 (cosines >= 0.93 within a chunk), 0.1 and 0.3, erase gates in
    [1.95, 2).  In bf16 a chunk whose T lies more than 0.5 off the identity is
    computed again with T and X as bf16 pairs in U = T X and dX = T^T gU: the
    alternating sums of near-reflections would otherwise amplify their rounding
    (about 2e-2 on dq at key noise 0.02).  Every chunk crosses that threshold at
    0.02 and 0.1; at 0.3 chunks lie on both sides of it."""
    d = case(200, dtype, 8300, eps)
    gen = torch.Generator().manual_seed(8301)
    d["dO"] = torch.randn(1, 200, 2, 128, generator=gen).to(dtype)
    d["dS_T"] = torch.randn(1, 2, 128, 128, generator=gen)
    dd = to_dev(d)
    got = g.gdn2_bwd_chunked(*(dd[n] for n in NAMES), dd["S0"], dd["dO"], dd["dS_T"])
    ref = oracle.bwd(*(d[n] for n in NAMES), d["S0"], d["dO"], d["dS_T"])
    tol = TOL_BF16 if dtype == torch.bfloat16 else TOL_F32
    errs = {n: rel_err(got[n], ref[n]) for n in GRADS}
    assert all(e <= tol for e in errs.values()), ", ".join(f"{n} {e:.3g}" for n, e in errs.items())


def test_backward_flagged_chunks_beyond_one_per_sm():
    """256 chunks (more than one per SM, so that the CTAs that recompute the
    flagged chunks take several each), near-collinear keys in the even chunks
    of every (batch, head) and random ones in the odd: the flagged chunks get
    the bf16 pairs, the others keep the plain path's gradients.  Sequences of
    four chunks: with erase gates near 2 the chunks are near-reflections, and
    over long sequences the bf16 records of the state chains (not the chunk
    gradients) would set the error."""
    B, T, H = 8, 256, 8
    d = synth.draw_fwd(B, T, H, 128, 128, seed=8400, dtype=torch.bfloat16, s0_sigma=0.05)
    ill = synth.collinear_keys(d, eps=0.02, seed=8401)
    even = ((torch.arange(T) // 64) % 2 == 0).view(1, T, 1, 1)
    for n in ("k", "b"):
        d[n] = torch.where(even, ill[n], d[n]).contiguous()
    gen = torch.Generator().manual_seed(8402)
    d["dO"] = torch.randn(B, T, H, 128, generator=gen).to(torch.bfloat16)
    d["dS_T"] = torch.randn(B, H, 128, 128, generator=gen)
    dd = to_dev(d)
    got = g.gdn2_bwd_chunked(*(dd[n] for n in NAMES), dd["S0"], dd["dO"], dd["dS_T"])
    assert g.gdn2_check_device_error() == g.GDN2_OK
    ref = oracle.bwd(*(d[n] for n in NAMES), d["S0"], d["dO"], d["dS_T"])
    errs = {n: rel_err(got[n], ref[n]) for n in GRADS}
    assert all(e <= TOL_BF16 for e in errs.values()), ", ".join(f"{n} {e:.3g}" for n, e in errs.items())
