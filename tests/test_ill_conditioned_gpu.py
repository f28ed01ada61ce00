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


@pytest.mark.parametrize("dtype,eps", [(torch.bfloat16, 0.1), (torch.float32, 0.02)], ids=["bf16", "f32"])
def test_backward_near_singular_chunks(dtype, eps):
    """bf16 at key noise 0.1; fp32 at 0.02.  At 0.02 (cosines >= 0.93 within a
    chunk, erase gates in [1.95, 2)) the bf16 gradient of q comes to about 2e-2:
    the alternating sums of near-reflections amplify the bf16 rounding of the
    operands X and T of U = T X."""
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
