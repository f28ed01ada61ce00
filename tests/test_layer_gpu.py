"""gdn2_layer_fwd (the operator with the layer's input and output processing
fused into its kernels) against the fp64 layer oracle (oracle/layer.py)."""
import pytest
import torch

import synth
import gated_delta_rule_118_b200 as g
from oracle import layer
from parity import TOL_BF16, TOL_F32, rel_err, to_dev

pytestmark = pytest.mark.gpu
EPS = 1e-6
IN = ("q", "k", "v", "b_logit", "w_logit", "decay_logit", "g_logit", "norm_weight")


def check(d, tol):
    dd = to_dev(d)
    y, st = g.gdn2_layer_fwd(*(dd[n] for n in IN), EPS, S0=dd["S0"])
    assert g.gdn2_check_device_error() == g.GDN2_OK
    y_ref, s_ref = layer.layer_fwd(*(d[n] for n in IN), EPS, S0=d["S0"])
    ey, es = rel_err(y, y_ref), rel_err(st, s_ref)
    assert ey <= tol and es <= tol, (ey, es)


@pytest.mark.parametrize("T", [1, 63, 64, 65, 200, 1000])
def test_layer_bf16_tensor_cores(T):
    check(synth.draw_layer(1, T, 4, 128, 128, seed=800 + T, dtype=torch.bfloat16, s0_sigma=0.03), TOL_BF16)


@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 64), (128, 64), (64, 128)])
def test_layer_fp32(dk, dv):
    check(synth.draw_layer(2, 150, 3, dk, dv, seed=810 + dk + dv, dtype=torch.float32, s0_sigma=0.05), TOL_F32)


def test_layer_every_schedule():
    """Layer-shaped persistent launch, windowed kernels, dv = 64, and bf16 dk = 64."""
    for B, T, H, dk, dv in ((1, 4096, 16, 128, 128), (2, 700, 12, 128, 128), (1, 500, 4, 128, 64),
                            (1, 300, 3, 64, 128)):
        check(synth.draw_layer(B, T, H, dk, dv, seed=820 + H, dtype=torch.bfloat16, s0_sigma=0.02), TOL_BF16)


def test_layer_zero_output_gate_and_large_scales():
    """A strongly closed output gate gives (near-)zero outputs; raw q, k scaled far
    from unit norm give the same results (the fused L2 norm)."""
    d = synth.draw_layer(1, 300, 4, 128, 128, seed=830, dtype=torch.bfloat16, s0_sigma=0.02)
    d["q"] = (d["q"].float() * 40.0).to(torch.bfloat16)
    d["k"] = (d["k"].float() * 0.05).to(torch.bfloat16)
    check(d, TOL_BF16)
    d["g_logit"] = torch.full_like(d["g_logit"], -30.0)
    dd = to_dev(d)
    y, _ = g.gdn2_layer_fwd(*(dd[n] for n in IN), EPS, S0=dd["S0"])
    assert y.float().abs().max().item() < 1e-10
