"""Gate-variant fast paths of the chunked forward against the fp64 oracle.

The pages obtain Kimi Delta Attention (b = w = beta, a scalar per token) and
Gated DeltaNet (also a scalar decay) as special cases of the operator
(iplexlaw.co.kr, section "Decisiones independientes en dos ejes"; gist.science,
section 1), and ablate a channel-averaged erase or write gate and an erase gate
in [0, 2] (iplexlaw.co.kr, section "Ablaciones y velocidad de entrenamiento").
Each layout passes its gates as [B,T,H]; the oracle gets the same values
broadcast over the channels.
"""
import pytest
import torch

import oracle
import synth
import gated_delta_rule_118_b200 as g
from parity import TOL_BF16, TOL_F32, rel_err, to_dev

pytestmark = pytest.mark.gpu
NAMES = ("q", "k", "v", "b", "w", "log_alpha")
LAYOUTS = {"erase": 1, "write": 2, "kda": 3, "decay": 4, "gdn": 7, "erase+decay": 5}


def expand(d):
    dk, dv = d["q"].shape[-1], d["v"].shape[-1]
    e = dict(d)
    for n, dd in (("b", dk), ("w", dv), ("log_alpha", dk)):
        if d[n].dim() == 3:
            e[n] = d[n][..., None].expand(*d[n].shape, dd).contiguous()
    return e


def check(d, tol):
    dd = to_dev(d)
    o, st = g.gdn2_fwd_chunked(*(dd[n] for n in NAMES), S0=dd["S0"])
    assert g.gdn2_check_device_error() == g.GDN2_OK
    e = expand(d)
    o_ref, s_ref = oracle.fwd(*(e[n] for n in NAMES), S0=d["S0"])
    eo, es = rel_err(o, o_ref), rel_err(st, s_ref)
    assert eo <= tol and es <= tol, (eo, es)


@pytest.mark.parametrize("name", list(LAYOUTS))
@pytest.mark.parametrize("T", [1, 130, 1000])
def test_layouts_bf16_tensor_cores(name, T):
    d = synth.draw_fwd(1, T, 4, 128, 128, seed=700 + T, dtype=torch.bfloat16, s0_sigma=0.03)
    check(synth.scalar_gates(d, LAYOUTS[name], seed=701 + T), TOL_BF16)


@pytest.mark.parametrize("name", list(LAYOUTS))
def test_layouts_fp32(name):
    d = synth.draw_fwd(2, 200, 2, 64, 128, seed=710, dtype=torch.float32, s0_sigma=0.05)
    check(synth.scalar_gates(d, LAYOUTS[name], seed=711), TOL_F32)


@pytest.mark.parametrize("name", ["kda", "gdn"])
def test_layouts_on_every_schedule(name):
    """Persistent launch (layer-shaped), windowed kernels beside the chain and
    alternating with it (wide batches), dk = 64 on the fp32 pipes."""
    for B, T, H, dk, dv, dtype, tol in ((1, 2000, 16, 128, 128, torch.bfloat16, TOL_BF16),
                                        (2, 700, 12, 128, 128, torch.bfloat16, TOL_BF16),
                                        (8, 200, 16, 128, 128, torch.bfloat16, TOL_BF16),
                                        (1, 300, 3, 64, 64, torch.bfloat16, TOL_BF16)):
        d = synth.draw_fwd(B, T, H, dk, dv, seed=720 + B, dtype=dtype, s0_sigma=0.02)
        check(synth.scalar_gates(d, LAYOUTS[name], seed=721 + B), tol)


def test_scalar_decay_strong_and_erase_up_to_2():
    d = synth.draw_fwd(1, 500, 4, 128, 128, seed=730, dtype=torch.bfloat16, s0_sigma=0.03)
    d = synth.scalar_gates(d, 7, seed=731)
    d["b"] = (2.0 * d["b"].float()).to(torch.bfloat16)  # KDA beta scaled into [0, 2]
    d["w"] = d["b"]
    gen = torch.Generator().manual_seed(732)
    d["log_alpha"] = -torch.exp(torch.rand(1, 500, 4, generator=gen) * 4.0 - 1.0)  # down to about -20
    check(d, TOL_BF16)
