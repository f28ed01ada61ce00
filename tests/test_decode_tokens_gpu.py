"""gdn2_decode_tokens (T tokens on a resident state) against the fp64 oracle.

Recurrent decoding with a fixed-size state (gist.science, "Problem
Statement"); a short run of tokens on a cached state is the same recurrence
over T tokens, so the oracle's token loop is the reference, element by element.
"""
import pytest
import torch

import oracle
import synth
import gated_delta_rule_118_b200 as g
from parity import TOL_BF16, TOL_F32, rel_err, to_dev

pytestmark = pytest.mark.gpu
NAMES = ("q", "k", "v", "b", "w", "log_alpha")


def run(d, S0):
    dd = to_dev(d)
    S = S0.cuda()
    o = g.gdn2_decode_tokens(*(dd[n] for n in NAMES), S)
    torch.cuda.synchronize()
    return o, S


def expand(d):
    """Per-channel copies of [B,T,H] gates (the oracle takes per-channel gates)."""
    dk, dv = d["q"].shape[-1], d["v"].shape[-1]
    e = dict(d)
    for n, dd in (("b", dk), ("w", dv), ("log_alpha", dk)):
        if d[n].dim() == 3:
            e[n] = d[n][..., None].expand(*d[n].shape, dd).contiguous()
    return e


@pytest.mark.parametrize("T", [1, 2, 7, 8, 9, 16, 17, 63, 100])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
def test_tokens_every_element(T, dtype):
    d = synth.draw_fwd(4, T, 8, 128, 128, seed=600 + T, dtype=dtype, s0_sigma=0.05)
    o, S = run(d, d["S0"])
    o_ref, s_ref = oracle.fwd(*(d[n] for n in NAMES), S0=d["S0"])
    tol = TOL_F32 if dtype == torch.float32 else TOL_BF16
    assert rel_err(o, o_ref) <= tol and rel_err(S, s_ref) <= tol


@pytest.mark.parametrize("dk,dv", [(64, 64), (128, 64), (64, 128)])
def test_tokens_head_sizes(dk, dv):
    d = synth.draw_fwd(3, 12, 5, dk, dv, seed=610 + dk + dv, dtype=torch.float32, s0_sigma=0.05)
    o, S = run(d, d["S0"])
    o_ref, s_ref = oracle.fwd(*(d[n] for n in NAMES), S0=d["S0"])
    assert rel_err(o, o_ref) <= TOL_F32 and rel_err(S, s_ref) <= TOL_F32


@pytest.mark.parametrize("layout", [1, 2, 3, 4, 7])
def test_tokens_gate_layouts(layout):
    d = synth.draw_fwd(2, 20, 4, 128, 128, seed=620 + layout, dtype=torch.float32, s0_sigma=0.05)
    d = synth.scalar_gates(d, layout, seed=621 + layout)
    o, S = run(d, d["S0"])
    e = expand(d)
    o_ref, s_ref = oracle.fwd(*(e[n] for n in NAMES), S0=d["S0"])
    assert rel_err(o, o_ref) <= TOL_F32 and rel_err(S, s_ref) <= TOL_F32


def test_tokens_strong_decay_and_zero_alpha():
    d = synth.draw_fwd(2, 30, 4, 128, 128, seed=630, dtype=torch.float32, s0_sigma=0.05)
    d["log_alpha"] = synth.draw_log_alpha(2, 30, 4, 128, "zeros", seed=631)
    o, S = run(d, d["S0"])
    o_ref, s_ref = oracle.fwd(*(d[n] for n in NAMES), S0=d["S0"])
    assert rel_err(o, o_ref) <= TOL_F32 and rel_err(S, s_ref) <= TOL_F32


def test_tokens_equal_decode_steps_at_full_decode_size():
    """B=256, H=16, d=128: 8 tokens in one call == 8 decode steps (same kernels'
    arithmetic per token), and == the oracle."""
    case = synth.DECODE_F32
    S0 = synth.draw_decode_state(case)
    xs = [synth.draw_decode_token(case, s) for s in range(8)]
    d = {n: torch.stack([x[n] for x in xs], 1).contiguous() for n in NAMES}
    o, S = run(d, S0)
    S2 = S0.cuda()
    steps = [g.gdn2_decode_step(*(x[n].cuda() for n in NAMES), S2) for x in xs]
    o2 = torch.stack(steps, 1)
    assert rel_err(o, o2.double().cpu().numpy()) <= 1e-5
    assert rel_err(S, S2.double().cpu().numpy()) <= 1e-5
    o_ref, s_ref = oracle.fwd(*(d[n] for n in NAMES), S0=S0)
    assert rel_err(o, o_ref) <= TOL_F32 and rel_err(S, s_ref) <= TOL_F32
