"""gdn2_decode_step on the GPU against the fp64 oracle (called through the C ABI)."""
import numpy as np
import pytest
import torch

import oracle
import synth
import gated_delta_rule_118_b200 as g
from parity import TOL_BF16, TOL_F32, rel_err, to_dev

pytestmark = pytest.mark.gpu
NAMES = ("q", "k", "v", "b", "w", "log_alpha")


@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 64), (128, 64), (64, 128)])
def test_one_step_every_element(dk, dv):
    case = synth.DecodeCase("t", 256 if dk == dv == 128 else 8, 16, dk, dv, steps=1)
    S = synth.draw_decode_state(case)
    x = synth.draw_decode_token(case, 0)
    o_ref, s_ref = oracle.decode_step(*(x[n] for n in NAMES), S)
    Sd = S.cuda()
    o = g.gdn2_decode_step(*(x[n].cuda() for n in NAMES), Sd)
    assert rel_err(o, o_ref) <= TOL_F32
    assert rel_err(Sd, s_ref) <= TOL_F32


def test_thousand_steps_every_state():
    """B=256, H=16, d=128, fp32 state in HBM updated in place for 1000 steps.
    The oracle follows all 4096 states (100 steps per call: n decode steps are
    one recurrence over n tokens); every output of every 100th step and every
    state element at the end are compared."""
    case = synth.DECODE_F32
    S = synth.draw_decode_state(case)
    S_ref = S.double().numpy()
    Sd = S.cuda()
    seg = 100
    for s0 in range(0, case.steps, seg):
        xs = {n: [] for n in NAMES}
        o_last = None
        for step in range(s0, s0 + seg):
            x = synth.draw_decode_token(case, step)
            o_last = g.gdn2_decode_step(*(x[n].cuda() for n in NAMES), Sd)
            for n in NAMES:
                xs[n].append(x[n])
        o_ref, S_ref = oracle.fwd(*(torch.stack(xs[n], 1) for n in NAMES), S0=S_ref)
        assert rel_err(o_last, o_ref[:, -1]) <= TOL_F32, s0 + seg
    assert rel_err(Sd, S_ref) <= TOL_F32
    assert g.gdn2_check_device_error() == g.GDN2_OK


def test_bf16_inputs():
    case = synth.DecodeCase("t", 64, 16, 128, 128, steps=1, dtype=torch.bfloat16)
    S = synth.draw_decode_state(case)
    x = synth.draw_decode_token(case, 3)
    o_ref, s_ref = oracle.decode_step(*(x[n] for n in NAMES), S)
    Sd = S.cuda()
    o = g.gdn2_decode_step(*(x[n].cuda() for n in NAMES), Sd)
    assert o.dtype == torch.bfloat16
    assert rel_err(o, o_ref) <= TOL_BF16 and rel_err(Sd, s_ref) <= TOL_BF16


@pytest.mark.parametrize("n", [1, 64, 100])
def test_decode_steps_equal_chunked_forward(n):
    """n decode steps from S0 == one chunked forward over T = n from S0."""
    d = synth.draw_fwd(2, n, 4, 128, 128, seed=50 + n, dtype=torch.float32, s0_sigma=0.05)
    dd = to_dev(d)
    o_f, s_f = g.gdn2_fwd_chunked(*(dd[n_] for n_ in NAMES), S0=dd["S0"])
    S = dd["S0"].clone()
    outs = [g.gdn2_decode_step(*(dd[n_][:, t].contiguous() for n_ in NAMES), S) for t in range(n)]
    o_d = torch.stack(outs, 1)
    assert rel_err(o_d, o_f.double().cpu().numpy()) <= TOL_F32
    assert rel_err(S, s_f.double().cpu().numpy()) <= TOL_F32
