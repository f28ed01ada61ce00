"""The tensor-core path's roundings, emulated in the fp64 chunk model (CPU).

The bf16 forward keeps the state and the decays in fp32 and rounds to bf16
only the tensor-core operands: each chunk's record (NG, QS, Y, PT, Z) and the
state image Sx = bf16(S) that enters the chunk's products; outputs are bf16.
This test applies exactly those roundings to the fp64 WY model and checks the
result against the token recurrence with the bf16 tolerance (max abs error
over the tensor / max abs reference <= 2e-2), on the layer distribution and
on the long-context one (strong and near-1 decays, gates near 0 and 1).  It
checks the precision design, not the kernels' arithmetic order."""
import numpy as np
import pytest
import torch

import oracle
import synth
from wy_model import chunk_record

TOL_BF16 = 2e-2


def _bf16(x):
    return torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.bfloat16).double().numpy()


def _f32(x):
    return np.asarray(x, dtype=np.float32).astype(np.float64)


def _emulated_forward(d, C=64):
    q, k, v, b, w, la = (d[n][0, :, 0].double().numpy() for n in ("q", "k", "v", "b", "w", "log_alpha"))
    T, dv = v.shape
    S = np.zeros((q.shape[1], dv))
    o = np.zeros((T, dv))
    for t0 in range(0, T, C):
        sl = slice(t0, min(T, t0 + C))
        gc, NG, QS, Y, PT = chunk_record(q[sl], k[sl], b[sl], la[sl], C)
        NG, QS, Y, PT, Z = (_bf16(x) for x in (NG, QS, Y, PT, w[sl] * v[sl]))
        Sx = _bf16(S)
        o[sl] = _bf16(QS @ Sx + PT @ Z)
        S = _f32(_f32(gc)[:, None] * S + NG @ Sx + Y @ Z)
    return o, S


@pytest.mark.parametrize("case,T", [(synth.LAYER_BF16, 4096), (synth.LONG_BF16, 8192)],
                         ids=["layer", "long_context"])
def test_bf16_roundings_meet_the_tolerance(case, T):
    d = synth.draw_fwd(1, T, 1, 128, 128, seed=9, dtype=torch.bfloat16, s0_sigma=0.0,
                       log_alpha_range=case.log_alpha_range, gate_sigma=case.gate_sigma)
    o_ref, s_ref = oracle.fwd(*(d[n] for n in ("q", "k", "v", "b", "w", "log_alpha")), S0=None)
    o_ref, s_ref = np.asarray(o_ref)[0, :, 0], np.asarray(s_ref)[0, 0]
    o, S = _emulated_forward(d)
    eo = np.abs(o - o_ref).max() / np.abs(o_ref).max()
    es = np.abs(S - s_ref).max() / np.abs(s_ref).max()
    assert eo <= TOL_BF16 and es <= TOL_BF16, (eo, es)
    # the roundings cost a few parts in a thousand, well inside the tolerance
    assert eo <= TOL_BF16 / 2 and es <= TOL_BF16 / 2, (eo, es)


@pytest.mark.parametrize("case,T", [(synth.LAYER_BF16, 4096), (synth.LONG_BF16, 8192)],
                         ids=["layer", "long_context"])
def test_grouped_chain_costs_no_accuracy(case, T):
    """A chain stepping once per group of m chunks, with the group's composed map
    and input term (worker-side, bf16 operands, fp32 accumulators; the input term
    read as bf16 too), against the chain over single chunks: the state's error
    stays within 1e-3 of it for m = 4 and 8, and every error under half the
    bf16 tolerance.  (Measured: the outputs' error is unchanged, 4.3e-3 on the
    layer and 6.9e-3 on the long context; the state's 3.1e-3 becomes 3.9e-3 and
    3.3e-3.)"""
    from wy_model import group_forward
    d = synth.draw_fwd(1, T, 1, 128, 128, seed=9, dtype=torch.bfloat16, s0_sigma=0.0,
                       log_alpha_range=case.log_alpha_range, gate_sigma=case.gate_sigma)
    ins = [d[n] for n in ("q", "k", "v", "b", "w", "log_alpha")]
    o_ref, s_ref = oracle.fwd(*ins, S0=None)
    o_ref, s_ref = np.asarray(o_ref), np.asarray(s_ref)
    errs = {}
    for m in (1, 4, 8):
        o, S = group_forward(*(x.double().numpy() for x in ins), m=m, rounding=_bf16, store=_f32, n_rounded=m > 1)
        errs[m] = (np.abs(o - o_ref).max() / np.abs(o_ref).max(), np.abs(S - s_ref).max() / np.abs(s_ref).max())
    for m in (4, 8):
        assert abs(errs[m][1] - errs[1][1]) <= 1e-3, errs
        assert abs(errs[m][0] - errs[1][0]) <= 1e-3, errs
    assert max(max(e) for e in errs.values()) <= TOL_BF16 / 2, errs
