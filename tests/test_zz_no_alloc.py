"""gdn2_fwd_chunked_noalloc: the chunked forward for callers that cannot let a
library allocate device memory (a runtime that owns all device memory, a hot
loop that must not enter the allocator, a process that must know its device
footprint up front).  It runs out of one fixed scratch buffer that every call
reuses, so each case calls it twice in a row and compares both results with
the fp64 oracle, and with gdn2_fwd_chunked.

This file is collected last, so a run that stops at the first failure has run
every other test first.
"""
import pytest
import torch

import oracle
import synth
import gated_delta_rule_118_b200 as g
from parity import TOL_BF16, TOL_F32, rel_err, to_dev

pytestmark = pytest.mark.gpu
NAMES = ("q", "k", "v", "b", "w", "log_alpha")


def _two_calls_against_oracle(d, tol):
    o_ref, s_ref = oracle.fwd(*(d[n] for n in NAMES), S0=d["S0"])
    dd = to_dev(d)
    args = [dd[n] for n in NAMES]
    o_alloc, s_alloc = g.gdn2_fwd_chunked(*args, S0=dd["S0"])
    assert g.gdn2_check_device_error() == g.GDN2_OK
    o = torch.empty_like(o_alloc)
    st = torch.empty_like(s_alloc)
    for _ in range(2):  # the second call reuses the scratch the first one left behind
        o.fill_(float("nan"))
        st.fill_(float("nan"))
        g.gdn2_fwd_chunked_noalloc(*args, S0=dd["S0"], o=o, S_T=st)
        assert g.gdn2_check_device_error() == g.GDN2_OK
        assert rel_err(o, o_ref) <= tol and rel_err(st, s_ref) <= tol
        # both entry points run the same kernels; their results agree far more closely
        assert rel_err(o, o_alloc.double().cpu().numpy()) <= tol / 4
        assert rel_err(st, s_alloc.double().cpu().numpy()) <= tol / 4


def test_noalloc_bf16_several_windows():
    # B*H = 32 pairs: the 32 MiB scratch holds a few chunks per window, so a
    # 1000-token sequence needs several windows and carries the state between them.
    d = synth.draw_fwd(2, 1000, 16, 128, 128, seed=31, dtype=torch.bfloat16, s0_sigma=0.02)
    _two_calls_against_oracle(d, TOL_BF16)


def test_noalloc_bf16_largest_accepted_problem():
    # B*H = 177 pairs at dv = 128, the most the scratch takes: one chunk per
    # window, the carried state filling about a third of the buffer.
    d = synth.draw_fwd(3, 150, 59, 128, 128, seed=33, dtype=torch.bfloat16, s0_sigma=0.02)
    _two_calls_against_oracle(d, TOL_BF16)


def test_noalloc_fp32():
    d = synth.draw_fwd(1, 200, 2, 64, 64, seed=32, dtype=torch.float32, s0_sigma=0.1)
    _two_calls_against_oracle(d, TOL_F32)


def test_noalloc_rejects_problems_beyond_its_scratch():
    # 12 x 16 = 192 (batch, head) pairs do not fit one chunk of records in 32 MiB.
    B, H = 12, 16
    q = torch.zeros(B, 64, H, 128, dtype=torch.bfloat16, device="cuda")
    la = torch.zeros(B, 64, H, 128, dtype=torch.float32, device="cuda")
    o = torch.empty_like(q)
    with pytest.raises(g.Gdn2Error) as exc:
        g.gdn2_fwd_chunked_noalloc(q, q, q, q, q, la, o=o)
    assert exc.value.status == g.GDN2_ERR_SCRATCH_LIMIT
