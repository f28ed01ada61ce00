"""gdn2_fwd_chunked_noalloc: the chunked forward for callers that cannot let a
library allocate device memory (a runtime that owns all device memory, a hot
loop that must not enter the allocator, a process that must know its device
footprint up front).  Its output must match gdn2_fwd_chunked's, call after call,
although it runs out of one fixed scratch buffer that every call reuses.

This file is collected last, so a run that stops at the first failure has run
every other test first.
"""
import pytest
import torch

import synth
import gated_delta_rule_118_b200 as g
from parity import TOL_BF16, TOL_F32, rel_err, to_dev

pytestmark = pytest.mark.gpu
NAMES = ("q", "k", "v", "b", "w", "log_alpha")


def _compare_two_calls(d, tol):
    dd = to_dev(d)
    args = [dd[n] for n in NAMES]
    o_ref, s_ref = g.gdn2_fwd_chunked(*args, S0=dd["S0"])
    torch.cuda.synchronize()
    assert g.gdn2_check_device_error() == g.GDN2_OK
    o = torch.empty_like(o_ref)
    st = torch.empty_like(s_ref)
    for _ in range(2):  # the second call reuses the scratch the first one left behind
        o.fill_(float("nan"))
        st.fill_(float("nan"))
        g.gdn2_fwd_chunked_noalloc(*args, S0=dd["S0"], o=o, S_T=st)
        assert g.gdn2_check_device_error() == g.GDN2_OK
        assert rel_err(o, o_ref.double().cpu().numpy()) <= tol
        assert rel_err(st, s_ref.double().cpu().numpy()) <= tol


def test_noalloc_matches_allocating_entry_bf16_several_windows():
    # B*H = 32 pairs: the 32 MiB scratch holds a few chunks per window, so a
    # 1000-token sequence needs several windows and carries the state between them.
    d = synth.draw_fwd(2, 1000, 16, 128, 128, seed=31, dtype=torch.bfloat16, s0_sigma=0.02)
    _compare_two_calls(d, TOL_BF16)


def test_noalloc_matches_allocating_entry_fp32():
    d = synth.draw_fwd(1, 200, 2, 64, 64, seed=32, dtype=torch.float32, s0_sigma=0.1)
    _compare_two_calls(d, TOL_F32)


def test_noalloc_rejects_problems_beyond_its_scratch():
    # 12 x 16 = 192 (batch, head) pairs do not fit one chunk of records in 32 MiB.
    B, H = 12, 16
    q = torch.zeros(B, 64, H, 128, dtype=torch.bfloat16, device="cuda")
    la = torch.zeros(B, 64, H, 128, dtype=torch.float32, device="cuda")
    o = torch.empty_like(q)
    with pytest.raises(g.Gdn2Error) as exc:
        g.gdn2_fwd_chunked_noalloc(q, q, q, q, q, la, o=o)
    assert exc.value.status == g.GDN2_ERR_SCRATCH_LIMIT
