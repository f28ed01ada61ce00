"""gdn2_fwd_chunked on the GPU against the fp64 oracle (called through the C ABI)."""
import numpy as np
import pytest
import torch

import oracle
import synth
import gated_delta_rule_118_b200 as g
from parity import TOL_BF16, TOL_F32, rel_err, to_dev

pytestmark = pytest.mark.gpu


def run_gpu(d, **kw):
    dd = to_dev(d)
    o, st = g.gdn2_fwd_chunked(dd["q"], dd["k"], dd["v"], dd["b"], dd["w"], dd["log_alpha"],
                               S0=dd["S0"], **kw)
    assert g.gdn2_check_device_error() == g.GDN2_OK
    return o, st


def oracle_ref(d, pairs=None):
    """Oracle on all (b, h) pairs, or on the listed ones (returned in that order)."""
    names = ("q", "k", "v", "b", "w", "log_alpha")
    if pairs is None:
        return oracle.fwd(*(d[n] for n in names), S0=d["S0"])
    outs = []
    for bi, h in pairs:
        sl = (slice(bi, bi + 1), slice(None), slice(h, h + 1))
        s0 = None if d["S0"] is None else d["S0"][bi:bi + 1, h:h + 1]
        outs.append(oracle.fwd(*(d[n][sl] for n in names), S0=s0))
    return outs


def tol(dtype):
    return TOL_F32 if dtype == torch.float32 else TOL_BF16


def test_oracle_sized_fp32_case_full():
    """B=1, H=2, T=256, dk=dv=64, fp32: every element against the oracle at 1e-4."""
    d = synth.draw_case(synth.ORACLE_FP32)
    o, st = run_gpu(d)
    o_ref, s_ref = oracle_ref(d)
    assert rel_err(o, o_ref) <= TOL_F32
    assert rel_err(st, s_ref) <= TOL_F32


SMALL = [
    # B, T, H, dk, dv, dtype, s0_sigma
    (1, 1, 1, 64, 64, torch.float32, 0.3),
    (2, 63, 3, 64, 64, torch.float32, 0.0),
    (1, 64, 2, 128, 128, torch.float32, 0.1),
    (1, 65, 2, 128, 64, torch.float32, 0.1),
    (2, 130, 2, 64, 128, torch.float32, 0.0),
    (1, 1, 2, 128, 128, torch.bfloat16, 0.1),
    (2, 63, 3, 128, 128, torch.bfloat16, 0.0),
    (1, 64, 2, 128, 128, torch.bfloat16, 0.05),
    (2, 200, 3, 128, 128, torch.bfloat16, 0.02),
    (1, 333, 2, 64, 64, torch.bfloat16, 0.02),
    (1, 129, 2, 128, 64, torch.bfloat16, 0.0),
    (1, 257, 2, 64, 128, torch.bfloat16, 0.02),
]


@pytest.mark.parametrize("B,T,H,dk,dv,dtype,s0", SMALL,
                         ids=[f"B{c[0]}T{c[1]}H{c[2]}k{c[3]}v{c[4]}{str(c[5])[6:]}" for c in SMALL])
def test_small_shapes_elementwise(B, T, H, dk, dv, dtype, s0):
    d = synth.draw_fwd(B, T, H, dk, dv, seed=1000 + T, dtype=dtype, s0_sigma=s0)
    o, st = run_gpu(d)
    o_ref, s_ref = oracle_ref(d)
    assert rel_err(o, o_ref) <= tol(dtype)
    assert rel_err(st, s_ref) <= tol(dtype)


FULL = [synth.LAYER_BF16, synth.TRAIN_BF16, synth.LONG_BF16]


@pytest.mark.parametrize("case", FULL, ids=[c.name for c in FULL])
def test_full_size_every_element(case):
    """The three bf16 workloads at full size, in the launch configuration the
    benchmark times: every output and every final-state element against the
    oracle (which runs all (batch, head) pairs on the host's cores)."""
    d = synth.draw_case(case)
    o, st = run_gpu(d)
    o_ref, s_ref = oracle_ref(d)
    eo, es = rel_err(o, o_ref), rel_err(st, s_ref)
    assert eo <= TOL_BF16 and es <= TOL_BF16, (case.name, eo, es)


# The bf16 forward has two schedules: one persistent launch whose chain CTAs
# (batch * heads * dv / 64) take at most a quarter of the SMs, with records in
# rings of 24 chunks per head, and windows otherwise (three launches beside the
# chain, two where prep and chain take turns).
SCHEDULES = [
    # B, T, H, dv, pairs checked, what it covers
    (1, 2600, 3, 128, None, "persistent, rings wrap, ragged tail"),
    (1, 1500, 2, 64, None, "persistent, dv = 64"),
    (1, 16500, 1, 128, None, "persistent, long sequence, ragged tail"),
    (2, 700, 12, 128, None, "windows beside the chain (24 heads x 2 tiles)"),
    (2, 700, 24, 64, None, "windows beside the chain (48 heads, dv = 64)"),
    (2, 300, 40, 64, None, "prep, then chains that compute the outputs (80 heads, dv = 64)"),
    (8, 4500, 16, 128, None, "prep, then chains that compute the outputs: two windows, the state carried"),
]


@pytest.mark.parametrize("B,T,H,dv,pairs,what", SCHEDULES, ids=[c[5] for c in SCHEDULES])
def test_schedules(B, T, H, dv, pairs, what):
    d = synth.draw_fwd(B, T, H, 128, dv, seed=31 + T, dtype=torch.bfloat16, s0_sigma=0.02)
    o, st = run_gpu(d)
    if pairs is None:
        o_ref, s_ref = oracle_ref(d)
        assert rel_err(o, o_ref) <= TOL_BF16 and rel_err(st, s_ref) <= TOL_BF16, what
        return
    for (bi, h), (o_ref, s_ref) in zip(pairs, oracle_ref(d, pairs)):
        eo = rel_err(o[bi:bi + 1, :, h:h + 1], o_ref)
        es = rel_err(st[bi:bi + 1, h:h + 1], s_ref)
        assert eo <= TOL_BF16 and es <= TOL_BF16, (what, bi, h, eo, es)


def test_state_in_place_and_optional_outputs():
    d = synth.draw_fwd(2, 150, 2, 128, 128, seed=7, dtype=torch.bfloat16, s0_sigma=0.05)
    o_ref, s_ref = oracle_ref(d)
    dd = to_dev(d)
    S = dd["S0"].clone()
    o, st = g.gdn2_fwd_chunked(dd["q"], dd["k"], dd["v"], dd["b"], dd["w"], dd["log_alpha"],
                               S0=S, S_T=S)
    assert st.data_ptr() == S.data_ptr()
    assert rel_err(S, s_ref) <= TOL_BF16 and rel_err(o, o_ref) <= TOL_BF16
    o2, st2 = g.gdn2_fwd_chunked(dd["q"], dd["k"], dd["v"], dd["b"], dd["w"], dd["log_alpha"],
                                 S0=dd["S0"], want_state=False)
    assert st2 is None and torch.equal(o2, o)


def test_zero_length_sequence_copies_state():
    d = synth.draw_fwd(1, 0, 2, 64, 64, seed=8, dtype=torch.float32, s0_sigma=0.1)
    dd = to_dev(d)
    o, st = g.gdn2_fwd_chunked(dd["q"], dd["k"], dd["v"], dd["b"], dd["w"], dd["log_alpha"],
                               S0=dd["S0"])
    torch.cuda.synchronize()
    assert o.numel() == 0 and torch.equal(st, dd["S0"])
    _, st0 = g.gdn2_fwd_chunked(dd["q"], dd["k"], dd["v"], dd["b"], dd["w"], dd["log_alpha"])
    torch.cuda.synchronize()
    assert torch.count_nonzero(st0) == 0


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_split_sequence_resumes_from_state(dtype):
    """fwd(0..T) == fwd(0..T1) then fwd(T1..T) from S_T1 (the state is the checkpoint)."""
    d = synth.draw_fwd(1, 300, 2, 128, 128, seed=9, dtype=dtype, s0_sigma=0.02)
    dd = to_dev(d)
    names = ("q", "k", "v", "b", "w", "log_alpha")
    o, st = g.gdn2_fwd_chunked(*(dd[n] for n in names), S0=dd["S0"])
    T1 = 100  # not a multiple of the chunk
    oa, sa = g.gdn2_fwd_chunked(*(dd[n][:, :T1].contiguous() for n in names), S0=dd["S0"])
    ob, sb = g.gdn2_fwd_chunked(*(dd[n][:, T1:].contiguous() for n in names), S0=sa)
    o_ref, s_ref = oracle_ref(d)
    assert rel_err(torch.cat([oa, ob], 1), o_ref) <= tol(dtype)
    assert rel_err(sb, s_ref) <= tol(dtype)
    assert rel_err(o, o_ref) <= tol(dtype)


def test_erase_gate_range_0_2_not_clamped():
    d = synth.draw_fwd(1, 200, 2, 128, 128, seed=10, dtype=torch.bfloat16)
    d["b"] = (2.0 * d["b"].float()).to(torch.bfloat16)
    o, st = run_gpu(d)
    o_ref, s_ref = oracle_ref(d)
    assert rel_err(o, o_ref) <= TOL_BF16 and rel_err(st, s_ref) <= TOL_BF16


def test_results_are_deterministic():
    d = to_dev(synth.draw_fwd(2, 300, 4, 128, 128, seed=11, dtype=torch.bfloat16, s0_sigma=0.02))
    names = ("q", "k", "v", "b", "w", "log_alpha")
    o1, s1 = g.gdn2_fwd_chunked(*(d[n] for n in names), S0=d["S0"])
    o2, s2 = g.gdn2_fwd_chunked(*(d[n] for n in names), S0=d["S0"])
    assert torch.equal(o1, o2) and torch.equal(s1, s2)


def test_bounded_wait_gives_up_and_reports():
    """A device wait on a flag nothing sets gives up after about a second and
    reports GDN2_ERR_DEVICE_TIMEOUT; the context stays usable (a forward after it
    runs and reports no error)."""
    import time
    assert g.gdn2_selftest_bounded_wait() == g.GDN2_OK
    t0 = time.perf_counter()
    assert g.gdn2_check_device_error() == g.GDN2_ERR_DEVICE_TIMEOUT
    assert 0.5 < time.perf_counter() - t0 < 10.0
    assert g.gdn2_check_device_error() == g.GDN2_OK  # the word was cleared
    d = synth.draw_fwd(1, 130, 2, 128, 128, seed=11, dtype=torch.bfloat16, s0_sigma=0.02)
    o, st = run_gpu(d)
    o_ref, s_ref = oracle_ref(d)
    assert rel_err(o, o_ref) <= TOL_BF16 and rel_err(st, s_ref) <= TOL_BF16
