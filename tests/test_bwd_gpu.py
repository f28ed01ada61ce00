"""gdn2_bwd_chunked on the GPU against the fp64 oracle's backpropagation
through the token recurrence (gdn2_oracle_bwd), every gradient, element by
element.  bf16 inputs with dk = 128 run on the tensor cores (bf16 operands,
fp32 accumulation and state) and are held to the bf16 tolerance; fp32 inputs,
and dk = 64, run in fp32 on the CUDA cores and are held to the fp32 one."""
import pytest
import torch

import oracle
import synth
import gated_delta_rule_118_b200 as g
from parity import TOL_BF16, TOL_F32, rel_err, to_dev

pytestmark = pytest.mark.gpu
NAMES = ("q", "k", "v", "b", "w", "log_alpha")
GRADS = ("dq", "dk", "dv", "db", "dw", "dlog_alpha", "dS0")


def case(B, T, H, dk, dv, dtype, seed, s0=0.05, with_dst=True, kind=None):
    d = synth.draw_fwd(B, T, H, dk, dv, seed=seed, dtype=dtype, s0_sigma=s0)
    if kind:
        d["log_alpha"] = synth.draw_log_alpha(B, T, H, dk, kind, seed=seed + 1)
    gen = torch.Generator().manual_seed(seed + 2)
    d["dO"] = torch.randn(B, T, H, dv, generator=gen).to(dtype)
    d["dS_T"] = torch.randn(B, H, dk, dv, generator=gen) if with_dst else None
    return d


def tolerance(d):
    return TOL_BF16 if d["q"].dtype == torch.bfloat16 and d["q"].shape[-1] == 128 else TOL_F32


def check(d, tol=None):
    tol = tolerance(d) if tol is None else tol
    dd = to_dev(d)
    got = g.gdn2_bwd_chunked(*(dd[n] for n in NAMES), dd["S0"], dd["dO"], dd["dS_T"])
    ref = oracle.bwd(*(d[n] for n in NAMES), d["S0"], d["dO"], d["dS_T"])
    errs = {n: rel_err(got[n], ref[n]) for n in GRADS}
    assert all(e <= tol for e in errs.values()), ", ".join(f"{n} {e:.3g}" for n, e in errs.items())
    return errs


SMALL = [
    # B, T, H, dk, dv, dtype
    (1, 1, 2, 64, 64, torch.float32),
    (2, 63, 3, 64, 64, torch.float32),
    (1, 64, 2, 128, 128, torch.float32),
    (1, 65, 2, 128, 64, torch.float32),
    (2, 130, 2, 64, 128, torch.float32),
    (1, 300, 2, 128, 128, torch.bfloat16),
    (2, 77, 3, 128, 128, torch.bfloat16),
    (1, 200, 2, 64, 64, torch.bfloat16),
]


@pytest.mark.parametrize("B,T,H,dk,dv,dtype", SMALL,
                         ids=[f"B{c[0]}T{c[1]}H{c[2]}k{c[3]}v{c[4]}{str(c[5])[6:]}" for c in SMALL])
def test_small_shapes_every_gradient(B, T, H, dk, dv, dtype):
    check(case(B, T, H, dk, dv, dtype, seed=900 + T))


def test_zero_initial_state_and_no_final_gradient():
    check(case(1, 150, 2, 128, 128, torch.bfloat16, seed=950, s0=0.0, with_dst=False))


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
@pytest.mark.parametrize("kind", synth.DECAY_KINDS)
def test_strong_decay_every_gradient(kind, dtype):
    """Chunks in the bounded form (running products of alpha) and, for bf16,
    the tensor-core backward's walks of the pairwise decays."""
    check(case(1, 200, 2, 128, 128, dtype, seed=960, kind=kind))


@pytest.mark.parametrize("dv", [64, 128])
def test_strong_decay_tensor_core_value_widths(dv):
    check(case(2, 130, 2, 128, dv, torch.bfloat16, seed=965, kind=synth.DECAY_KINDS[-1]))


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
def test_erase_gate_up_to_2(dtype):
    d = case(1, 150, 2, 128, 128, dtype, seed=970)
    d["b"] = (2.0 * d["b"].float()).to(dtype)
    check(d)


@pytest.mark.parametrize("T", [64, 65, 127, 640])
def test_tensor_core_chunk_edges(T):
    """Whole and ragged last chunks, one chunk and many, dv = 64 and 128."""
    check(case(1, T, 3, 128, 64 if T % 2 else 128, torch.bfloat16, seed=975 + T))


def test_oracle_sized_fp32_workload():
    c = synth.ORACLE_FP32
    d = synth.draw_case(c)
    gen = torch.Generator().manual_seed(980)
    d["dO"] = torch.randn(c.B, c.T, c.H, c.dv, generator=gen)
    d["dS_T"] = torch.randn(c.B, c.H, c.dk, c.dv, generator=gen)
    check(d)


@pytest.mark.parametrize("wl", [synth.LAYER_BF16, synth.TRAIN_BF16, synth.LONG_BF16], ids=lambda c: c.name)
def test_full_size_every_gradient(wl):
    """The layer, the training batch and the long context at full size (gradients of the
    bf16 forward's inputs)."""
    d = synth.draw_case(wl)
    gen = torch.Generator().manual_seed(990)
    d["dO"] = torch.randn(wl.B, wl.T, wl.H, wl.dv, generator=gen).to(wl.dtype)
    d["dS_T"] = torch.randn(wl.B, wl.H, wl.dk, wl.dv, generator=gen)
    check(d)


def test_zero_length_sequence():
    d = case(1, 0, 2, 64, 64, torch.float32, seed=995)
    dd = to_dev(d)
    got = g.gdn2_bwd_chunked(*(dd[n] for n in NAMES), dd["S0"], dd["dO"], dd["dS_T"])
    torch.cuda.synchronize()
    assert torch.equal(got["dS0"], dd["dS_T"])
