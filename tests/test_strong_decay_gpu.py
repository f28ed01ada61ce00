"""The chunked forward where the decay is strong, against the fp64 oracle.

The method is defined for every alpha in (0, 1] (and alpha = 0 gives complete
forgetting): "Gated DeltaNet-2", iplexlaw.co.kr, section "Procesamiento del
token y entrenamiento paralelo", folds the per-channel decay into asymmetric
factors and warns that the decay must be cumulated in fp32.  Chunks whose
cumulative decay is too strong for the split factors around the chunk midpoint
take a bounded form in the kernels; these cases cover that form (and chunks of
both forms in one sequence), element by element, in bf16 and fp32.
"""
import pytest
import torch

import oracle
import synth
import gated_delta_rule_118_b200 as g
from parity import TOL_BF16, TOL_F32, rel_err, to_dev

pytestmark = pytest.mark.gpu

NAMES = ("q", "k", "v", "b", "w", "log_alpha")


def case(kind, T, dtype, seed, H=2, dk=128, dv=128):
    d = synth.draw_fwd(1, T, H, dk, dv, seed=seed, dtype=dtype, s0_sigma=0.05)
    d["log_alpha"] = synth.draw_log_alpha(1, T, H, dk, kind, seed=seed + 1)
    return d


def check(d, dtype):
    dd = to_dev(d)
    o, st = g.gdn2_fwd_chunked(*(dd[n] for n in NAMES), S0=dd["S0"])
    assert g.gdn2_check_device_error() == g.GDN2_OK
    o_ref, s_ref = oracle.fwd(*(d[n] for n in NAMES), S0=d["S0"])
    tol = TOL_F32 if dtype == torch.float32 else TOL_BF16
    eo, es = rel_err(o, o_ref), rel_err(st, s_ref)
    assert torch.isfinite(o).all() and torch.isfinite(st).all()
    assert eo <= tol and es <= tol, (eo, es)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32], ids=["bf16", "f32"])
@pytest.mark.parametrize("T", [64, 200, 4096])
@pytest.mark.parametrize("kind", synth.DECAY_KINDS)
def test_strong_decay_elementwise(kind, T, dtype):
    check(case(kind, T, dtype, seed=5000 + T), dtype)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32], ids=["bf16", "f32"])
def test_strong_and_weak_chunks_in_one_sequence(dtype):
    """Alternating 64-token stretches of strong (-3 per token) and workload decay,
    offset by 32 tokens so that chunks of both forms and mixed chunks occur."""
    d = case("all3", 700, dtype, seed=77)
    weak = synth.draw_fwd(1, 700, 2, 128, 128, seed=78)["log_alpha"]
    t = torch.arange(700).view(1, 700, 1, 1)
    d["log_alpha"] = torch.where(((t + 32) // 64) % 2 == 0, d["log_alpha"], weak).contiguous()
    check(d, dtype)


@pytest.mark.parametrize("dv", [64, 128])
def test_strong_decay_dk64_and_narrow_values(dv):
    for dtype in (torch.bfloat16, torch.float32):
        check(case("wide", 333, dtype, seed=91, dk=64, dv=dv), dtype)
        check(case("wide", 333, dtype, seed=92, dk=128, dv=dv), dtype)


def test_strong_decay_persistent_and_windowed_schedules():
    """Layer-shaped launch (persistent kernel) and a wide batch (windowed kernels)."""
    for B, H, T in ((1, 16, 1024), (2, 24, 300)):
        d = synth.draw_fwd(B, T, H, 128, 128, seed=93 + H, dtype=torch.bfloat16, s0_sigma=0.02)
        d["log_alpha"] = synth.draw_log_alpha(B, T, H, 128, "wide", seed=94 + H)
        check(d, torch.bfloat16)
