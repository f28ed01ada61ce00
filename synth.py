"""Seeded synthetic inputs for the Gated DeltaNet-2 operator.

This module is shared by the tests, the benchmark and the smoke check, and by
both sides of every parity comparison (the CUDA library and the fp64 oracle).
It holds only the input recipe -- random draws and the pre-processing a layer
applies before the operator (L2-normalised q/k, SiLU values, sigmoid gates,
negative log-decay) -- and none of the operator's own arithmetic.

Recipe (all draws on a CPU ``torch.Generator`` seeded per case, in the order
q, k, v, b, w, log_alpha, S0):
  * q, k ~ N(0, 1) in fp32, L2-normalised over the head dimension per
    (batch, token, head), then cast to the input dtype;
  * v = SiLU(N(0, 1));
  * b (dk channels) and w (dv channels) = sigmoid(N(0, sigma_gate));
  * log_alpha = -exp(U(lo, hi)), fp32, one value per token and key channel;
  * S0 = 0, or N(0, sigma_s0) in fp32.
The shapes follow the layer described on the pages: 16 heads with a 128 x 128
state per head and a 4K training context ("Gated DeltaNet-2" on iplexlaw.co.kr,
section "Condiciones de comparación"), stand-ins for the FineWeb-Edu
activations of a trained 1.3B model, which are not available here.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class FwdCase:
    name: str
    B: int
    T: int
    H: int
    dk: int
    dv: int
    dtype: torch.dtype
    seed: int
    log_alpha_range: tuple = (-5.0, -1.0)
    gate_sigma: float = 1.0
    s0_sigma: float = 0.0  # 0 => zero initial state


@dataclass(frozen=True)
class DecodeCase:
    name: str
    B: int
    H: int
    dk: int
    dv: int
    steps: int
    dtype: torch.dtype = torch.float32
    seed: int = 4
    state_sigma: float = 0.05
    step_seed_base: int = 4_000_000


# The five workloads of the operator (sizes, distributions and seeds).
ORACLE_FP32 = FwdCase("oracle_fp32_B1_H2_T256_d64", 1, 256, 2, 64, 64, torch.float32, seed=0)
LAYER_BF16 = FwdCase("layer_bf16_B1_H16_T4096_d128", 1, 4096, 16, 128, 128, torch.bfloat16, seed=1)
TRAIN_BF16 = FwdCase("train_bf16_B8_H16_T4096_d128", 8, 4096, 16, 128, 128, torch.bfloat16, seed=2,
                     s0_sigma=0.02)
LONG_BF16 = FwdCase("long_bf16_B1_H16_T65536_d128", 1, 65536, 16, 128, 128, torch.bfloat16, seed=3,
                    log_alpha_range=(-9.0, 0.0), gate_sigma=2.0)
DECODE_F32 = DecodeCase("decode_f32_B256_H16_d128_1000steps", 256, 16, 128, 128, steps=1000)

FWD_CASES = {c.name: c for c in (ORACLE_FP32, LAYER_BF16, TRAIN_BF16, LONG_BF16)}


def _l2norm(x: torch.Tensor) -> torch.Tensor:
    return x / x.norm(dim=-1, keepdim=True).clamp_min(1e-12)


def draw_fwd(B, T, H, dk, dv, *, seed, dtype=torch.float32, log_alpha_range=(-5.0, -1.0),
             gate_sigma=1.0, s0_sigma=0.0, with_s0=None):
    """Draw one forward batch.  Returns a dict of CPU tensors.

    q, k, v, b, w are in ``dtype``; log_alpha and S0 are fp32.  ``S0`` is None
    when ``s0_sigma == 0`` unless ``with_s0`` forces a zero tensor.
    """
    g = torch.Generator(device="cpu").manual_seed(int(seed))
    q = _l2norm(torch.randn(B, T, H, dk, generator=g))
    k = _l2norm(torch.randn(B, T, H, dk, generator=g))
    v = torch.nn.functional.silu(torch.randn(B, T, H, dv, generator=g))
    b = torch.sigmoid(gate_sigma * torch.randn(B, T, H, dk, generator=g))
    w = torch.sigmoid(gate_sigma * torch.randn(B, T, H, dv, generator=g))
    lo, hi = log_alpha_range
    u = torch.rand(B, T, H, dk, generator=g) * (hi - lo) + lo
    log_alpha = -torch.exp(u)
    if s0_sigma > 0:
        S0 = s0_sigma * torch.randn(B, H, dk, dv, generator=g)
    elif with_s0:
        S0 = torch.zeros(B, H, dk, dv)
    else:
        S0 = None
    out = dict(q=q, k=k, v=v, b=b, w=w)
    out = {n: t.to(dtype).contiguous() for n, t in out.items()}
    out["log_alpha"] = log_alpha.contiguous()
    out["S0"] = S0
    return out


def draw_case(case: FwdCase, *, T=None, B=None, seed=None):
    """Draw a workload's inputs, optionally at a different T/B/seed."""
    return draw_fwd(B or case.B, T or case.T, case.H, case.dk, case.dv,
                    seed=case.seed if seed is None else seed, dtype=case.dtype,
                    log_alpha_range=case.log_alpha_range, gate_sigma=case.gate_sigma,
                    s0_sigma=case.s0_sigma)


def draw_decode_state(case: DecodeCase, B=None):
    g = torch.Generator(device="cpu").manual_seed(int(case.seed))
    return case.state_sigma * torch.randn(B or case.B, case.H, case.dk, case.dv, generator=g)


def draw_decode_token(case: DecodeCase, step: int, B=None):
    """Per-token decode inputs for one step ([B,H,d]); drawn like the fp32 forward case."""
    d = draw_fwd(B or case.B, 1, case.H, case.dk, case.dv, seed=case.step_seed_base + step,
                 dtype=case.dtype)
    return {n: (t[:, 0].contiguous() if t is not None else None) for n, t in d.items()
            if n != "S0"}


def draw_fwd_device(B, T, H, dk, dv, *, seed, device, dtype=torch.bfloat16,
                    log_alpha_range=(-5.0, -1.0), gate_sigma=1.0):
    """Same recipe drawn with a device generator (for timing-only buffers)."""
    g = torch.Generator(device=device).manual_seed(int(seed))

    def rn(*s):
        return torch.randn(*s, generator=g, device=device)
    q = _l2norm(rn(B, T, H, dk))
    k = _l2norm(rn(B, T, H, dk))
    v = torch.nn.functional.silu(rn(B, T, H, dv))
    b = torch.sigmoid(gate_sigma * rn(B, T, H, dk))
    w = torch.sigmoid(gate_sigma * rn(B, T, H, dv))
    lo, hi = log_alpha_range
    u = torch.rand(B, T, H, dk, generator=g, device=device) * (hi - lo) + lo
    out = {n: t.to(dtype).contiguous() for n, t in dict(q=q, k=k, v=v, b=b, w=w).items()}
    out["log_alpha"] = (-torch.exp(u)).contiguous()
    return out


# Decay distributions beyond the workloads' own, for the edge of the method
# where alpha approaches 0 (fast-forgetting channels):
#   "wide":   log_alpha = -exp(U(-1, 3)), i.e. from about -0.37 down to about -20 per token;
#   "all3":   every channel at -3 per token;
#   "mixed":  per (head, channel) either -20 (forgets within a token) or -1e-4 (keeps);
#   "zeros":  the workload distribution, with alpha = 0 exactly (log_alpha = -inf)
#             at a random 2% of (token, channel) entries.
DECAY_KINDS = ("wide", "all3", "mixed", "zeros")


def draw_log_alpha(B, T, H, dk, kind, *, seed):
    """log_alpha [B,T,H,dk] (fp32) of one of the DECAY_KINDS distributions."""
    g = torch.Generator(device="cpu").manual_seed(int(seed))
    if kind == "wide":
        return (-torch.exp(torch.rand(B, T, H, dk, generator=g) * 4.0 - 1.0)).contiguous()
    if kind == "all3":
        return torch.full((B, T, H, dk), -3.0)
    if kind == "mixed":
        fast = torch.rand(1, 1, H, dk, generator=g) < 0.5
        la = torch.where(fast, torch.tensor(-20.0), torch.tensor(-1e-4))
        return la.expand(B, T, H, dk).contiguous()
    if kind == "zeros":
        la = -torch.exp(torch.rand(B, T, H, dk, generator=g) * 4.0 - 5.0)
        la[torch.rand(B, T, H, dk, generator=g) < 0.02] = float("-inf")
        return la.contiguous()
    raise ValueError(kind)


def collinear_keys(d, *, eps, seed, erase_lo=1.95):
    """Ill-conditioned chunks: within each 64-token chunk of a (batch, head) the
    keys are one unit direction plus eps * noise (normalised), and the erase gate
    is drawn in [erase_lo, 2).  Replaces k and b of a forward batch."""
    B, T, H, dk = d["k"].shape
    g = torch.Generator(device="cpu").manual_seed(int(seed))
    nc = (T + 63) // 64
    base = torch.randn(B, nc, H, dk, generator=g)
    base = base.repeat_interleave(64, dim=1)[:, :T]
    k = _l2norm(_l2norm(base) + eps * torch.randn(B, T, H, dk, generator=g))
    b = erase_lo + (2.0 - erase_lo) * torch.rand(B, T, H, dk, generator=g)
    out = dict(d)
    out["k"] = k.to(d["k"].dtype).contiguous()
    out["b"] = b.to(d["b"].dtype).contiguous()
    return out


def scalar_gates(d, layout, *, seed, gate_sigma=1.0):
    """Replace b, w and/or log_alpha of a forward batch by one value per (token,
    head) ([B,T,H]), as the gdn2_gate_layout bits in `layout` say: bit 1 erase
    gate b, bit 2 write gate w (bits 1 and 2 together: one beta for both, the
    same tensor), bit 4 the decay.  Drawn like the per-channel values."""
    B, T, H, _ = d["q"].shape
    g = torch.Generator(device="cpu").manual_seed(int(seed))
    out = dict(d)
    dtype = d["q"].dtype
    beta = torch.sigmoid(gate_sigma * torch.randn(B, T, H, generator=g)).to(dtype).contiguous()
    if layout & 1:
        out["b"] = beta
    if layout & 2:
        out["w"] = beta if layout & 1 else \
            torch.sigmoid(gate_sigma * torch.randn(B, T, H, generator=g)).to(dtype).contiguous()
    if layout & 4:
        out["log_alpha"] = (-torch.exp(torch.rand(B, T, H, generator=g) * 4.0 - 5.0)).contiguous()
    return out


def draw_layer(B, T, H, dk, dv, *, seed, dtype=torch.float32, s0_sigma=0.0):
    """Inputs of the fused layer entry point: q, k and v as they leave the
    layer's convolution and SiLU (no L2 normalisation), pre-sigmoid logits for
    the erase, write, decay and output gates, and the RMS-norm weight.  Logit
    scales put the gates and alpha = sigmoid(decay_logit) across (0, 1), with
    decays near 1 (as the workloads' log_alpha = -exp(U(-5, -1))) and a spread
    of faster ones.  Returns a dict of CPU tensors (logits of the decay and the
    weight in fp32, the rest in ``dtype``)."""
    g = torch.Generator(device="cpu").manual_seed(int(seed))
    silu = torch.nn.functional.silu
    q = silu(torch.randn(B, T, H, dk, generator=g))
    k = silu(torch.randn(B, T, H, dk, generator=g))
    v = silu(torch.randn(B, T, H, dv, generator=g))
    b_logit = torch.randn(B, T, H, dk, generator=g)
    w_logit = torch.randn(B, T, H, dv, generator=g)
    decay_logit = 2.0 + 2.5 * torch.randn(B, T, H, dk, generator=g)
    g_logit = torch.randn(B, T, H, dv, generator=g)
    norm_weight = 1.0 + 0.1 * torch.randn(dv, generator=g)
    S0 = s0_sigma * torch.randn(B, H, dk, dv, generator=g) if s0_sigma > 0 else None
    out = {n: t.to(dtype).contiguous() for n, t in
           dict(q=q, k=k, v=v, b_logit=b_logit, w_logit=w_logit, g_logit=g_logit).items()}
    out["decay_logit"] = decay_logit.contiguous()
    out["norm_weight"] = norm_weight.contiguous()
    out["S0"] = S0
    return out
