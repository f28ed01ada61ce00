"""Helpers for GPU-vs-oracle parity tests."""
import numpy as np
import torch

# Tolerances on max|x - x_ref| / max|x_ref| over a tensor (stated for the operator):
TOL_F32 = 1e-4   # fp32 inputs
TOL_BF16 = 2e-2  # bf16 inputs, fp32 accumulation and state


def rel_err(x, ref):
    x = x.detach().double().cpu().numpy() if isinstance(x, torch.Tensor) else np.asarray(x, np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert x.shape == ref.shape, (x.shape, ref.shape)
    denom = np.abs(ref).max()
    return float(np.abs(x - ref).max() / (denom if denom > 0 else 1.0))


def to_dev(d, device="cuda"):
    return {n: (t.to(device) if t is not None else None) for n, t in d.items()}
