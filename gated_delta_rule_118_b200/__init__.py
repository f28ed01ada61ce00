"""Gated DeltaNet-2 operator on B200: Python binding of libgdn2.so.

The binding only marshals torch tensors (device memory) and the current CUDA
stream into the C ABI declared in ``include/gdn2.h``; every step of the
operator runs in the library's CUDA kernels.  There is no CPU fallback: if the
native library is missing or cannot be loaded, every call raises.
"""
from __future__ import annotations

import ctypes
from pathlib import Path

import torch

_PKG = Path(__file__).resolve().parent
LIBRARY_PATH = _PKG / "libgdn2.so"

GDN2_OK = 0
GDN2_ERR_NULL = 1
GDN2_ERR_SHAPE = 2
GDN2_ERR_DTYPE = 3
GDN2_ERR_ALIGN = 4
GDN2_ERR_UNSUPPORTED = 5
GDN2_ERR_CUDA = 6
GDN2_ERR_DEVICE_TIMEOUT = 7
GDN2_ERR_RANGE = 8
GDN2_ERR_SCRATCH_LIMIT = 9

GDN2_F32 = 0
GDN2_BF16 = 1

# gdn2_gate_layout bits: which gates hold one value per (token, head)
GDN2_GATES_PER_CHANNEL = 0
GDN2_ERASE_SCALAR = 1
GDN2_WRITE_SCALAR = 2
GDN2_DECAY_SCALAR = 4

# Every symbol include/gdn2.h declares.
EXPORTED = ("gdn2_fwd_chunked", "gdn2_fwd_chunked_gates", "gdn2_fwd_chunked_noalloc",
            "gdn2_layer_fwd", "gdn2_bwd_chunked", "gdn2_decode_step", "gdn2_decode_tokens", "gdn2_check_device_error",
            "gdn2_selftest_bounded_wait", "gdn2_fwd_chunked_launches", "gdn2_status_string")

_lib = None


class Gdn2Error(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)}")


def lib() -> ctypes.CDLL:
    """Load libgdn2.so (built in-tree by ``gated_delta_rule_118_b200.build``)."""
    global _lib
    if _lib is None:
        if not LIBRARY_PATH.exists():
            raise RuntimeError(f"native library {LIBRARY_PATH} is missing; run "
                               "`python -m gated_delta_rule_118_b200.build` (there is no fallback)")
        L = ctypes.CDLL(str(LIBRARY_PATH))
        vp, fp, ci = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int
        L.gdn2_fwd_chunked.argtypes = [vp] * 5 + [fp, fp, vp, fp] + [ci] * 6 + [vp]
        L.gdn2_fwd_chunked.restype = ci
        L.gdn2_fwd_chunked_gates.argtypes = [vp] * 5 + [fp, fp, vp, fp] + [ci] * 6 + [ctypes.c_uint, vp]
        L.gdn2_fwd_chunked_gates.restype = ci
        L.gdn2_decode_tokens.argtypes = [vp] * 5 + [fp, fp, vp] + [ci] * 6 + [ctypes.c_uint, vp]
        L.gdn2_decode_tokens.restype = ci
        L.gdn2_layer_fwd.argtypes = [vp] * 5 + [fp, vp, fp, ctypes.c_float, fp, vp, fp] + [ci] * 6 + [vp]
        L.gdn2_layer_fwd.restype = ci
        L.gdn2_bwd_chunked.argtypes = [vp] * 5 + [fp, fp, vp, fp] + [fp] * 7 + [ci] * 6 + [vp]
        L.gdn2_bwd_chunked.restype = ci
        L.gdn2_fwd_chunked_noalloc.argtypes = [vp] * 5 + [fp, fp, vp, fp] + [ci] * 6 + [vp]
        L.gdn2_fwd_chunked_noalloc.restype = ci
        L.gdn2_decode_step.argtypes = [vp] * 5 + [fp, fp, vp] + [ci] * 5 + [vp]
        L.gdn2_decode_step.restype = ci
        L.gdn2_check_device_error.argtypes = [vp]
        L.gdn2_check_device_error.restype = ci
        L.gdn2_selftest_bounded_wait.argtypes = [vp]
        L.gdn2_selftest_bounded_wait.restype = ci
        L.gdn2_fwd_chunked_launches.argtypes = [ci] * 6
        L.gdn2_fwd_chunked_launches.restype = ci
        L.gdn2_status_string.argtypes = [ci]
        L.gdn2_status_string.restype = ctypes.c_char_p
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().gdn2_status_string(int(status)).decode()


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return GDN2_F32
    if t.dtype == torch.bfloat16:
        return GDN2_BF16
    raise TypeError(f"unsupported dtype {t.dtype}")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _gate_layout(q, b, w, log_alpha):
    """gdn2_gate_layout bits from the shapes: a gate of shape q.shape[:-1] is per (token, head)."""
    tok = tuple(q.shape[:-1])
    return ((GDN2_ERASE_SCALAR if tuple(b.shape) == tok else 0)
            | (GDN2_WRITE_SCALAR if tuple(w.shape) == tok else 0)
            | (GDN2_DECAY_SCALAR if tuple(log_alpha.shape) == tok else 0))


def gdn2_fwd_chunked(q, k, v, b, w, log_alpha, S0=None, o=None, S_T=None, *,
                     stream=None, want_state=True, check=True):
    """Chunked forward.  Tensors are CUDA, contiguous, [B,T,H,d]; returns (o, S_T).

    ``o`` and ``S_T`` are allocated with torch when not given (S_T only when
    ``want_state``).  b, w or log_alpha of shape [B,T,H] (one value per token and
    head) select the matching gate layout (gdn2_fwd_chunked_gates).  Raises
    Gdn2Error on a non-OK status.
    """
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if o is None:
        o = torch.empty((B, T, H, dv), dtype=q.dtype, device=q.device)
    if S_T is None and want_state:
        S_T = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device)
    for name, t in (("q", q), ("k", k), ("v", v), ("b", b), ("w", w), ("log_alpha", log_alpha),
                    ("o", o), ("S0", S0), ("S_T", S_T)):
        if t is not None and not (t.is_cuda and t.is_contiguous()):
            raise ValueError(f"{name} must be a contiguous CUDA tensor")
    if log_alpha.dtype != torch.float32 or (S0 is not None and S0.dtype != torch.float32):
        raise TypeError("log_alpha and S0 must be float32")
    layout = _gate_layout(q, b, w, log_alpha)
    if layout:
        st = lib().gdn2_fwd_chunked_gates(_ptr(q), _ptr(k), _ptr(v), _ptr(b), _ptr(w), _ptr(log_alpha),
                                          _ptr(S0), _ptr(o), _ptr(S_T), B, T, H, dk, dv, _dtype_code(q),
                                          layout, _stream(stream))
    else:
        st = lib().gdn2_fwd_chunked(_ptr(q), _ptr(k), _ptr(v), _ptr(b), _ptr(w), _ptr(log_alpha),
                                    _ptr(S0), _ptr(o), _ptr(S_T), B, T, H, dk, dv, _dtype_code(q),
                                    _stream(stream))
    if check and st != GDN2_OK:
        raise Gdn2Error(st, "gdn2_fwd_chunked_gates" if layout else "gdn2_fwd_chunked")
    return o, S_T


def gdn2_fwd_chunked_noalloc(q, k, v, b, w, log_alpha, S0=None, o=None, S_T=None, *, stream=None,
                             check=True):
    """The chunked forward through the entry point that allocates no device memory.

    Pass ``o`` (and ``S_T`` when the final state is wanted) preallocated; the
    native call itself uses only its fixed scratch buffer.  Returns (o, S_T).
    """
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if o is None:
        raise ValueError("gdn2_fwd_chunked_noalloc needs a preallocated output o")
    for name, t in (("q", q), ("k", k), ("v", v), ("b", b), ("w", w), ("log_alpha", log_alpha),
                    ("o", o), ("S0", S0), ("S_T", S_T)):
        if t is not None and not (t.is_cuda and t.is_contiguous()):
            raise ValueError(f"{name} must be a contiguous CUDA tensor")
    st = lib().gdn2_fwd_chunked_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(b), _ptr(w),
                                        _ptr(log_alpha), _ptr(S0), _ptr(o), _ptr(S_T),
                                        B, T, H, dk, dv, _dtype_code(q), _stream(stream))
    if check and st != GDN2_OK:
        raise Gdn2Error(st, "gdn2_fwd_chunked_noalloc")
    return o, S_T


def gdn2_decode_step(q, k, v, b, w, log_alpha, S, o=None, *, stream=None, check=True):
    """One recurrent token: [B,H,d] inputs, S [B,H,dk,dv] fp32 updated in place; returns o."""
    B, H, dk = q.shape
    dv = v.shape[-1]
    if o is None:
        o = torch.empty((B, H, dv), dtype=q.dtype, device=q.device)
    st = lib().gdn2_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(b), _ptr(w), _ptr(log_alpha),
                                _ptr(S), _ptr(o), B, H, dk, dv, _dtype_code(q), _stream(stream))
    if check and st != GDN2_OK:
        raise Gdn2Error(st, "gdn2_decode_step")
    return o


def gdn2_layer_fwd(q, k, v, b_logit, w_logit, decay_logit, g_logit, norm_weight, eps=1e-6, S0=None,
                   y=None, S_T=None, *, stream=None, want_state=True, check=True):
    """The operator with the layer's processing fused around it: L2-normalised q and
    k, sigmoid gates from logits, log_alpha = log sigmoid(decay_logit), and
    y = RMSNorm(o) * norm_weight * sigmoid(g_logit).  Tensors are CUDA, contiguous,
    [B,T,H,d] (norm_weight [dv] fp32, decay_logit fp32); returns (y, S_T)."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if y is None:
        y = torch.empty((B, T, H, dv), dtype=q.dtype, device=q.device)
    if S_T is None and want_state:
        S_T = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device)
    for name, t in (("q", q), ("k", k), ("v", v), ("b_logit", b_logit), ("w_logit", w_logit),
                    ("decay_logit", decay_logit), ("g_logit", g_logit), ("norm_weight", norm_weight),
                    ("y", y), ("S0", S0), ("S_T", S_T)):
        if t is not None and not (t.is_cuda and t.is_contiguous()):
            raise ValueError(f"{name} must be a contiguous CUDA tensor")
    if decay_logit.dtype != torch.float32 or norm_weight.dtype != torch.float32:
        raise TypeError("decay_logit and norm_weight must be float32")
    st = lib().gdn2_layer_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(b_logit), _ptr(w_logit), _ptr(decay_logit),
                              _ptr(g_logit), _ptr(norm_weight), ctypes.c_float(eps), _ptr(S0), _ptr(y),
                              _ptr(S_T), B, T, H, dk, dv, _dtype_code(q), _stream(stream))
    if check and st != GDN2_OK:
        raise Gdn2Error(st, "gdn2_layer_fwd")
    return y, S_T


def gdn2_bwd_chunked(q, k, v, b, w, log_alpha, S0, dO, dS_T=None, *, stream=None, check=True,
                     want_dS0=True):
    """Backward of the chunked forward: gradients of sum(o * dO) + sum(S_T * dS_T).
    Inputs as for gdn2_fwd_chunked plus dO [B,T,H,dv] (input dtype) and dS_T
    [B,H,dk,dv] fp32 or None; returns a dict of fp32 tensors dq, dk, dv, db, dw,
    dlog_alpha and dS0 (None unless want_dS0)."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    f32 = dict(dtype=torch.float32, device=q.device)
    g = {n: torch.empty((B, T, H, dk), **f32) for n in ("dq", "dk", "db", "dlog_alpha")}
    g.update({n: torch.empty((B, T, H, dv), **f32) for n in ("dv", "dw")})
    g["dS0"] = torch.empty((B, H, dk, dv), **f32) if want_dS0 else None
    for name, t in (("q", q), ("k", k), ("v", v), ("b", b), ("w", w), ("log_alpha", log_alpha),
                    ("S0", S0), ("dO", dO), ("dS_T", dS_T)):
        if t is not None and not (t.is_cuda and t.is_contiguous()):
            raise ValueError(f"{name} must be a contiguous CUDA tensor")
    st = lib().gdn2_bwd_chunked(_ptr(q), _ptr(k), _ptr(v), _ptr(b), _ptr(w), _ptr(log_alpha), _ptr(S0),
                                _ptr(dO), _ptr(dS_T), _ptr(g["dq"]), _ptr(g["dk"]), _ptr(g["dv"]),
                                _ptr(g["db"]), _ptr(g["dw"]), _ptr(g["dlog_alpha"]), _ptr(g["dS0"]),
                                B, T, H, dk, dv, _dtype_code(q), _stream(stream))
    if check and st != GDN2_OK:
        raise Gdn2Error(st, "gdn2_bwd_chunked")
    return g


def gdn2_decode_tokens(q, k, v, b, w, log_alpha, S, o=None, *, stream=None, check=True):
    """T recurrent tokens on a resident state: [B,T,H,d] inputs (b, w, log_alpha may be
    [B,T,H]: one value per token and head), S [B,H,dk,dv] fp32 updated in place;
    returns o [B,T,H,dv]."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if o is None:
        o = torch.empty((B, T, H, dv), dtype=q.dtype, device=q.device)
    for name, t in (("q", q), ("k", k), ("v", v), ("b", b), ("w", w), ("log_alpha", log_alpha),
                    ("S", S), ("o", o)):
        if not (t.is_cuda and t.is_contiguous()):
            raise ValueError(f"{name} must be a contiguous CUDA tensor")
    st = lib().gdn2_decode_tokens(_ptr(q), _ptr(k), _ptr(v), _ptr(b), _ptr(w), _ptr(log_alpha),
                                  _ptr(S), _ptr(o), B, T, H, dk, dv, _dtype_code(q),
                                  _gate_layout(q, b, w, log_alpha), _stream(stream))
    if check and st != GDN2_OK:
        raise Gdn2Error(st, "gdn2_decode_tokens")
    return o


def gdn2_check_device_error(stream=None) -> int:
    """Synchronise ``stream`` and return (and clear) the device error status."""
    return int(lib().gdn2_check_device_error(_stream(stream)))


def gdn2_selftest_bounded_wait(stream=None) -> int:
    """Queue the bounded-wait self-test (a wait that runs out after one second)."""
    return int(lib().gdn2_selftest_bounded_wait(_stream(stream)))


def gdn2_fwd_chunked_launches(B, T, H, dk, dv, dtype=torch.bfloat16) -> int:
    """Kernel launches one gdn2_fwd_chunked call makes for this problem."""
    code = GDN2_BF16 if dtype == torch.bfloat16 else GDN2_F32
    return int(lib().gdn2_fwd_chunked_launches(B, T, H, dk, dv, code))


def gdn2_status_string(status: int) -> str:
    return status_string(status)
