"""fp64 CPU oracle for the Gated DeltaNet-2 operator -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its Python binding) never imports it; the two share no code.

The arithmetic lives in ``gdn2_oracle.c`` (plain C, double precision, one token
at a time): the per-token update of "Gated DeltaNet-2: Decoupling Erase and
Write in Linear Attention" as stated on the iplexlaw.co.kr page, section
"Decisiones independientes en dos ejes", and in the update equation of the
zubnet.ai news page.  This module only compiles that file and marshals numpy
arrays into it.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from pathlib import Path

import numpy as np

_HERE = Path(__file__).resolve().parent
SOURCE = _HERE / "gdn2_oracle.c"
LIBRARY = _HERE / "libgdn2_oracle.so"


def compile_oracle(source: Path = SOURCE, out: Path = LIBRARY) -> Path:
    """Compile an oracle C source into a shared library with gcc (-O2, OpenMP)."""
    cmd = ["gcc", "-O2", "-std=c99", "-fopenmp", "-fPIC", "-shared",
           str(source), "-o", str(out), "-lm"]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    return out


def _stale(lib: Path, src: Path) -> bool:
    return (not lib.exists()) or lib.stat().st_mtime < src.stat().st_mtime


class Oracle:
    """Handle on one compiled oracle library."""

    def __init__(self, path: Path):
        self.path = Path(path)
        self._lib = ctypes.CDLL(str(self.path))
        dp = ctypes.POINTER(ctypes.c_double)
        self._lib.gdn2_oracle_fwd.argtypes = [dp] * 9 + [ctypes.c_int] * 6
        self._lib.gdn2_oracle_fwd.restype = ctypes.c_int
        self._lib.gdn2_oracle_bwd.argtypes = [dp] * 16 + [ctypes.c_int] * 6
        self._lib.gdn2_oracle_bwd.restype = ctypes.c_int
        self._lib.gdn2_oracle_max_threads.argtypes = []
        self._lib.gdn2_oracle_max_threads.restype = ctypes.c_int

    def max_threads(self) -> int:
        return int(self._lib.gdn2_oracle_max_threads())

    @staticmethod
    def _f64(x) -> np.ndarray:
        if hasattr(x, "detach"):  # a torch tensor: take its exact values
            x = x.detach().to("cpu").double().numpy()
        return np.ascontiguousarray(np.asarray(x, dtype=np.float64))

    def fwd(self, q, k, v, b, w, log_alpha, S0=None, nthreads: int = 0):
        """Run the recurrence over [B,T,H,d] inputs; return (o, S_T) in fp64.

        q, k, b, log_alpha: [B,T,H,dk]; v, w: [B,T,H,dv]; S0: [B,H,dk,dv] or
        None for a zero initial state.  o: [B,T,H,dv]; S_T: [B,H,dk,dv].
        """
        q, k, v, b, w, la = (self._f64(a) for a in (q, k, v, b, w, log_alpha))
        B, T, H, dk = q.shape
        dv = v.shape[-1]
        for name, a, last in (("k", k, dk), ("b", b, dk), ("log_alpha", la, dk),
                              ("w", w, dv)):
            if a.shape != (B, T, H, last):
                raise ValueError(f"{name} has shape {a.shape}, expected {(B, T, H, last)}")
        if v.shape != (B, T, H, dv):
            raise ValueError(f"v has shape {v.shape}")
        s0 = None
        if S0 is not None:
            s0 = self._f64(S0)
            if s0.shape != (B, H, dk, dv):
                raise ValueError(f"S0 has shape {s0.shape}, expected {(B, H, dk, dv)}")
        o = np.zeros((B, T, H, dv), dtype=np.float64)
        st = np.zeros((B, H, dk, dv), dtype=np.float64)
        dp = ctypes.POINTER(ctypes.c_double)

        def ptr(a):
            return a.ctypes.data_as(dp) if a is not None else None

        rc = self._lib.gdn2_oracle_fwd(ptr(q), ptr(k), ptr(v), ptr(b), ptr(w), ptr(la),
                                       ptr(s0), ptr(o), ptr(st),
                                       B, T, H, dk, dv, int(nthreads))
        if rc != 0:
            raise RuntimeError(f"gdn2_oracle_fwd failed with code {rc}")
        return o, st

    def bwd(self, q, k, v, b, w, log_alpha, S0, dO, dS_T=None, nthreads: int = 0):
        """Gradients of sum(o * dO) + sum(S_T * dS_T) (backpropagation through
        the recurrence, fp64): returns dict dq, dk, dv, db, dw, dlog_alpha, dS0."""
        q, k, v, b, w, la, dO = (self._f64(a) for a in (q, k, v, b, w, log_alpha, dO))
        B, T, H, dk = q.shape
        dv = v.shape[-1]
        if dO.shape != (B, T, H, dv):
            raise ValueError(f"dO has shape {dO.shape}")
        s0 = None if S0 is None else self._f64(S0)
        dst = None if dS_T is None else self._f64(dS_T)
        out = {n: np.zeros((B, T, H, dk)) for n in ("dq", "dk", "db", "dlog_alpha")}
        out.update({n: np.zeros((B, T, H, dv)) for n in ("dv", "dw")})
        out["dS0"] = np.zeros((B, H, dk, dv))
        dp = ctypes.POINTER(ctypes.c_double)

        def ptr(a):
            return a.ctypes.data_as(dp) if a is not None else None

        rc = self._lib.gdn2_oracle_bwd(ptr(q), ptr(k), ptr(v), ptr(b), ptr(w), ptr(la), ptr(s0), ptr(dO),
                                       ptr(dst), ptr(out["dq"]), ptr(out["dk"]), ptr(out["dv"]), ptr(out["db"]),
                                       ptr(out["dw"]), ptr(out["dlog_alpha"]), ptr(out["dS0"]),
                                       B, T, H, dk, dv, int(nthreads))
        if rc != 0:
            raise RuntimeError(f"gdn2_oracle_bwd failed with code {rc}")
        return out

    def decode_step(self, q, k, v, b, w, log_alpha, S, nthreads: int = 0):
        """One token of the recurrence: [B,H,d] inputs and state -> (o, S_new)."""
        ins = [self._f64(a)[:, None] for a in (q, k, v, b, w, log_alpha)]
        o, s_new = self.fwd(*ins, S0=S, nthreads=nthreads)
        return o[:, 0], s_new


_default: Oracle | None = None


def load(path: Path | None = None) -> Oracle:
    """Return the oracle, compiling ``gdn2_oracle.c`` first if needed."""
    global _default
    if path is not None:
        return Oracle(path)
    if _default is None:
        if _stale(LIBRARY, SOURCE):
            compile_oracle()
        _default = Oracle(LIBRARY)
    return _default


def fwd(*args, **kwargs):
    return load().fwd(*args, **kwargs)


def decode_step(*args, **kwargs):
    return load().decode_step(*args, **kwargs)


def bwd(*args, **kwargs):
    return load().bwd(*args, **kwargs)


def host_cores() -> int:
    return len(os.sched_getaffinity(0))
