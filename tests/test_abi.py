"""The C-ABI library builds, loads, exports every declared symbol and rejects
bad arguments on the host before touching a GPU (CPU-only tests)."""
import ctypes
import re
from pathlib import Path

import pytest

import gated_delta_rule_118_b200 as g
from gated_delta_rule_118_b200 import build

HEADER = Path(__file__).resolve().parent.parent / "include" / "gdn2.h"


@pytest.fixture(scope="module")
def lib():
    build.build_library()
    return g.lib()


def declared_functions():
    text = re.sub(r"/\*.*?\*/", "", HEADER.read_text(), flags=re.S)
    return sorted(set(re.findall(r"\b(gdn2_[a-z0-9_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert set(names) == set(g.EXPORTED), names
    for n in names:
        assert hasattr(lib, n), f"{n} not exported by {g.LIBRARY_PATH}"


def test_library_is_built_for_sm100a(lib):
    # the build passes only compute_100a/sm_100a to nvcc
    assert build.ARCH == ["-gencode", "arch=compute_100a,code=sm_100a"]


def test_launch_count_query(lib):
    # one persistent launch where the chains take at most a quarter of the SMs
    # (16 heads x 2 value tiles of 64, of 148), else per window of chunks
    assert g.gdn2_fwd_chunked_launches(1, 4096, 16, 128, 128) == 1
    assert g.gdn2_fwd_chunked_launches(1, 65536, 16, 128, 128) == 1
    # the training batch: prep and chains with the outputs, one window over 64 chunks
    assert g.gdn2_fwd_chunked_launches(8, 4096, 16, 128, 128) == 2
    # chains on more than a quarter but at most half of the SMs: three kernels a window
    assert g.gdn2_fwd_chunked_launches(2, 4096, 16, 128, 128) % 3 == 0
    assert g.gdn2_fwd_chunked_launches(1, 256, 2, 64, 64, __import__("torch").float32) == 1
    assert g.gdn2_fwd_chunked_launches(1, 0, 2, 128, 128) == 0
    assert g.gdn2_fwd_chunked_launches(0, 10, 2, 128, 128) == -1


def test_status_strings(lib):
    for code in range(10):
        s = g.status_string(code)
        assert s.startswith("GDN2_")
    assert "unknown" in g.status_string(99)


# Host-side validation.  Fake (never dereferenced) device addresses: every
# call below must be rejected before any CUDA call is made.
P = ctypes.c_void_p(0x10000)       # 16-byte aligned
MIS = ctypes.c_void_p(0x10008)     # misaligned


def fwd(lib, *, q=P, o=P, S0=None, B=1, T=8, H=2, dk=64, dv=64, dtype=1):
    return lib.gdn2_fwd_chunked(q, P, P, P, P, P, S0, o, None, B, T, H, dk, dv, dtype, None)


def dec(lib, *, S=P, B=1, H=2, dk=64, dv=64, dtype=0, q=P):
    return lib.gdn2_decode_step(q, P, P, P, P, P, S, P, B, H, dk, dv, dtype, None)


@pytest.mark.parametrize("kw,code", [
    (dict(dtype=5), g.GDN2_ERR_DTYPE),
    (dict(B=0), g.GDN2_ERR_SHAPE),
    (dict(H=-1), g.GDN2_ERR_SHAPE),
    (dict(T=-3), g.GDN2_ERR_SHAPE),
    (dict(dk=0), g.GDN2_ERR_SHAPE),
    (dict(dk=96), g.GDN2_ERR_UNSUPPORTED),
    (dict(dv=256), g.GDN2_ERR_UNSUPPORTED),
    (dict(B=70000), g.GDN2_ERR_UNSUPPORTED),
    (dict(q=None), g.GDN2_ERR_NULL),
    (dict(o=None), g.GDN2_ERR_NULL),
    (dict(q=MIS), g.GDN2_ERR_ALIGN),
    (dict(S0=MIS), g.GDN2_ERR_ALIGN),
])
def test_fwd_rejects_bad_arguments(lib, kw, code):
    assert fwd(lib, **kw) == code


@pytest.mark.parametrize("kw,code", [
    (dict(dtype=2), g.GDN2_ERR_DTYPE),
    (dict(B=0), g.GDN2_ERR_SHAPE),
    (dict(dk=32), g.GDN2_ERR_UNSUPPORTED),
    (dict(S=None), g.GDN2_ERR_NULL),
    (dict(q=MIS), g.GDN2_ERR_ALIGN),
])
def test_decode_rejects_bad_arguments(lib, kw, code):
    assert dec(lib, **kw) == code


def test_noalloc_rejects_pairs_beyond_its_scratch(lib):
    # One chunk of records and state image plus the carried state take 185 KiB per
    # (batch, head) pair at dv = 128: 178 pairs exceed the 32 MiB buffer.  (Only
    # the rejection is checked here: an accepted call would launch.)
    for B, H in ((1, 178), (2, 89), (178, 1)):
        st = lib.gdn2_fwd_chunked_noalloc(P, P, P, P, P, P, None, P, None, B, 64, H, 128, 128, 1, None)
        assert st == g.GDN2_ERR_SCRATCH_LIMIT, (B, H)


def fwd_gates(lib, *, layout=0, B=1, T=8, H=2, dk=64, dv=64, dtype=1, b=P):
    return lib.gdn2_fwd_chunked_gates(P, P, P, b, P, P, None, P, None, B, T, H, dk, dv, dtype, layout, None)


def dec_tokens(lib, *, layout=0, B=1, T=4, H=2, dk=64, dv=64, dtype=0, o=P):
    return lib.gdn2_decode_tokens(P, P, P, P, P, P, P, o, B, T, H, dk, dv, dtype, layout, None)


@pytest.mark.parametrize("kw,code", [
    (dict(layout=8), g.GDN2_ERR_UNSUPPORTED),
    (dict(layout=0xFFFF), g.GDN2_ERR_UNSUPPORTED),
    (dict(dtype=7), g.GDN2_ERR_DTYPE),
    (dict(B=0), g.GDN2_ERR_SHAPE),
    (dict(dk=48), g.GDN2_ERR_UNSUPPORTED),
    (dict(b=None), g.GDN2_ERR_NULL),
    (dict(b=MIS, layout=1), g.GDN2_ERR_ALIGN),
])
def test_fwd_gates_rejects_bad_arguments(lib, kw, code):
    assert fwd_gates(lib, **kw) == code


@pytest.mark.parametrize("kw,code", [
    (dict(T=0), g.GDN2_ERR_SHAPE),
    (dict(T=-1), g.GDN2_ERR_SHAPE),
    (dict(layout=16), g.GDN2_ERR_UNSUPPORTED),
    (dict(dtype=3), g.GDN2_ERR_DTYPE),
    (dict(dv=32), g.GDN2_ERR_UNSUPPORTED),
    (dict(o=None), g.GDN2_ERR_NULL),
    (dict(o=MIS), g.GDN2_ERR_ALIGN),
])
def test_decode_tokens_rejects_bad_arguments(lib, kw, code):
    assert dec_tokens(lib, **kw) == code


def test_gate_layout_from_shapes():
    import torch
    q = torch.empty(2, 5, 3, 8)
    per_ch = torch.empty(2, 5, 3, 8)
    tok = torch.empty(2, 5, 3)
    assert g._gate_layout(q, per_ch, per_ch, per_ch) == g.GDN2_GATES_PER_CHANNEL
    assert g._gate_layout(q, tok, tok, per_ch) == g.GDN2_ERASE_SCALAR | g.GDN2_WRITE_SCALAR
    assert g._gate_layout(q, tok, tok, tok) == 7
    assert g._gate_layout(q, per_ch, tok, per_ch) == g.GDN2_WRITE_SCALAR


def test_layer_fwd_rejects_bad_arguments(lib):
    import ctypes as ct
    f = lambda **kw: lib.gdn2_layer_fwd(P, P, P, P, P, P, kw.get("g", P), kw.get("nw", P),
                                        ct.c_float(kw.get("eps", 1e-6)), None, P, None,
                                        1, 8, 2, 64, 64, 1, None)
    assert f(g=None) == g.GDN2_ERR_NULL
    assert f(nw=None) == g.GDN2_ERR_NULL
    assert f(g=MIS) == g.GDN2_ERR_ALIGN
    assert f(eps=-1.0) == g.GDN2_ERR_SHAPE


def test_bwd_rejects_bad_arguments(lib):
    f = lambda **kw: lib.gdn2_bwd_chunked(P, P, P, P, P, P, None, kw.get("dO", P), None, P, P, P, P, P,
                                          kw.get("dla", P), None, kw.get("B", 1), 8, 2, kw.get("dk", 64), 64,
                                          kw.get("dtype", 1), None)
    assert f(dO=None) == g.GDN2_ERR_NULL
    assert f(dla=MIS) == g.GDN2_ERR_ALIGN
    assert f(B=0) == g.GDN2_ERR_SHAPE
    assert f(dk=32) == g.GDN2_ERR_UNSUPPORTED
    assert f(dtype=9) == g.GDN2_ERR_DTYPE
