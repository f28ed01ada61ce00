"""The chunkwise WY algebra used by the kernels equals the token recurrence."""
import numpy as np
import pytest

import oracle
from oracle_pins import _inputs
from wy_model import wy_forward


@pytest.mark.parametrize("C", [1, 2, 4, 16, 64])
def test_wy_model_matches_oracle(C):
    q, k, v, b, w, la, s0 = _inputs(150, 8, 6, seed=200 + C, B=1, H=2)
    o_ref, s_ref = oracle.fwd(q, k, v, b, w, la, S0=s0)
    o, s = wy_forward(q, k, v, b, w, la, S0=s0, C=C)
    scale = np.abs(o_ref).max()
    assert np.abs(o - o_ref).max() <= 1e-12 * scale
    assert np.abs(s - s_ref).max() <= 1e-12 * np.abs(s_ref).max()


def test_wy_model_strong_decay_and_wide_erase():
    """Long-context decay range (log alpha down to -1) and erase gates in [0, 2]."""
    r = np.random.default_rng(7)
    q, k, v, b, w, _, s0 = _inputs(200, 16, 8, seed=8)
    la = -np.exp(r.uniform(-9.0, 0.0, q.shape))
    o_ref, s_ref = oracle.fwd(q, k, v, 2 * b, w, la, S0=s0)
    o, s = wy_forward(q, k, v, 2 * b, w, la, S0=s0, C=64)
    assert np.abs(o - o_ref).max() <= 1e-11 * np.abs(o_ref).max()
    assert np.abs(s - s_ref).max() <= 1e-11 * np.abs(s_ref).max()


@pytest.mark.parametrize("C,T", [(4, 37), (8, 64), (16, 150), (64, 200)])
def test_pair_composition_matches_oracle(C, T):
    """Two chunk records composed into one state map (the form the persistent
    forward's chain steps over) equal the token recurrence; an odd last chunk
    (T = 37 with C = 4: ten chunks, T = 150 with C = 16: ten, T = 200 with C = 64: four)
    and a lone pair (T = 64 with C = 8: eight chunks)."""
    from wy_model import wy_forward_pairs
    q, k, v, b, w, la, s0 = _inputs(T, 8, 6, seed=300 + C, B=1, H=2)
    o_ref, s_ref = oracle.fwd(q, k, v, b, w, la, S0=s0)
    o, s = wy_forward_pairs(q, k, v, b, w, la, S0=s0, C=C)
    assert np.abs(o - o_ref).max() <= 1e-11 * np.abs(o_ref).max()
    assert np.abs(s - s_ref).max() <= 1e-11 * np.abs(s_ref).max()


def test_pair_composition_odd_chunk_count():
    """Three chunks: one composed pair and a lone last chunk."""
    from wy_model import wy_forward_pairs
    q, k, v, b, w, la, s0 = _inputs(40, 8, 6, seed=401, B=1, H=1)
    o_ref, s_ref = oracle.fwd(q, k, v, b, w, la, S0=s0)
    o, s = wy_forward_pairs(q, k, v, b, w, la, S0=s0, C=16)
    assert np.abs(o - o_ref).max() <= 1e-11 * np.abs(o_ref).max()
    assert np.abs(s - s_ref).max() <= 1e-11 * np.abs(s_ref).max()


@pytest.mark.parametrize("m,C,T", [(2, 16, 150), (3, 16, 150), (4, 64, 200), (8, 8, 100), (5, 4, 37)])
def test_group_composition_matches_oracle(m, C, T):
    """m chunk records composed into one state map per step of the chain (the
    chain then takes one step per m chunks), each chunk's entry state from its
    group's by the prefix of the composed product; ragged last groups and
    chunks."""
    from wy_model import group_forward
    q, k, v, b, w, la, s0 = _inputs(T, 8, 6, seed=400 + m * C, B=1, H=2)
    o_ref, s_ref = oracle.fwd(q, k, v, b, w, la, S0=s0)
    o, s = group_forward(q, k, v, b, w, la, S0=s0, C=C, m=m)
    assert np.abs(o - o_ref).max() <= 1e-12 * np.abs(o_ref).max()
    assert np.abs(s - s_ref).max() <= 1e-12 * np.abs(s_ref).max()
