"""The fp64 oracle against what the pages and the mathematics fix (CPU only)."""
import pytest

import oracle
from oracle_pins import ALL_PINS


@pytest.mark.parametrize("pin", ALL_PINS, ids=[p.__name__ for p in ALL_PINS])
def test_oracle_pin(pin):
    pin(oracle.load())


def test_oracle_threads_agree():
    """OpenMP over (batch, head) pairs does not change any value."""
    import numpy as np
    from oracle_pins import _inputs
    q, k, v, b, w, la, s0 = _inputs(9, 6, 5, seed=5, B=3, H=4)
    o1, s1 = oracle.fwd(q, k, v, b, w, la, S0=s0, nthreads=1)
    o4, s4 = oracle.fwd(q, k, v, b, w, la, S0=s0, nthreads=4)
    assert np.array_equal(o1, o4) and np.array_equal(s1, s4)


def test_oracle_zero_length_sequence():
    """T = 0: no output rows, and the state passes through unchanged."""
    import numpy as np
    from oracle_pins import _inputs
    q, k, v, b, w, la, s0 = _inputs(0, 4, 3, seed=6, B=2, H=2)
    o, st = oracle.fwd(q, k, v, b, w, la, S0=s0)
    assert o.shape == (2, 0, 2, 3)
    assert np.array_equal(st, s0)
