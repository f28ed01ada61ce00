"""Each plausible mistake planted in a copy of the oracle fails at least one pin.

The copies are made from ``oracle/gdn2_oracle.c`` by text substitution, built
with gcc into a temporary directory and run on the CPU.  The oracle itself is
never modified.
"""
import pytest

import oracle
from oracle_pins import ALL_PINS

MUTATIONS = {
    "decay_dropped": ("alpha[i] = exp(log_alpha[rk + i]);", "alpha[i] = 1.0;"),
    "decay_not_exponentiated": ("alpha[i] = exp(log_alpha[rk + i]);", "alpha[i] = log_alpha[rk + i];"),
    "erase_gate_dropped": ("e[i] = b[rk + i] * k[rk + i];", "e[i] = k[rk + i];"),
    "write_gate_dropped": ("z[j] = w[rv + j] * v[rv + j];", "z[j] = v[rv + j];"),
    "update_sign_flipped": ("+= ki * (z[j] - r[j]);", "+= ki * (r[j] - z[j]);"),
    "read_before_decay": ("acc += S[(long)i * dv + j] * e[i];",
                          "acc += S[(long)i * dv + j] * e[i] / alpha[i];"),
    "read_with_key_not_erase": ("acc += S[(long)i * dv + j] * e[i];",
                                "acc += S[(long)i * dv + j] * k[rk + i];"),
    "write_along_erase_key": ("const double ki = k[rk + i];", "const double ki = e[i];"),
    "query_reads_old_state": ("acc += S[(long)i * dv + j] * q[rk + i];",
                              "acc += (S[(long)i * dv + j] - k[rk + i] * (z[j] - r[j])) * q[rk + i];"),
    "output_reads_key": ("acc += S[(long)i * dv + j] * q[rk + i];",
                         "acc += S[(long)i * dv + j] * k[rk + i];"),
    "initial_state_ignored": ("S[i] = s0 ? s0[i] : 0.0;", "S[i] = 0.0;"),
    "layout_head_major": ("const long rk = ((bi * T + t) * H + hi) * dk;",
                          "const long rk = ((bi * H + hi) * T + t) * dk;"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name, tmp_path):
    before, after = MUTATIONS[name]
    src = oracle.SOURCE.read_text()
    assert src.count(before) == 1, f"mutation anchor for {name} not found exactly once"
    mutated = tmp_path / "oracle_mutant.c"
    mutated.write_text(src.replace(before, after))
    lib = oracle.compile_oracle(mutated, tmp_path / "liboracle_mutant.so")
    orc = oracle.load(lib)
    caught = []
    for pin in ALL_PINS:
        try:
            pin(orc)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"no pin catches the planted mistake '{name}'"
