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


# Mistakes planted in the backward (gdn2_oracle_bwd), caught by the backward's pins.
BWD_MUTATIONS = {
    "bwd_erase_read_adjoint_dropped": ("dS[(long)i * dv + j] -= e[i] * du[j];", ""),
    "bwd_decay_gradient_on_updated_state": ("acc += dS[(long)i * dv + j] * Sbar[(long)i * dv + j];",
                                            "acc += dS[(long)i * dv + j] * cur[(long)i * dv + j];"),
    "bwd_write_gate_and_value_swapped": ("dw[rv + j] = du[j] * v[rv + j]; dval[rv + j] = du[j] * w[rv + j];",
                                         "dw[rv + j] = du[j] * w[rv + j]; dval[rv + j] = du[j] * v[rv + j];"),
    "bwd_erase_gate_left_out_of_key_gradient": ("dkey[rk + i] = dkv[i] + de[i] * b[rk + i];",
                                                "dkey[rk + i] = dkv[i] + de[i];"),
    "bwd_query_gradient_from_old_state": ("acc += cur[(long)i * dv + j] * dO[rv + j];",
                                          "acc += prev[(long)i * dv + j] * dO[rv + j];"),
}

SPLIT = "int gdn2_oracle_bwd("


def _mutant(tmp_path, before, after, backward):
    src = oracle.SOURCE.read_text()
    fwd, bwd = src.split(SPLIT)
    part = bwd if backward else fwd
    assert part.count(before) == 1, f"mutation anchor {before!r} not found exactly once"
    part = part.replace(before, after)
    mutated = tmp_path / "oracle_mutant.c"
    mutated.write_text((fwd + SPLIT + part) if backward else (part + SPLIT + bwd))
    return oracle.compile_oracle(mutated, tmp_path / "liboracle_mutant.so")


@pytest.mark.parametrize("name", sorted(BWD_MUTATIONS))
def test_planted_backward_mistake_is_caught(name, tmp_path, monkeypatch):
    import test_oracle_bwd_pins as pins
    before, after = BWD_MUTATIONS[name]
    monkeypatch.setattr(oracle, "_default", oracle.load(_mutant(tmp_path, before, after, backward=True)))
    checks = [lambda: pins.test_every_gradient_matches_central_differences(9),
              pins.test_pure_decay_closed_form, pins.test_kda_reduction_of_the_gate_gradients]
    caught = 0
    for check in checks:
        try:
            check()
        except AssertionError:
            caught += 1
    assert caught, f"no backward pin catches the planted mistake '{name}'"


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name, tmp_path):
    before, after = MUTATIONS[name]
    orc = oracle.load(_mutant(tmp_path, before, after, backward=False))
    caught = []
    for pin in ALL_PINS:
        try:
            pin(orc)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"no pin catches the planted mistake '{name}'"
