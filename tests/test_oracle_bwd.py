"""The oracle's backward scan against its pins, and planted mistakes in a copy
of it that the pins must catch (CPU only; the oracle source in the repo is
never modified)."""
import os

import pytest

import oracle
from tests.oracle_bwd_pins import BWD_PINS

SRC = os.path.join(os.path.dirname(oracle.__file__), "oracle_ssm.c")


@pytest.mark.parametrize("pin", BWD_PINS, ids=lambda f: f.__name__)
def test_oracle_bwd_pin(pin, oracle_lib):
    pin(oracle_lib)


# (name, exact text in the oracle's backward function, replacement)
MUTATIONS = [
    ("carry_not_decayed", "g[n] = abar * g[n];", "g[n] = g[n];"),
    ("silu_derivative", "sz * (1.0 + z[i] * (1.0 - sz))", "sz * (1.0 - z[i] * sz)"),
    ("softplus_derivative_dropped", "dDelta / (1.0 + exp(-v))", "dDelta"),
    ("dA_without_delta", "dA[d * d_state + n] += dabar * abar * dv;",
     "dA[d * d_state + n] += dabar * abar;"),
    ("dB_without_x", "dBt[n] += g[n] * dv * xv;", "dBt[n] += g[n] * dv;"),
    ("dC_from_previous_state", "dCt[n] += dy * h_now[n];", "dCt[n] += dy * h_prev[n];"),
    ("readout_gradient_through_B", "g[n] += dy * Ct[n];", "g[n] += dy * Bt[n];"),
    ("decay_term_of_dDelta_dropped", "dDelta += dabar * abar * an + g[n] * Bt[n] * xv;",
     "dDelta += g[n] * Bt[n] * xv;"),
    ("gate_gradient_without_gate", "double dy = dout[i] * (z[i] * sz);", "double dy = dout[i];"),
    ("skip_gradient_dropped", "double dxi = dy * Dd, dDelta = 0.0;",
     "double dxi = 0.0, dDelta = 0.0;"),
    ("dh_final_ignored", "g[n] = dh_final ? dh_final[(b * d_inner + d) * d_state + n] : 0.0;",
     "g[n] = 0.0;"),
]


@pytest.mark.parametrize("name,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_bwd_pins_catch_planted_mistake(name, old, new, tmp_path):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} is not unique in the oracle"
    path = tmp_path / "mutant.c"
    path.write_text(src.replace(old, new, 1))
    lib = oracle.load(oracle.build(str(path), str(tmp_path / "libmutant.so")))
    caught = []
    for pin in BWD_PINS:
        try:
            pin(lib)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"no pin notices the planted mistake {name!r}"
