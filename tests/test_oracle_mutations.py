"""Plant plausible mistakes in a copy of the oracle and check that the pins
catch every one (CPU only; the oracle source in the repo is never modified).

Each mutation rewrites one expression of oracle/oracle_ssm.c in a temporary
copy, builds it with gcc, and runs every pin against the broken library.  A
mutation that no pin notices would mean the pins leave that part of the
oracle unchecked.
"""
import os

import pytest

import oracle
from tests.oracle_pins import ALL_PINS

SRC = os.path.join(os.path.dirname(oracle.__file__), "oracle_ssm.c")

# (name, exact text in the oracle, replacement): each is a plausible slip.
MUTATIONS = [
    ("drop_skip", "double skip = D ? D[d] * xv : 0.0;", "double skip = 0.0;"),
    ("sign_of_decay", "exp(dv * A[d * d_state + n])", "exp(-dv * A[d * d_state + n])"),
    ("B_for_C_in_readout", "y += Ct[n] * h[n];", "y += Bt[n] * h[n];"),
    ("readout_before_update",
     "h[n] = abar * h[n] + bbar_x;\n                    y += Ct[n] * h[n];",
     "y += Ct[n] * h[n];\n                    h[n] = abar * h[n] + bbar_x;"),
    ("softplus_without_log", "return log1p(exp(v));", "return exp(v);"),
    ("gate_sign", "return z / (1.0 + exp(-z));", "return z / (1.0 + exp(z));"),
    ("bias_dropped", "double v = raw + (delta_bias ? delta_bias[d] : 0.0);", "double v = raw;"),
    ("state_index_reversed", "exp(dv * A[d * d_state + n])",
     "exp(dv * A[d * d_state + (d_state - 1 - n)])"),
    ("h0_ignored", "h[n] = h0 ? h0[(b * d_inner + d) * d_state + n] : 0.0;", "h[n] = 0.0;"),
    ("B_one_step_late", "const double *Bt = B + (b * seqlen + t) * d_state;",
     "const double *Bt = B + (b * seqlen + (t > 0 ? t - 1 : t)) * d_state;"),
    ("x_missing_from_input", "double bbar_x = dv * Bt[n] * xv;", "double bbar_x = dv * Bt[n];"),
    ("delta_missing_from_input", "double bbar_x = dv * Bt[n] * xv;",
     "double bbar_x = Bt[n] * xv;"),
    ("gate_before_skip", "out[i] = (y + skip) * oracle_silu(z[i]);",
     "out[i] = y * oracle_silu(z[i]) + skip;"),
]


@pytest.mark.parametrize("name,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_pins_catch_planted_mistake(name, old, new, tmp_path):
    src = open(SRC).read()
    assert old in src, f"mutation anchor for {name} not found in the oracle"
    mutated = src.replace(old, new, 1)
    path = tmp_path / "mutant.c"
    path.write_text(mutated)
    lib = oracle.load(oracle.build(str(path), str(tmp_path / "libmutant.so")))
    caught = []
    for pin in ALL_PINS:
        try:
            pin(lib)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"no pin notices the planted mistake {name!r}"
