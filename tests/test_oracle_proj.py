"""The oracle's projection step against its pins, and planted mistakes in a
copy of it that the pins must catch (CPU only; the oracle source in the repo is
never modified)."""
import os

import pytest

import oracle
from tests.oracle_proj_pins import PROJ_PINS

SRC = os.path.join(os.path.dirname(oracle.__file__), "oracle_ssm.c")


@pytest.mark.parametrize("pin", PROJ_PINS, ids=lambda f: f.__name__)
def test_oracle_proj_pin(pin, oracle_lib):
    pin(oracle_lib)


# (name, exact text in the oracle, replacement): each is a plausible slip.
MUTATIONS = [
    ("B_C_swapped", "*Bv = xdbl + dt_rank, *Cv = xdbl + dt_rank + d_state;",
     "*Bv = xdbl + dt_rank + d_state, *Cv = xdbl + dt_rank;"),
    ("B_slice_off_by_one", "*Bv = xdbl + dt_rank, *Cv", "*Bv = xdbl + dt_rank - 1, *Cv"),
    ("W_x_transposed", "acc += W_x[j * d_inner + k] * ut[k];",
     "acc += W_x[k * rows + j] * ut[k];"),
    ("W_dt_transposed", "acc += W_dt[d * dt_rank + r] * dt_low[r];",
     "acc += W_dt[r * d_inner + d] * dt_low[r];"),
    ("norm_sum_not_mean", "double inv = 1.0 / sqrt(ss / (double)len + eps);",
     "double inv = 1.0 / sqrt(ss + eps);"),
    ("norm_eps_dropped", "double inv = 1.0 / sqrt(ss / (double)len + eps);",
     "double inv = 1.0 / sqrt(ss / (double)len);"),
    ("norm_weight_ignored", "v[i] = w[i] * (v[i] * inv);", "v[i] = v[i] * inv;"),
    ("B_normed_with_C_weights", "oracle_rmsnorm(Bv, d_state, w_B, eps);",
     "oracle_rmsnorm(Bv, d_state, w_C, eps);"),
    ("norm_without_sqrt", "double inv = 1.0 / sqrt(ss / (double)len + eps);",
     "double inv = 1.0 / (ss / (double)len + eps);"),
    ("dt_low_slice_off_by_one",
     "oracle_low_rank_row(d_inner, dt_rank, W_dt, dt_low, delta + t * d_inner);",
     "oracle_low_rank_row(d_inner, dt_rank, W_dt, xdbl + 1, delta + t * d_inner);"),
    ("dt_proj_last_token_dropped",
     "for (int64_t t = t_lo; t < t_hi; ++t)\n        oracle_low_rank_row",
     "for (int64_t t = t_lo; t + 1 < t_hi; ++t)\n        oracle_low_rank_row"),
]


@pytest.mark.parametrize("name,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_proj_pins_catch_planted_mistake(name, old, new, tmp_path):
    src = open(SRC).read()
    assert old in src, f"mutation anchor for {name} not found in the oracle"
    path = tmp_path / "mutant.c"
    path.write_text(src.replace(old, new, 1))
    lib = oracle.load(oracle.build(str(path), str(tmp_path / "libmutant.so")))
    caught = []
    for pin in PROJ_PINS:
        try:
            pin(lib)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"no pin notices the planted mistake {name!r}"
