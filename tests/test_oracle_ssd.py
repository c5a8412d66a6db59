"""Runs the pins of the scalar-identity (Mamba-2) oracle, and checks that a
pin catches each of a set of plausible mistakes planted in a copy of the C
source (CPU)."""
import os

import pytest

import oracle
from tests import oracle_ssd_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "oracle_ssm.c")


@pytest.mark.parametrize("pin", pins.PINS, ids=lambda f: f.__name__)
def test_ssd_oracle_pin(pin):
    pin()


# (what, original text, planted text) inside oracle_ssd_scan_f64
MUTATIONS = [
    ("decay sign", "const double decay = exp(dv * A[hd]);", "const double decay = exp(-dv * A[hd]);"),
    ("decay per channel index", "const double decay = exp(dv * A[hd]);",
     "const double decay = exp(dv * A[p % nheads]);"),
    ("no Delta on the input", "h[n] = decay * h[n] + dv * Bt[n] * x[i];",
     "h[n] = decay * h[n] + Bt[n] * x[i];"),
    ("readout before update", "h[n] = decay * h[n] + dv * Bt[n] * x[i];\n                        y += Ct[n] * h[n];",
     "y += Ct[n] * h[n];\n                        h[n] = decay * h[n] + dv * Bt[n] * x[i];"),
    ("B for C", "y += Ct[n] * h[n];", "y += Bt[n] * h[n];"),
    ("dropped skip", "y += (D ? D[d] : 0.0) * x[i];", "y += 0.0;"),
    ("wrong head of delta", "delta[(b * seqlen + t) * nheads + hd]",
     "delta[(b * seqlen + t) * nheads + (nheads - 1 - hd)]"),
    ("gate before skip", "y += (D ? D[d] : 0.0) * x[i];\n                    out[i] = y * oracle_silu(z[i]);",
     "out[i] = y * oracle_silu(z[i]) + (D ? D[d] : 0.0) * x[i];"),
]


@pytest.mark.parametrize("what,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_a_pin_catches_planted_mistake(tmp_path, what, old, new):
    src = open(SRC).read()
    body = src[src.index("int oracle_ssd_scan_f64"):]
    assert body.count(old) == 1, what
    mutated = src[:src.index("int oracle_ssd_scan_f64")] + body.replace(old, new)
    path = tmp_path / "mut.c"
    path.write_text(mutated)
    so = str(tmp_path / "libmut.so")
    oracle.build(str(path), so)
    lib = oracle.load(so)
    orig = oracle.ssd_scan

    def patched(*a, **k):
        k["lib"] = lib
        return orig(*a, **k)
    failed = False
    try:
        oracle.ssd_scan = patched
        for pin in pins.PINS:
            try:
                pin()
            except AssertionError:
                failed = True
                break
    finally:
        oracle.ssd_scan = orig
    assert failed, f"no pin caught the planted mistake: {what}"

