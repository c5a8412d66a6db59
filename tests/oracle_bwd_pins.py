"""Pins of the oracle's reverse-mode gradient of the scan (the layer's backward
pass) against facts that do not come from the gradient code:

  * central finite differences of the forward oracle (itself pinned by
    tests/oracle_pins.py): every element of every gradient, on tiny problems
    with softplus on and off, with and without D, bias and h0;
  * closed forms of the state gradient: with dL/dout = 0 and dL/dh_final a
    one-hot e_n, unrolling the linear recurrence gives
        dL/dh0[n]   = exp(A[n] * sum_t Delta_t),
        dL/dB[t, n] = exp(A[n] * sum_{s>t} Delta_s) * Delta_t * x_t,
    with Delta computed here by numpy's logaddexp (softplus);
  * causality: a loss on out_s alone has no gradient through steps t > s;
  * linearity of the gradient in (dL/dout, dL/dh_final).
The same functions run against broken copies of the oracle in
test_oracle_bwd.py, which checks that every planted mistake trips one.

The method is the S6 recurrence of "Jamba: A Hybrid Transformer-Mamba Language
Model" (obsidian-dorae222 notes), section "Mamba 레이어"; its gradient is the
chain rule applied to that recurrence in reverse time.
"""
from __future__ import annotations

import numpy as np

import oracle
from tests.oracle_pins import _tiny_case

_GRAD_NAME = {"x": "dx", "delta": "ddelta", "z": "dz", "B": "dB", "C": "dC", "A": "dA",
              "D": "dD", "delta_bias": "ddelta_bias", "h0": "dh0"}


def _loss(case, dout, dh_final, lib):
    out, hf = oracle.scan(lib=lib, **case)
    return float(np.sum(out * dout) + np.sum(hf * dh_final))


def pin_bwd_finite_differences(lib):
    for seed, softplus in ((41, True), (42, False)):
        case = _tiny_case(seed, batch=2, seqlen=6, d_inner=3, d_state=3)
        case["delta_softplus"] = softplus
        if not softplus:  # keep Delta positive and moderate without the softplus
            case["delta"] = np.abs(case["delta"]) * 0.3
            case["delta_bias"] = np.abs(case["delta_bias"]) * 0.1
        r = np.random.default_rng(seed)
        out, hf = oracle.scan(lib=lib, **case)
        dout, dhf = r.standard_normal(out.shape), r.standard_normal(hf.shape)
        g = oracle.scan_bwd(dout=dout, dh_final=dhf, lib=lib, **case)
        eps = 1e-6
        for name, gname in _GRAD_NAME.items():
            base = case[name]
            for idx in np.ndindex(base.shape):
                a = base.copy()
                a[idx] += eps
                lp = _loss(dict(case, **{name: a}), dout, dhf, lib)
                a[idx] -= 2 * eps
                lm = _loss(dict(case, **{name: a}), dout, dhf, lib)
                fd = (lp - lm) / (2 * eps)
                got = g[gname][idx]
                assert abs(fd - got) <= 2e-6 * max(1.0, abs(fd)), \
                    f"d{name}{idx}: finite difference {fd:.9g}, gradient {got:.9g}"


def pin_bwd_state_closed_form(lib):
    case = _tiny_case(43, batch=1, seqlen=7, d_inner=2, d_state=3)
    delta = np.logaddexp(0.0, case["delta"] + case["delta_bias"])  # softplus, [1, L, d]
    for d in range(2):
        for n in range(3):
            dhf = np.zeros((1, 2, 3))
            dhf[0, d, n] = 1.0
            g = oracle.scan_bwd(dout=np.zeros_like(case["x"]), dh_final=dhf, lib=lib, **case)
            a_n = case["A"][d, n]
            want_h0 = np.zeros((1, 2, 3))
            want_h0[0, d, n] = np.exp(a_n * delta[0, :, d].sum())
            assert np.allclose(g["dh0"], want_h0, rtol=1e-13, atol=0), "dh0 closed form"
            for t in range(7):
                tail = delta[0, t + 1:, d].sum()
                want = np.exp(a_n * tail) * delta[0, t, d] * case["x"][0, t, d]
                got = g["dB"][0, t]
                assert abs(got[n] - want) <= 1e-13 * max(1.0, abs(want)), f"dB[{t},{n}]"
                assert np.all(np.delete(got, n) == 0.0), "dB leaks into other states"


def pin_bwd_causality_and_linearity(lib):
    case = _tiny_case(44, batch=2, seqlen=8, d_inner=3, d_state=4)
    r = np.random.default_rng(44)
    s = 3
    dout = np.zeros_like(case["x"])
    dout[:, s] = r.standard_normal(dout[:, s].shape)
    g = oracle.scan_bwd(dout=dout, lib=lib, **case)
    for k in ("dx", "ddelta", "dz", "dB", "dC"):
        assert np.all(g[k][:, s + 1:] == 0.0), f"{k} reaches past step {s}"
    assert np.any(g["dx"][:, s] != 0.0)
    d1, d2 = r.standard_normal(case["x"].shape), r.standard_normal(case["x"].shape)
    h1, h2 = r.standard_normal((2, 3, 4)), r.standard_normal((2, 3, 4))
    g1 = oracle.scan_bwd(dout=d1, dh_final=h1, lib=lib, **case)
    g2 = oracle.scan_bwd(dout=d2, dh_final=h2, lib=lib, **case)
    g12 = oracle.scan_bwd(dout=2.0 * d1 - 0.5 * d2, dh_final=2.0 * h1 - 0.5 * h2, lib=lib, **case)
    for k in g12:
        want = 2.0 * g1[k] - 0.5 * g2[k]
        assert np.allclose(g12[k], want, rtol=1e-12, atol=1e-12 * np.abs(want).max()), k


BWD_PINS = [pin_bwd_finite_differences, pin_bwd_state_closed_form,
            pin_bwd_causality_and_linearity]
