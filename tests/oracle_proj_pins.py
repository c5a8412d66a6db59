"""Pins of the oracle's projection step (Delta, B, C from the scan's input)
against facts that do not come from the oracle.

Without normalisation the step is linear in u, in W_x and in W_dt, and a linear
map is fixed by what it does to basis vectors; so the pins check
  * linearity in each of the three operands, and
  * that basis inputs select the entries the definition names: token u = e_k
    gives B = column k of W_x's B rows and C = column k of its C rows, and a
    single-entry W_x = E_{r,k} with u = e_k gives delta = column r of W_dt;
  * that delta has rank at most dt_rank over any set of tokens (the low-rank
    form of the step), with or without the RMSNorm on dt_low;
  * the RMSNorm by closed forms: a vector of equal-magnitude entries +-a maps to
    +-a / sqrt(a^2 + eps) times the weight, unit weights give unit RMS when
    eps = 0, and the result does not change when its input is scaled.
Each part is normalised over its own length (dt_rank differs from d_state in
every case here, so a norm over the wrong length shows).

The same functions run against broken copies of the oracle in
test_oracle_proj.py, which checks that every planted mistake trips one.

Source of the step: "Jamba: A Hybrid Transformer-Mamba Language Model"
(obsidian-dorae222 notes), section "Mamba 레이어": Bbar_t, C_t and Delta_t are
functions of x_t, and the Mamba layer carries an RMSNorm.
"""
from __future__ import annotations

import numpy as np

import oracle


def _rng(seed):
    return np.random.default_rng(seed)


def _weights(r, d_inner, dt_rank, d_state):
    return (r.standard_normal((dt_rank + 2 * d_state, d_inner)),
            r.standard_normal((d_inner, dt_rank)))


def _close(a, b, tol, what):
    err = float(np.max(np.abs(np.asarray(a) - np.asarray(b))))
    scale = max(1.0, float(np.max(np.abs(b))))
    assert err <= tol * scale, f"{what}: max |diff| {err:.3e} > {tol:.1e} * {scale:.3e}"


def pin_proj_basis_selection(lib):
    d_inner, dt_rank, d_state = 7, 3, 2
    r = _rng(11)
    W_x, W_dt = _weights(r, d_inner, dt_rank, d_state)
    eye = np.eye(d_inner)
    delta, B, C = oracle.project(eye, W_x, W_dt, d_state, lib=lib)
    for k in range(d_inner):
        assert np.array_equal(B[k], W_x[dt_rank:dt_rank + d_state, k]), "B of e_k"
        assert np.array_equal(C[k], W_x[dt_rank + d_state:, k]), "C of e_k"
    for rr in range(dt_rank):
        for k in (0, d_inner - 1, rr + 2):
            E = np.zeros_like(W_x)
            E[rr, k] = 1.0
            d1, _, _ = oracle.project(eye[k:k + 1], E, W_dt, d_state, lib=lib)
            assert np.array_equal(d1[0], W_dt[:, rr]), f"delta of E_({rr},{k}) e_{k}"


def pin_proj_linearity(lib):
    d_inner, dt_rank, d_state = 9, 4, 3
    r = _rng(12)
    W_x, W_dt = _weights(r, d_inner, dt_rank, d_state)
    u1, u2 = r.standard_normal((5, d_inner)), r.standard_normal((5, d_inner))
    a, b = 0.75, -1.5
    f = lambda u, wx=W_x, wdt=W_dt: oracle.project(u, wx, wdt, d_state, lib=lib)
    for what, lhs, rhs1, rhs2 in (
            ("u", f(a * u1 + b * u2), f(u1), f(u2)),
            ("W_x", f(u1, wx=a * W_x + b * W_x[::-1]), f(u1, wx=W_x), f(u1, wx=W_x[::-1])),
            ("W_dt", f(u1, wdt=a * W_dt + b * W_dt[::-1]), f(u1, wdt=W_dt),
             f(u1, wdt=W_dt[::-1]))):
        for name, l, p, q in zip(("delta", "B", "C"), lhs, rhs1, rhs2):
            if what == "W_dt" and name != "delta":
                _close(l, p, 1e-13, f"{name} does not depend on W_dt")
            else:
                _close(l, a * p + b * q, 1e-12, f"{name} linear in {what}")


def pin_proj_low_rank(lib):
    d_inner, dt_rank, d_state, ntok = 24, 3, 4, 40
    r = _rng(13)
    W_x, W_dt = _weights(r, d_inner, dt_rank, d_state)
    u = r.standard_normal((ntok, d_inner))
    for w_dt in (None, r.uniform(0.5, 1.5, dt_rank)):
        delta, _, _ = oracle.project(u, W_x, W_dt, d_state, w_dt=w_dt, lib=lib)
        s = np.linalg.svd(delta, compute_uv=False)
        assert s[dt_rank - 1] > 1e-3 * s[0], "delta should have rank dt_rank"
        assert s[dt_rank] <= 1e-12 * s[0], f"delta has rank above dt_rank: {s[:dt_rank + 2]}"


def _identity_case(dt_rank, d_state):
    """d_inner = dt_rank + 2 d_state with W_x = I, so xdbl is the token itself,
    and W_dt = [I; 0], so delta's first dt_rank channels are dt_low."""
    d_inner = dt_rank + 2 * d_state
    W_dt = np.zeros((d_inner, dt_rank))
    W_dt[:dt_rank] = np.eye(dt_rank)
    return d_inner, np.eye(d_inner), W_dt


def pin_proj_rmsnorm_closed_forms(lib):
    dt_rank, d_state = 5, 3
    d_inner, W_x, W_dt = _identity_case(dt_rank, d_state)
    r = _rng(14)
    signs = np.where(r.random((4, d_inner)) < 0.5, -1.0, 1.0)
    w_dt, w_B, w_C = (r.uniform(0.5, 2.0, n) for n in (dt_rank, d_state, d_state))
    for a, eps in ((1e-3, 1e-6), (0.5, 0.0), (2.0, 1e-2)):
        u = a * signs
        delta, B, C = oracle.project(u, W_x, W_dt, d_state, w_dt=w_dt, w_B=w_B, w_C=w_C,
                                     eps=eps, lib=lib)
        k = a / np.sqrt(a * a + eps)
        _close(delta[:, :dt_rank], k * signs[:, :dt_rank] * w_dt, 1e-14, "norm of dt_low")
        _close(B, k * signs[:, dt_rank:dt_rank + d_state] * w_B, 1e-14, "norm of B")
        _close(C, k * signs[:, dt_rank + d_state:] * w_C, 1e-14, "norm of C")
    ones = [np.ones(n) for n in (dt_rank, d_state, d_state)]
    u = r.standard_normal((6, d_inner))
    parts = oracle.project(u, W_x, W_dt, d_state, *ones, eps=0.0, lib=lib)
    parts2 = oracle.project(37.0 * u, W_x, W_dt, d_state, *ones, eps=0.0, lib=lib)
    for name, p, p2 in zip(("dt_low", "B", "C"), parts, parts2):
        p = p[:, :dt_rank] if name == "dt_low" else p
        p2 = p2[:, :dt_rank] if name == "dt_low" else p2
        _close(np.mean(p * p, axis=1), np.ones(len(p)), 1e-14, f"unit RMS of {name}")
        _close(p2, p, 1e-14, f"scale invariance of {name}")


def pin_proj_norm_off_is_plain(lib):
    """With no weights the step takes no normalisation: basis selection and a
    token of all zeros (mapped to all zeros) hold exactly."""
    dt_rank, d_state = 2, 3
    d_inner, W_x, W_dt = _identity_case(dt_rank, d_state)
    u = _rng(15).standard_normal((3, d_inner))
    delta, B, C = oracle.project(u, W_x, W_dt, d_state, lib=lib)
    assert np.array_equal(delta[:, :dt_rank], u[:, :dt_rank])
    assert np.array_equal(B, u[:, dt_rank:dt_rank + d_state])
    assert np.array_equal(C, u[:, dt_rank + d_state:])
    z = oracle.project(np.zeros((1, d_inner)), W_x, W_dt, d_state, eps=1e-6,
                       w_dt=np.ones(dt_rank), w_B=np.ones(d_state), w_C=np.ones(d_state),
                       lib=lib)
    for p in z:
        assert np.array_equal(p, np.zeros_like(p)), "zero token with eps > 0"


def pin_dt_proj_alone(lib):
    """The last product on its own: one-hot rows of dt_low select the columns
    of W_dt, the product is linear in dt_low, and it is the delta of the whole
    step when W_x's first R rows are [I_R 0] and no norm is taken."""
    d_inner, dt_rank, d_state = 11, 4, 2
    r = _rng(16)
    W_x, W_dt = _weights(r, d_inner, dt_rank, d_state)
    delta = oracle.dt_proj(np.eye(dt_rank), W_dt, lib=lib)
    for k in range(dt_rank):
        assert np.array_equal(delta[k], W_dt[:, k]), f"dt_proj of e_{k}"
    v1, v2 = r.standard_normal((6, dt_rank)), r.standard_normal((6, dt_rank))
    _close(oracle.dt_proj(0.5 * v1 - 2.0 * v2, W_dt, lib=lib),
           0.5 * oracle.dt_proj(v1, W_dt, lib=lib) - 2.0 * oracle.dt_proj(v2, W_dt, lib=lib),
           1e-12, "dt_proj linear in dt_low")
    W_x[:dt_rank] = 0.0
    W_x[:dt_rank, :dt_rank] = np.eye(dt_rank)
    u = r.standard_normal((5, d_inner))
    d_full, _, _ = oracle.project(u, W_x, W_dt, d_state, lib=lib)
    assert np.array_equal(d_full, oracle.dt_proj(u[:, :dt_rank], W_dt, lib=lib)), \
        "dt_proj is the last product of the step"


def pin_proj_dt_low_output(lib):
    """The dt_low the step returns is the one its delta was made from
    (delta == dt_proj(dt_low)); without a norm a one-hot token selects column k
    of W_x's first R rows; with unit weights and eps = 0 its RMS is 1."""
    d_inner, dt_rank, d_state = 10, 4, 3
    r = _rng(17)
    W_x, W_dt = _weights(r, d_inner, dt_rank, d_state)
    _, _, _, low = oracle.project(np.eye(d_inner), W_x, W_dt, d_state, return_dt_low=True,
                                  lib=lib)
    for k in range(d_inner):
        assert np.array_equal(low[k], W_x[:dt_rank, k]), f"dt_low of e_{k}"
    u = r.standard_normal((7, d_inner))
    delta, _, _, low = oracle.project(u, W_x, W_dt, d_state, w_dt=np.ones(dt_rank), eps=0.0,
                                      return_dt_low=True, lib=lib)
    _close(np.mean(low * low, axis=1), np.ones(7), 1e-14, "unit RMS of the returned dt_low")
    _close(delta, oracle.dt_proj(low, W_dt, lib=lib), 1e-14, "delta == dt_proj(dt_low)")


PROJ_PINS = [pin_proj_basis_selection, pin_proj_linearity, pin_proj_low_rank,
             pin_proj_rmsnorm_closed_forms, pin_proj_norm_off_is_plain, pin_dt_proj_alone,
             pin_proj_dt_low_output]
