"""Property-based pins of the oracle (CPU): for randomly drawn tiny problems --
shapes, optional D / delta_bias / h0, softplus on or off, random negative A --
the sequential fp64 oracle equals the brute-force unrolled sums of the
recurrence, and the scan is causal and split-invariant."""
import numpy as np
from hypothesis import given, settings
from hypothesis import strategies as st

import oracle
from tests.oracle_pins import _close, bruteforce


@st.composite
def problems(draw):
    batch = draw(st.integers(1, 2))
    seqlen = draw(st.integers(1, 12))
    d_inner = draw(st.integers(1, 3))
    d_state = draw(st.sampled_from([1, 2, 4, 8]))
    seed = draw(st.integers(0, 2**31 - 1))
    softplus = draw(st.booleans())
    r = np.random.default_rng(seed)
    case = dict(
        x=r.standard_normal((batch, seqlen, d_inner)),
        delta=r.standard_normal((batch, seqlen, d_inner)),
        z=r.standard_normal((batch, seqlen, d_inner)),
        B=r.standard_normal((batch, seqlen, d_state)),
        C=r.standard_normal((batch, seqlen, d_state)),
        A=-np.exp(r.standard_normal((d_inner, d_state))),
        D=r.standard_normal(d_inner) if draw(st.booleans()) else None,
        delta_bias=r.uniform(-3.0, 0.5, d_inner) if draw(st.booleans()) else None,
        h0=r.standard_normal((batch, d_inner, d_state)) if draw(st.booleans()) else None,
    )
    if not softplus:  # keep Delta positive and O(0.1) without softplus
        case["delta"] = np.abs(case["delta"]) * 0.1
        case["delta_bias"] = None
    return case, softplus


@settings(max_examples=60, deadline=None)
@given(problems())
def test_oracle_equals_bruteforce(p):
    case, sp = p
    out, hf = oracle.scan(**case, delta_softplus=sp)
    ref_out, ref_hf = bruteforce(case, sp)
    _close(out, ref_out, 1e-11, "out")
    _close(hf, ref_hf, 1e-11, "h_final")


@settings(max_examples=30, deadline=None)
@given(problems(), st.integers(0, 11))
def test_split_and_causality(p, cut):
    case, sp = p
    L = case["x"].shape[1]
    cut = min(cut, L)
    out, hf = oracle.scan(**case, delta_softplus=sp)
    # scanning [0, cut) then [cut, L) from the intermediate state is the same scan
    first = {k: (v[:, :cut] if k in ("x", "delta", "z", "B", "C") else v) for k, v in case.items()}
    o1, h1 = oracle.scan(**first, delta_softplus=sp)
    second = {k: (v[:, cut:] if k in ("x", "delta", "z", "B", "C") else v) for k, v in case.items()}
    second["h0"] = h1
    o2, h2 = oracle.scan(**second, delta_softplus=sp)
    _close(np.concatenate([o1, o2], axis=1), out, 1e-12, "split out")
    _close(h2, hf, 1e-12, "split h_final")
    # outputs before `cut` do not depend on inputs from `cut` on
    if cut < L:
        changed = dict(case, x=case["x"].copy())
        changed["x"][:, cut:] += 1.0
        oc, _ = oracle.scan(**changed, delta_softplus=sp)
        assert np.array_equal(oc[:, :cut], out[:, :cut])


@settings(max_examples=25, deadline=None)
@given(problems(), st.integers(0, 2**31 - 1))
def test_backward_equals_finite_differences(p, seed):
    """On random tiny problems the backward oracle's gradient, projected on a
    random direction of every input at once, equals the central finite
    difference of the forward oracle along that direction."""
    case, sp = p
    r = np.random.default_rng(seed)
    out, hf = oracle.scan(**case, delta_softplus=sp)
    dout, dhf = r.standard_normal(out.shape), r.standard_normal(hf.shape)
    g = oracle.scan_bwd(dout=dout, dh_final=dhf, delta_softplus=sp, **case)
    names = {"x": "dx", "delta": "ddelta", "z": "dz", "B": "dB", "C": "dC", "A": "dA",
             "D": "dD", "delta_bias": "ddelta_bias", "h0": "dh0"}
    dirs = {k: r.standard_normal(np.shape(case[k])) for k in names if case[k] is not None}
    eps = 1e-6

    def loss(sign):
        moved = {k: (v + sign * eps * dirs[k] if k in dirs else v) for k, v in case.items()}
        o, h = oracle.scan(**moved, delta_softplus=sp)
        return float(np.sum(o * dout) + np.sum(h * dhf))

    fd = (loss(1.0) - loss(-1.0)) / (2 * eps)
    an = sum(float(np.sum(g[names[k]] * dirs[k])) for k in dirs)
    assert abs(fd - an) <= 1e-6 * max(1.0, abs(fd)), (fd, an)


@settings(max_examples=40, deadline=None)
@given(st.integers(1, 6), st.integers(1, 9), st.integers(1, 5), st.integers(1, 4),
       st.integers(0, 2**31 - 1), st.booleans())
def test_projection_is_rms_normalised_low_rank_map(ntok, d_inner, dt_rank, d_state, seed, norm):
    """For random shapes: delta has rank <= dt_rank and equals dt_proj of the
    returned dt_low; with the norm and unit weights at eps = 0 every part has
    unit RMS; without it, B and C of a one-hot token are W_x's columns."""
    r = np.random.default_rng(seed)
    W_x = r.standard_normal((dt_rank + 2 * d_state, d_inner))
    W_dt = r.standard_normal((d_inner, dt_rank))
    u = r.standard_normal((ntok, d_inner))
    ws = dict(w_dt=np.ones(dt_rank), w_B=np.ones(d_state), w_C=np.ones(d_state)) if norm else {}
    delta, B, C, low = oracle.project(u, W_x, W_dt, d_state, eps=0.0, return_dt_low=True, **ws)
    _close(delta, oracle.dt_proj(low, W_dt), 1e-13, "delta from dt_low")
    assert np.linalg.matrix_rank(delta, tol=1e-9 * max(1.0, np.abs(delta).max())) <= dt_rank
    if norm:
        for part in (low, B, C):
            _close(np.mean(part * part, axis=1), np.ones(ntok), 1e-12, "unit RMS")
    else:
        k = int(r.integers(0, d_inner))
        _, Bk, Ck = oracle.project(np.eye(d_inner)[k:k + 1], W_x, W_dt, d_state)
        assert np.array_equal(Bk[0], W_x[dt_rank:dt_rank + d_state, k])
        assert np.array_equal(Ck[0], W_x[dt_rank + d_state:, k])
