"""The oracle's host-thread split is not part of its arithmetic (CPU).

The Python wrapper hands disjoint ranges of channels (scan) or tokens
(project, dt_proj) to host threads; inside a range every floating-point
operation happens in the order the definition states.  So any thread count
must give the same bits as one thread.  Every GPU parity test uses the
threaded oracle as its checker, so this pins that the split itself (range
bounds, a dropped or doubled last range, an output written by the wrong range)
cannot change what is checked against."""
import numpy as np
import pytest

import oracle


def _scan_case(seed, batch=2, seqlen=37, d_inner=23, d_state=16):
    r = np.random.default_rng(seed)
    return dict(
        x=r.standard_normal((batch, seqlen, d_inner)),
        delta=r.standard_normal((batch, seqlen, d_inner)),
        z=r.standard_normal((batch, seqlen, d_inner)),
        B=r.standard_normal((batch, seqlen, d_state)),
        C=r.standard_normal((batch, seqlen, d_state)),
        A=-np.exp(r.standard_normal((d_inner, d_state))),
        D=r.standard_normal(d_inner),
        delta_bias=r.uniform(-4.0, 0.0, d_inner),
        h0=r.standard_normal((batch, d_inner, d_state)),
    )


@pytest.mark.parametrize("threads", [3, 7])
def test_scan_threads_bitwise_equal_one_thread(threads):
    c = _scan_case(1)
    one = oracle.scan(**c, threads=1)
    many = oracle.scan(**c, threads=threads)
    for a, b in zip(one, many):
        assert np.array_equal(a, b)


@pytest.mark.parametrize("threads", [3, 7])
def test_project_and_dt_proj_threads_bitwise_equal_one_thread(threads):
    r = np.random.default_rng(4)
    ntok, d_inner, R, N = 29, 40, 12, 4
    u = r.standard_normal((ntok, d_inner))
    W_x = r.standard_normal((R + 2 * N, d_inner)) / np.sqrt(d_inner)
    W_dt = r.standard_normal((d_inner, R)) / np.sqrt(R)
    w = r.uniform(0.5, 1.5, R + 2 * N)
    kw = dict(w_dt=w[:R], w_B=w[R:R + N], w_C=w[R + N:], return_dt_low=True)
    one = oracle.project(u, W_x, W_dt, N, threads=1, **kw)
    many = oracle.project(u, W_x, W_dt, N, threads=threads, **kw)
    for a, b in zip(one, many):
        assert np.array_equal(a, b)
    dl = r.standard_normal((ntok, R))
    assert np.array_equal(oracle.dt_proj(dl, W_dt, threads=1),
                          oracle.dt_proj(dl, W_dt, threads=threads))


def test_more_threads_than_work():
    """More threads than channels or tokens still covers every one once."""
    c = _scan_case(5, batch=1, seqlen=5, d_inner=3, d_state=2)
    one = oracle.scan(**c, threads=1)
    many = oracle.scan(**c, threads=16)
    for a, b in zip(one, many):
        assert np.array_equal(a, b)
