"""Pins of the oracle's serving-layout helpers (CPU): the packed layout and
the state-cache slots reduce to the batched definitions in the cases where
both apply, and empty sequences / negative slots behave as specified."""
import numpy as np

import oracle
from tests.oracle_pins import _tiny_case


def test_packed_equal_lengths_is_the_batched_scan():
    case = _tiny_case(5, batch=3, seqlen=9, d_inner=2, d_state=4)
    out, hf = oracle.scan(**case)
    cu = np.array([0, 9, 18, 27])
    pk = {k: (v.reshape(-1, v.shape[-1]) if k in ("x", "delta", "z", "B", "C") else v)
          for k, v in case.items()}
    po, ph = oracle.scan_packed(cu_seqlens=cu, **pk)
    assert np.array_equal(po, out.reshape(-1, out.shape[-1]))
    assert np.array_equal(ph, hf)


def test_packed_ragged_sequences_and_empty_one():
    case = _tiny_case(6, batch=3, seqlen=7, d_inner=3, d_state=2)
    lens = [7, 0, 4]
    cu = np.concatenate([[0], np.cumsum(lens)])
    pk = {k: (np.concatenate([v[b, :n] for b, n in enumerate(lens)])
              if k in ("x", "delta", "z", "B", "C") else v) for k, v in case.items()}
    po, ph = oracle.scan_packed(cu_seqlens=cu, **pk)
    for b, n in enumerate(lens):
        one = {k: (v[b:b + 1, :n] if k in ("x", "delta", "z", "B", "C") else
                   (v[b:b + 1] if k == "h0" else v)) for k, v in case.items()}
        if n:
            o, h = oracle.scan(**one)
            assert np.array_equal(po[cu[b]:cu[b + 1]], o[0])
            assert np.array_equal(ph[b], h[0])
        else:
            assert np.array_equal(ph[b], case["h0"][b])  # empty: final = initial


def test_packed_state_slots():
    case = _tiny_case(7, batch=3, seqlen=5, d_inner=2, d_state=4)
    cache = np.random.default_rng(1).standard_normal((6, 2, 4))
    idx = np.array([4, -1, 0])
    pk = {k: (v.reshape(-1, v.shape[-1]) if k in ("x", "delta", "z", "B", "C") else v)
          for k, v in case.items() if k != "h0"}
    po, pc = oracle.scan_packed(cu_seqlens=np.array([0, 5, 10, 15]), h0=cache,
                                state_indices=idx, **pk)
    plain_h0 = np.stack([cache[4], np.zeros((2, 4)), cache[0]])
    o, h = oracle.scan(**dict(case, h0=plain_h0))
    assert np.array_equal(po, o.reshape(-1, o.shape[-1]))
    assert np.array_equal(pc[4], h[0]) and np.array_equal(pc[0], h[2])
    assert np.array_equal(pc[[1, 2, 3, 5]], cache[[1, 2, 3, 5]])


def test_decode_slots():
    r = np.random.default_rng(3)
    cache = r.standard_normal((5, 3, 4))
    x, dt, z = (r.standard_normal((3, 3)) for _ in range(3))
    B, C = r.standard_normal((3, 4)), r.standard_normal((3, 4))
    A = -np.exp(r.standard_normal((3, 4)))
    idx = np.array([2, -1, 4])
    out, new = oracle.state_update_slots(cache, x, dt, z, B, C, A, idx)
    o, s = oracle.state_update(cache[[2, 4]], x[[0, 2]], dt[[0, 2]], z[[0, 2]], B[[0, 2]],
                               C[[0, 2]], A)
    assert np.array_equal(out[[0, 2]], o) and np.isnan(out[1]).all()
    assert np.array_equal(new[[2, 4]], s)
    assert np.array_equal(new[[0, 1, 3]], cache[[0, 1, 3]])
