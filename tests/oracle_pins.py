"""Pins of the fp64 oracle against facts that do not come from the oracle.

Each ``pin_*`` function takes a loaded oracle library and raises AssertionError
when the oracle disagrees with:
  * libm / numpy / scipy routines the definition reduces to (softplus, silu);
  * a brute-force unrolled sum of the recurrence, written independently with
    products of decays replaced by exponentials of cumulative sums of Delta;
  * the closed form of the geometric series for constant parameters;
  * the Delta -> 0 limit (out = D x silu(z), state unchanged) and the
    large-Delta limit (memoryless: y_t = Delta x_t (C_t . B_t) + D x_t);
  * structural identities: split scan == whole scan, L decode steps == scan,
    channel / batch independence, causality.
The same functions run against deliberately broken copies of the oracle in
test_oracle_mutations.py, which checks that every planted mistake trips one.

Sources of the method: "Jamba: A Hybrid Transformer-Mamba Language Model"
(obsidian-dorae222 notes), section "Mamba 레이어"; "Jamba -- Hybrid
SSM-Transformer" (factory.pai-world.com), section "한 페이지로 보는 SSM".
"""
from __future__ import annotations

import math

import numpy as np
from scipy.special import expit

import oracle


def _rng(seed):
    return np.random.default_rng(seed)


def _tiny_case(seed, batch=2, seqlen=11, d_inner=3, d_state=4, h0=True):
    r = _rng(seed)
    return dict(
        x=r.standard_normal((batch, seqlen, d_inner)),
        delta=r.standard_normal((batch, seqlen, d_inner)),
        z=r.standard_normal((batch, seqlen, d_inner)),
        B=r.standard_normal((batch, seqlen, d_state)),
        C=r.standard_normal((batch, seqlen, d_state)),
        A=-np.exp(r.standard_normal((d_inner, d_state))),
        D=r.standard_normal(d_inner),
        delta_bias=r.uniform(-3.0, 0.5, d_inner),
        h0=r.standard_normal((batch, d_inner, d_state)) if h0 else None,
    )


def _silu_ref(z):
    return z * expit(z)


def _close(a, b, rtol, what):
    a, b = np.asarray(a), np.asarray(b)
    scale = max(1.0, float(np.max(np.abs(b))) if b.size else 1.0)
    err = float(np.max(np.abs(a - b))) if b.size else 0.0
    assert err <= rtol * scale, f"{what}: max |diff| {err:.3e} > {rtol:.1e} * {scale:.3e}"


def pin_softplus_silu_libm(lib):
    for v in np.linspace(-40.0, 40.0, 161):
        ref = np.logaddexp(0.0, v)  # log(1 + e^v)
        got = oracle.softplus(v, lib=lib)
        assert abs(got - ref) <= 1e-15 * max(1.0, abs(ref)) + 1e-300, (v, got, ref)
        assert abs(oracle.silu(v, lib=lib) - _silu_ref(v)) <= 1e-15 * max(1.0, abs(v)), v
    for v in (-745.0, -100.0, -1e-8, 0.0, 1e-8, 100.0, 700.0):
        assert math.isclose(oracle.softplus(v, lib=lib), float(np.logaddexp(0.0, v)),
                            rel_tol=1e-15, abs_tol=1e-320)


def bruteforce(case, delta_softplus=True):
    """y_t = sum_{s<=t} C_t diag(exp(A (S_t - S_s))) Delta_s B_s x_s
             + C_t diag(exp(A S_t)) h0 + D x_t,  gated by silu(z_t).
    S is the inclusive cumulative sum of Delta, so exp(A (S_t - S_s)) is the
    product of the per-step decays Abar_r for r = s+1..t."""
    x, dl, z, B, C, A = (case[k] for k in ("x", "delta", "z", "B", "C", "A"))
    D = case["D"] if case["D"] is not None else np.zeros(x.shape[2])
    bias = case["delta_bias"] if case["delta_bias"] is not None else np.zeros(x.shape[2])
    h0 = case["h0"]
    bsz, L, Dn = x.shape
    N = A.shape[1]
    v = dl + bias[None, None, :]
    Delta = np.logaddexp(0.0, v) if delta_softplus else v
    S = np.cumsum(Delta, axis=1)
    out = np.zeros_like(x)
    hf = np.zeros((bsz, Dn, N))
    for b in range(bsz):
        for d in range(Dn):
            for t in range(L):
                # state after step t, as an unrolled sum over the inputs s <= t
                h = np.zeros(N)
                for s in range(t + 1):
                    h += np.exp(A[d] * (S[b, t, d] - S[b, s, d])) * Delta[b, s, d] * B[b, s] * x[b, s, d]
                if h0 is not None:
                    h += np.exp(A[d] * S[b, t, d]) * h0[b, d]
                y = float(np.dot(C[b, t], h)) + D[d] * x[b, t, d]
                out[b, t, d] = y * _silu_ref(z[b, t, d])
                if t == L - 1:
                    hf[b, d] = h
            if L == 0 and h0 is not None:
                hf[b, d] = h0[b, d]
    return out, hf


def pin_bruteforce_tiny(lib):
    for seed, kw in [(1, {}), (2, dict(batch=1, seqlen=23, d_inner=2, d_state=16)),
                     (3, dict(batch=3, seqlen=1, d_inner=4, d_state=2, h0=False)),
                     (4, dict(batch=1, seqlen=40, d_inner=5, d_state=4))]:
        case = _tiny_case(seed, **kw)
        for sp in (True, False):
            if not sp:  # keep Delta positive and O(0.1) without softplus
                case = dict(case, delta=np.abs(case["delta"]) * 0.1, delta_bias=np.zeros(case["x"].shape[2]))
            out, hf = oracle.scan(**case, delta_softplus=sp, lib=lib)
            ref_out, ref_hf = bruteforce(case, sp)
            _close(out, ref_out, 1e-11, f"brute-force out (seed {seed}, softplus {sp})")
            _close(hf, ref_hf, 1e-11, f"brute-force h_final (seed {seed}, softplus {sp})")


def pin_closed_form_geometric(lib):
    # constant Delta, x, B, C, z: h_t = b (1 - a^t) / (1 - a) with a = e^{Delta A},
    # b = Delta B x (t counted from 1), starting from h0 = 0.
    L, Dn, N = 50, 2, 5
    r = _rng(7)
    A = -np.exp(r.standard_normal((Dn, N)))
    Dv = np.array([0.7, -1.3])
    xc, dc, zc = np.array([0.9, -1.7]), np.array([0.05, 0.3]), np.array([1.1, -0.4])
    Bc, Cc = r.standard_normal(N), r.standard_normal(N)
    x = np.broadcast_to(xc, (1, L, Dn)).copy()
    dl = np.broadcast_to(dc, (1, L, Dn)).copy()
    z = np.broadcast_to(zc, (1, L, Dn)).copy()
    B = np.broadcast_to(Bc, (1, L, N)).copy()
    C = np.broadcast_to(Cc, (1, L, N)).copy()
    out, hf = oracle.scan(x, dl, z, B, C, A, D=Dv, delta_bias=None, delta_softplus=False,
                          lib=lib)
    t = np.arange(1, L + 1)[:, None, None]  # [L, 1, 1]
    a = np.exp(dc[:, None] * A)             # [Dn, N]
    b = dc[:, None] * Bc[None, :] * xc[:, None]
    h = b * (1 - a ** t) / (1 - a)          # [L, Dn, N]
    y = np.einsum("n,ldn->ld", Cc, h) + Dv * xc
    ref = y * _silu_ref(zc)
    _close(out[0], ref, 1e-12, "geometric closed form (out)")
    _close(hf[0], h[-1], 1e-12, "geometric closed form (h_final)")


def pin_delta_zero_limit(lib):
    case = _tiny_case(11, batch=2, seqlen=9, d_inner=3, d_state=4)
    case = dict(case, delta=np.zeros_like(case["x"]), delta_bias=None)
    out, hf = oracle.scan(**case, delta_softplus=False, lib=lib)
    # Delta = 0: Abar = 1, Bbar x = 0, so h stays h0 and y_t = C_t . h0 + D x_t.
    h0 = case["h0"]
    y = np.einsum("bln,bdn->bld", case["C"], h0) + case["D"] * case["x"]
    _close(out, y * _silu_ref(case["z"]), 1e-13, "Delta=0 limit (out)")
    assert np.array_equal(hf, h0), "Delta=0 must leave the state unchanged"
    case0 = dict(case, h0=None)
    out0, hf0 = oracle.scan(**case0, delta_softplus=False, lib=lib)
    _close(out0, case["D"] * case["x"] * _silu_ref(case["z"]), 1e-14, "Delta=0, h0=0")
    assert not np.any(hf0)


def pin_large_delta_memoryless(lib):
    case = _tiny_case(12, batch=2, seqlen=13, d_inner=4, d_state=8)
    A = -1.0 - np.abs(case["A"])  # A <= -1 so exp(Delta A) <= e^-60
    case = dict(case, A=A, delta=np.full_like(case["x"], 60.0), delta_bias=None)
    out, hf = oracle.scan(**case, delta_softplus=False, lib=lib)
    cb = np.einsum("bln,bln->bl", case["C"], case["B"])[:, :, None]
    y = 60.0 * case["x"] * cb + case["D"] * case["x"]
    _close(out, y * _silu_ref(case["z"]), 1e-12, "large-Delta memoryless limit")
    _close(hf, 60.0 * case["B"][:, -1, None, :] * case["x"][:, -1, :, None], 1e-12,
           "large-Delta final state")


def pin_split_scan(lib):
    case = _tiny_case(21, batch=2, seqlen=30, d_inner=3, d_state=4)
    whole, hw = oracle.scan(**case, lib=lib)
    for cut in (1, 13, 29):
        first = {k: (v[:, :cut] if k in ("x", "delta", "z", "B", "C") else v)
                 for k, v in case.items()}
        second = {k: (v[:, cut:] if k in ("x", "delta", "z", "B", "C") else v)
                  for k, v in case.items()}
        o1, h1 = oracle.scan(**first, lib=lib)
        second["h0"] = h1
        o2, h2 = oracle.scan(**second, lib=lib)
        assert np.array_equal(np.concatenate([o1, o2], axis=1), whole), cut
        assert np.array_equal(h2, hw), cut


def pin_decode_equals_scan(lib):
    case = _tiny_case(31, batch=3, seqlen=17, d_inner=4, d_state=8)
    out, hf = oracle.scan(**case, lib=lib)
    st = case["h0"]
    for t in range(case["x"].shape[1]):
        o, st = oracle.state_update(st, case["x"][:, t], case["delta"][:, t], case["z"][:, t],
                                    case["B"][:, t], case["C"][:, t], case["A"], D=case["D"],
                                    delta_bias=case["delta_bias"], lib=lib)
        assert np.array_equal(o, out[:, t]), t
    assert np.array_equal(st, hf)


def pin_independence_and_causality(lib):
    case = _tiny_case(41, batch=3, seqlen=15, d_inner=5, d_state=4)
    out, hf = oracle.scan(**case, lib=lib)
    # channel permutation commutes with the scan
    perm = np.array([3, 0, 4, 2, 1])
    pc = dict(case)
    for k in ("x", "delta", "z"):
        pc[k] = case[k][:, :, perm]
    pc["A"], pc["D"], pc["delta_bias"] = case["A"][perm], case["D"][perm], case["delta_bias"][perm]
    pc["h0"] = case["h0"][:, perm]
    po, ph = oracle.scan(**pc, lib=lib)
    assert np.array_equal(po, out[:, :, perm]) and np.array_equal(ph, hf[:, perm])
    # each sequence alone gives the same result
    for b in range(3):
        sb = {k: (v[b:b + 1] if k in ("x", "delta", "z", "B", "C", "h0") else v)
              for k, v in case.items()}
        ob, hb = oracle.scan(**sb, lib=lib)
        assert np.array_equal(ob[0], out[b]) and np.array_equal(hb[0], hf[b])
    # causality: changing step k leaves steps < k untouched and changes step k
    k = 7
    for key in ("x", "delta", "B"):
        cc = {kk: (vv.copy() if vv is not None else None) for kk, vv in case.items()}
        cc[key][:, k] += 1.0
        oc, _ = oracle.scan(**cc, lib=lib)
        assert np.array_equal(oc[:, :k], out[:, :k]), key
        assert not np.allclose(oc[:, k], out[:, k]), key


def pin_optional_parameters(lib):
    case = _tiny_case(51, batch=1, seqlen=6, d_inner=3, d_state=4)
    a, ha = oracle.scan(**dict(case, D=None, delta_bias=None, h0=None), lib=lib)
    b, hb = oracle.scan(**dict(case, D=np.zeros(3), delta_bias=np.zeros(3),
                               h0=np.zeros((1, 3, 4))), lib=lib)
    assert np.array_equal(a, b) and np.array_equal(ha, hb)


ALL_PINS = [pin_softplus_silu_libm, pin_bruteforce_tiny, pin_closed_form_geometric,
            pin_delta_zero_limit, pin_large_delta_memoryless, pin_split_scan,
            pin_decode_equals_scan, pin_independence_and_causality, pin_optional_parameters]
