"""Pins of the scalar-identity (Mamba-2) variant of the oracle (CPU).

oracle.ssd_scan is the sequential definition.  It is pinned against:
  * the dual, quadratic form of the same map -- the "state space duality" the
    Mamba-2 paper is named for -- written here in numpy:
        y_t = sum_{s <= t} (C_t . B_s) exp(A sum_{r=s+1..t} Delta_r) Delta_s x_s
              + exp(A sum_{r<=t} Delta_r) (C_t . h0) + D x_t,
    out_t = y_t silu(z_t); an attention-like matrix L o (C B^T) applied to the
    inputs, with no recurrence at all;
  * the diagonal (Mamba-1) oracle, which must give the same map when every
    state of a head's channels decays by the head's scalar A and every channel
    of the head takes the head's Delta;
  * the split identity (scan L1, then L2 from the final state).
"""
import numpy as np

import oracle


def case(seed, batch=2, seqlen=23, nheads=3, headdim=4, d_state=5, h0=True, bias=True,
         D=True, softplus=True):
    r = np.random.default_rng(seed)
    d_inner = nheads * headdim
    c = dict(x=r.standard_normal((batch, seqlen, d_inner)),
             delta=r.standard_normal((batch, seqlen, nheads)),
             z=r.standard_normal((batch, seqlen, d_inner)),
             B=r.standard_normal((batch, seqlen, d_state)),
             C=r.standard_normal((batch, seqlen, d_state)),
             A=-np.exp(r.standard_normal(nheads)),
             D=r.standard_normal(d_inner) if D else None,
             delta_bias=r.uniform(-3.0, 0.5, nheads) if bias else None,
             h0=r.standard_normal((batch, d_inner, d_state)) if h0 else None)
    if not softplus:
        c["delta"] = np.abs(c["delta"]) * 0.1
        c["delta_bias"] = None
    return c, nheads, softplus


def _softplus(v):
    return np.where(v > 0, v + np.log1p(np.exp(-v)), np.log1p(np.exp(v)))


def dual_form(c, nheads, softplus):
    """The quadratic (dual) form of the scalar-identity SSM, in numpy."""
    x, delta, z, B, C, A = c["x"], c["delta"], c["z"], c["B"], c["C"], c["A"]
    batch, L, d_inner = x.shape
    P = d_inner // nheads
    out = np.empty_like(x)
    for b in range(batch):
        v = delta[b] + (c["delta_bias"] if c["delta_bias"] is not None else 0.0)
        dl = _softplus(v) if softplus else v                      # [L, H]
        cum = np.cumsum(dl, axis=0)                                # sum_{r<=t} Delta_r
        CB = C[b] @ B[b].T                                         # [L, L]: C_t . B_s
        for hd in range(nheads):
            seg = cum[:, hd][:, None] - cum[:, hd][None, :]         # sum_{r=s+1..t}
            Lmask = np.where(np.tril(np.ones((L, L), bool)), np.exp(A[hd] * np.tril(seg)), 0.0)
            M = Lmask * CB                                         # [t, s]
            cols = slice(hd * P, (hd + 1) * P)
            u = dl[:, hd][:, None] * x[b][:, cols]                 # Delta_s x_s
            y = M @ u
            if c["h0"] is not None:
                dec0 = np.exp(A[hd] * cum[:, hd])                  # exp(A sum_{r<=t})
                y += dec0[:, None] * (C[b] @ c["h0"][b, cols, :].T)
            if c["D"] is not None:
                y += c["D"][cols][None, :] * x[b][:, cols]
            zz = z[b][:, cols]
            out[b][:, cols] = y * zz / (1.0 + np.exp(-zz))
    return out


def _rel(a, b):
    return float(np.max(np.abs(a - b)) / max(1e-300, np.max(np.abs(b))))


def pin_dual_form():
    for seed, kw in [(1, {}), (2, dict(h0=False)), (3, dict(D=False, bias=False)),
                     (4, dict(softplus=False)), (5, dict(seqlen=1)), (6, dict(headdim=1, nheads=5))]:
        c, H, sp = case(seed, **kw)
        out, _ = oracle.ssd_scan(**c, nheads=H, delta_softplus=sp)
        ref = dual_form(c, H, sp)
        assert _rel(out, ref) < 1e-11, (seed, kw, _rel(out, ref))


def pin_equals_diagonal_oracle_with_tied_parameters():
    c, H, sp = case(7, seqlen=40)
    out, hf = oracle.ssd_scan(**c, nheads=H, delta_softplus=sp, threads=2)
    P = c["x"].shape[2] // H
    N = c["B"].shape[2]
    head = np.repeat(np.arange(H), P)                               # head of each channel
    A_diag = np.repeat(c["A"][head][:, None], N, axis=1)            # [D, N]
    delta_c = c["delta"][:, :, head]                                 # [B, L, D]
    bias_c = c["delta_bias"][head]
    ref, ref_h = oracle.scan(c["x"], delta_c, c["z"], c["B"], c["C"], A_diag, D=c["D"],
                             delta_bias=bias_c, h0=c["h0"], threads=3)
    assert _rel(out, ref) < 1e-13 and _rel(hf, ref_h) < 1e-13


def pin_split_scan():
    c, H, sp = case(8, seqlen=30)
    whole, hw = oracle.ssd_scan(**c, nheads=H, delta_softplus=sp)
    cut = 11
    first = {k: (v[:, :cut] if k in ("x", "delta", "z", "B", "C") else v) for k, v in c.items()}
    second = {k: (v[:, cut:] if k in ("x", "delta", "z", "B", "C") else v) for k, v in c.items()}
    o1, h1 = oracle.ssd_scan(**first, nheads=H, delta_softplus=sp)
    second["h0"] = h1
    o2, h2 = oracle.ssd_scan(**second, nheads=H, delta_softplus=sp)
    assert _rel(np.concatenate([o1, o2], axis=1), whole) < 1e-13 and _rel(h2, hw) < 1e-13


def pin_threads_bitwise():
    c, H, sp = case(9, nheads=7)
    a = oracle.ssd_scan(**c, nheads=H, delta_softplus=sp, threads=1)
    b = oracle.ssd_scan(**c, nheads=H, delta_softplus=sp, threads=3)
    assert all(np.array_equal(u, v) for u, v in zip(a, b))


PINS = [pin_dual_form, pin_equals_diagonal_oracle_with_tied_parameters, pin_split_scan,
        pin_threads_bitwise]
