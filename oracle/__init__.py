"""fp64 CPU oracle of the Mamba-1 selective scan (S6) and its decode update.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  The product path (the CUDA library and its Python binding) never
imports, loads or calls anything here, and this package never imports the
product package.

The arithmetic lives in ``oracle_ssm.c`` (plain C, double precision, evaluated
in the order the definition states).  This module only compiles it with gcc,
widens inputs to float64 and splits the independent channels across host
threads (ctypes releases the GIL during the call), which does not change the
order of any floating-point operation inside a channel.

``scan_bwd`` is the scan's reverse-mode gradient (the backward pass).
``ssd_scan`` is the scalar-identity variant (Mamba-2's state matrix: one decay
per head and step, shared by all of the head's channels and states).
``project`` is the step before the scan (Delta, B and C from the scan's
input through the x / dt projections and RMSNorm).  ``scan_packed`` and
``state_update_slots`` define the serving layouts (packed
variable-length batches, state-cache slots) as loops over the batched
definitions.

Sources: "Jamba: A Hybrid Transformer-Mamba Language Model" (obsidian-dorae222
notes), section "Mamba 레이어" -- the S6 recurrence h_t = Abar_t h_{t-1} +
Bbar_t x_t, y_t = C_t h_t with input-dependent Bbar, C, Delta; and "Jamba --
Hybrid SSM-Transformer" (factory.pai-world.com), section "한 페이지로 보는 SSM"
-- the O(1)-per-token decode step.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle_ssm.c")
_LIB_PATH = os.path.join(_HERE, "liboracle_ssm.so")
_lock = threading.Lock()
_lib = None

_dp = ctypes.POINTER(ctypes.c_double)
_i64 = ctypes.c_int64


def build(src: str = _SRC, out: str = _LIB_PATH) -> str:
    """Compile the oracle with gcc (strict IEEE: no fast-math, no FMA contraction)."""
    cmd = ["gcc", "-O2", "-fno-fast-math", "-ffp-contract=off", "-fPIC", "-shared",
           "-o", out, src, "-lm"]
    subprocess.run(cmd, check=True)
    return out


def _declare(lib):
    lib.oracle_softplus.restype = ctypes.c_double
    lib.oracle_softplus.argtypes = [ctypes.c_double]
    lib.oracle_silu.restype = ctypes.c_double
    lib.oracle_silu.argtypes = [ctypes.c_double]
    lib.oracle_scan_f64.restype = ctypes.c_int
    lib.oracle_scan_f64.argtypes = [_i64] * 6 + [_dp] * 8 + [ctypes.c_int, _dp, _dp, _dp]
    lib.oracle_project_f64.restype = ctypes.c_int
    lib.oracle_project_f64.argtypes = ([_i64] * 6 + [_dp] * 6 + [ctypes.c_double]
                                       + [_dp] * 4)
    lib.oracle_scan_bwd_f64.restype = ctypes.c_int
    lib.oracle_scan_bwd_f64.argtypes = ([_i64] * 6 + [_dp] * 8 + [ctypes.c_int]
                                        + [_dp] * 3 + [_dp] * 9)
    lib.oracle_dt_proj_f64.restype = ctypes.c_int
    lib.oracle_dt_proj_f64.argtypes = [_i64] * 5 + [_dp] * 3
    lib.oracle_state_update_f64.restype = ctypes.c_int
    lib.oracle_state_update_f64.argtypes = ([_i64] * 3 + [_dp] * 9
                                            + [ctypes.c_int, _dp])
    lib.oracle_ssd_scan_f64.restype = ctypes.c_int
    lib.oracle_ssd_scan_f64.argtypes = ([_i64] * 7 + [_dp] * 8 + [ctypes.c_int]
                                        + [_dp] * 3)
    return lib


def load(path: str | None = None):
    """Load (building first if needed) the oracle shared library."""
    global _lib
    with _lock:
        if path is not None:
            return _declare(ctypes.CDLL(path))
        if _lib is None:
            if (not os.path.exists(_LIB_PATH)
                    or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)):
                build()
            _lib = _declare(ctypes.CDLL(_LIB_PATH))
        return _lib


def _f64(a):
    if a is None:
        return None
    if hasattr(a, "detach"):  # torch tensor -> numpy, exact widening
        a = a.detach().to("cpu")
        import torch
        a = a.to(torch.float64).numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a):
    return None if a is None else a.ctypes.data_as(_dp)


def softplus(v: float, lib=None) -> float:
    return (lib or load()).oracle_softplus(float(v))


def silu(v: float, lib=None) -> float:
    return (lib or load()).oracle_silu(float(v))


def scan(x, delta, z, B, C, A, D=None, delta_bias=None, delta_softplus=True,
         h0=None, threads: int = 1, lib=None):
    """Sequential fp64 scan.

    Shapes: x, delta, z [batch, seqlen, d_inner]; B, C [batch, seqlen, d_state];
    A [d_inner, d_state]; D, delta_bias [d_inner]; h0 [batch, d_inner, d_state].
    Returns (out [batch, seqlen, d_inner], h_final [batch, d_inner, d_state]) as
    float64 numpy arrays.  Inputs are widened exactly to float64 first.
    """
    lib = lib or load()
    x, delta, z, B, C, A = map(_f64, (x, delta, z, B, C, A))
    D, delta_bias, h0 = _f64(D), _f64(delta_bias), _f64(h0)
    batch, seqlen, d_inner = x.shape
    d_state = A.shape[1]
    assert delta.shape == x.shape and z.shape == x.shape
    assert B.shape == (batch, seqlen, d_state) and C.shape == B.shape
    assert A.shape == (d_inner, d_state)
    out = np.empty_like(x)
    h_final = np.empty((batch, d_inner, d_state), dtype=np.float64)

    def run(lo, hi):
        rc = lib.oracle_scan_f64(batch, seqlen, d_inner, d_state, lo, hi,
                                 _ptr(x), _ptr(delta), _ptr(z), _ptr(B), _ptr(C),
                                 _ptr(A), _ptr(D), _ptr(delta_bias),
                                 int(bool(delta_softplus)), _ptr(h0), _ptr(out),
                                 _ptr(h_final))
        if rc != 0:
            raise ValueError("oracle_scan_f64 rejected its arguments")

    threads = max(1, min(int(threads), d_inner))
    if threads == 1:
        run(0, d_inner)
    else:
        bounds = np.linspace(0, d_inner, threads + 1).astype(np.int64)
        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(lambda i: run(int(bounds[i]), int(bounds[i + 1])), range(threads)))
    return out, h_final


def state_update(state, x, delta, z, B, C, A, D=None, delta_bias=None,
                 delta_softplus=True, lib=None):
    """One fp64 decode step.  Returns (out [batch, d_inner], new_state)."""
    lib = lib or load()
    st = _f64(state).copy()
    x, delta, z, B, C, A = map(_f64, (x, delta, z, B, C, A))
    D, delta_bias = _f64(D), _f64(delta_bias)
    batch, d_inner = x.shape
    d_state = A.shape[1]
    assert st.shape == (batch, d_inner, d_state)
    out = np.empty_like(x)
    rc = lib.oracle_state_update_f64(batch, d_inner, d_state, _ptr(st), _ptr(x),
                                     _ptr(delta), _ptr(z), _ptr(B), _ptr(C), _ptr(A),
                                     _ptr(D), _ptr(delta_bias),
                                     int(bool(delta_softplus)), _ptr(out))
    if rc != 0:
        raise ValueError("oracle_state_update_f64 rejected its arguments")
    return out, st


def scan_bwd(x, delta, z, B, C, A, dout, D=None, delta_bias=None, delta_softplus=True,
             h0=None, dh_final=None, lib=None):
    """Reverse-mode gradient of `scan` in fp64 for a loss whose gradient is dout
    with respect to out and dh_final (None: zero) with respect to h_final.

    Returns a dict with dx, ddelta, dz [batch, seqlen, d_inner]; dB, dC [batch,
    seqlen, d_state]; dA [d_inner, d_state]; dD, ddelta_bias [d_inner]; dh0
    [batch, d_inner, d_state] (gradients of the parameters that were given;
    an absent D, bias or h0 still gets its gradient, as if it were zero).
    """
    lib = lib or load()
    x, delta, z, B, C, A, dout = map(_f64, (x, delta, z, B, C, A, dout))
    D, delta_bias, h0, dh_final = map(_f64, (D, delta_bias, h0, dh_final))
    batch, seqlen, d_inner = x.shape
    d_state = A.shape[1]
    assert dout.shape == x.shape
    g = dict(dx=np.empty_like(x), ddelta=np.empty_like(x), dz=np.empty_like(x),
             dB=np.zeros_like(B), dC=np.zeros_like(C), dA=np.zeros_like(A),
             dD=np.zeros(d_inner), ddelta_bias=np.zeros(d_inner),
             dh0=np.empty((batch, d_inner, d_state)))
    # an absent D or bias is zero in the forward pass; its gradient is still defined
    D0 = D if D is not None else np.zeros(d_inner)
    b0 = delta_bias if delta_bias is not None else np.zeros(d_inner)
    rc = lib.oracle_scan_bwd_f64(batch, seqlen, d_inner, d_state, 0, d_inner, _ptr(x),
                                 _ptr(delta), _ptr(z), _ptr(B), _ptr(C), _ptr(A), _ptr(D0),
                                 _ptr(b0), int(bool(delta_softplus)), _ptr(h0), _ptr(dout),
                                 _ptr(dh_final), _ptr(g["dx"]), _ptr(g["ddelta"]), _ptr(g["dz"]),
                                 _ptr(g["dB"]), _ptr(g["dC"]), _ptr(g["dA"]), _ptr(g["dD"]),
                                 _ptr(g["ddelta_bias"]), _ptr(g["dh0"]))
    if rc != 0:
        raise ValueError("oracle_scan_bwd_f64 rejected its arguments")
    return g


def project(u, W_x, W_dt, d_state, w_dt=None, w_B=None, w_C=None, eps=1e-6,
            threads: int = 1, lib=None, return_dt_low: bool = False):
    """Delta (raw, before bias and softplus), B and C of every token from the
    scan's input u, in fp64.

    u [..., d_inner]; W_x [dt_rank + 2 d_state, d_inner]; W_dt [d_inner,
    dt_rank]; w_dt [dt_rank], w_B / w_C [d_state] are RMSNorm weights (None: that
    part is not normalised).  Returns (delta [..., d_inner], B [..., d_state],
    C [..., d_state]), and with ``return_dt_low`` also dt_low [..., dt_rank]
    after its RMSNorm (the input of the last product).
    """
    lib = lib or load()
    u, W_x, W_dt = map(_f64, (u, W_x, W_dt))
    w_dt, w_B, w_C = map(_f64, (w_dt, w_B, w_C))
    lead = u.shape[:-1]
    d_inner = u.shape[-1]
    dt_rank = W_dt.shape[1]
    assert W_x.shape == (dt_rank + 2 * d_state, d_inner) and W_dt.shape == (d_inner, dt_rank)
    u2 = u.reshape(-1, d_inner)
    ntok = u2.shape[0]
    delta = np.empty((ntok, d_inner))
    B = np.empty((ntok, d_state))
    C = np.empty((ntok, d_state))
    dt_low = np.empty((ntok, dt_rank)) if return_dt_low else None

    def run(lo, hi):
        rc = lib.oracle_project_f64(ntok, d_inner, dt_rank, d_state, lo, hi, _ptr(u2),
                                    _ptr(W_x), _ptr(W_dt), _ptr(w_dt), _ptr(w_B), _ptr(w_C),
                                    float(eps), _ptr(delta), _ptr(B), _ptr(C), _ptr(dt_low))
        if rc != 0:
            raise ValueError("oracle_project_f64 rejected its arguments")

    threads = max(1, min(int(threads), ntok))
    if threads == 1:
        run(0, ntok)
    else:
        bounds = np.linspace(0, ntok, threads + 1).astype(np.int64)
        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(lambda i: run(int(bounds[i]), int(bounds[i + 1])), range(threads)))
    res = (delta.reshape(*lead, d_inner), B.reshape(*lead, d_state), C.reshape(*lead, d_state))
    if return_dt_low:
        res += (dt_low.reshape(*lead, dt_rank),)
    return res


def dt_proj(dt_low, W_dt, threads: int = 1, lib=None):
    """The last product of `project` alone: delta = dt_low @ W_dt.T in fp64.
    dt_low [..., dt_rank]; W_dt [d_inner, dt_rank].  Returns delta [..., d_inner]."""
    lib = lib or load()
    dt_low, W_dt = _f64(dt_low), _f64(W_dt)
    d_inner, dt_rank = W_dt.shape
    lead = dt_low.shape[:-1]
    a = dt_low.reshape(-1, dt_rank)
    ntok = a.shape[0]
    delta = np.empty((ntok, d_inner))

    def run(lo, hi):
        if lib.oracle_dt_proj_f64(ntok, d_inner, dt_rank, lo, hi, _ptr(a), _ptr(W_dt),
                                  _ptr(delta)) != 0:
            raise ValueError("oracle_dt_proj_f64 rejected its arguments")

    threads = max(1, min(int(threads), ntok))
    if threads == 1:
        run(0, ntok)
    else:
        bounds = np.linspace(0, ntok, threads + 1).astype(np.int64)
        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(lambda i: run(int(bounds[i]), int(bounds[i + 1])), range(threads)))
    return delta.reshape(*lead, d_inner)


def scan_packed(x, delta, z, B, C, A, cu_seqlens, D=None, delta_bias=None,
                delta_softplus=True, h0=None, state_indices=None, threads: int = 1, lib=None):
    """The packed variable-length layout, by definition one `scan` per sequence.

    x, delta, z [total_tokens, d_inner] and B, C [total_tokens, d_state] hold
    sequence b in rows cu_seqlens[b] .. cu_seqlens[b+1]-1.  Without
    `state_indices`, h0 is [batch, d_inner, d_state] (or None) and the final
    states are returned as [batch, d_inner, d_state].  With it, h0 is a
    [num_slots, d_inner, d_state] cache (or None), sequence b starts from row
    state_indices[b] (zero for a negative index) and the returned cache is h0
    with row state_indices[b] replaced by sequence b's final state (rows of
    negative indices untouched).  An empty sequence's final state is its
    initial state.  Returns (out [total_tokens, d_inner], final states).
    """
    x, delta, z, B, C, A = map(_f64, (x, delta, z, B, C, A))
    cu = np.asarray(_f64(cu_seqlens), dtype=np.int64)
    h0 = _f64(h0)
    batch = cu.size - 1
    d_inner, d_state = A.shape
    out = np.zeros((x.shape[0], d_inner), dtype=np.float64)
    if state_indices is not None:
        idx = np.asarray(_f64(state_indices), dtype=np.int64)
        final = (h0.copy() if h0 is not None else None)
    else:
        final = np.zeros((batch, d_inner, d_state), dtype=np.float64)
    for b in range(batch):
        lo, hi = int(cu[b]), int(cu[b + 1])
        if state_indices is not None:
            row = int(idx[b])
            init = h0[row] if (row >= 0 and h0 is not None) else np.zeros((d_inner, d_state))
        else:
            init = h0[b] if h0 is not None else np.zeros((d_inner, d_state))
        if hi > lo:
            o, hf = scan(x[None, lo:hi], delta[None, lo:hi], z[None, lo:hi], B[None, lo:hi],
                         C[None, lo:hi], A, D=D, delta_bias=delta_bias,
                         delta_softplus=delta_softplus, h0=init[None], threads=threads, lib=lib)
            out[lo:hi] = o[0]
            hf = hf[0]
        else:
            hf = np.array(init, dtype=np.float64)
        if state_indices is None:
            final[b] = hf
        elif row >= 0:
            if final is None:
                final = np.zeros((int(idx.max()) + 1, d_inner, d_state), dtype=np.float64)
            final[row] = hf
    return out, final


def state_update_slots(cache, x, delta, z, B, C, A, state_indices, D=None, delta_bias=None,
                       delta_softplus=True, lib=None):
    """One decode step through a state cache: request b updates row
    state_indices[b]; a negative index skips the request.  Returns (out
    [batch, d_inner] with NaN rows for skipped requests, the updated cache)."""
    st = _f64(cache).copy()
    idx = np.asarray(_f64(state_indices), dtype=np.int64)
    x, delta, z, B, C = map(_f64, (x, delta, z, B, C))
    live = [b for b in range(idx.size) if idx[b] >= 0]
    out = np.full(x.shape, np.nan)
    if live:
        rows = idx[live]
        o, new = state_update(st[rows], x[live], delta[live], z[live], B[live], C[live], A, D=D,
                              delta_bias=delta_bias, delta_softplus=delta_softplus, lib=lib)
        out[live] = o
        st[rows] = new
    return out, st


def ssd_scan(x, delta, z, B, C, A, nheads, D=None, delta_bias=None, delta_softplus=True,
             h0=None, threads: int = 1, lib=None):
    """Sequential fp64 scan of the scalar-identity (Mamba-2) variant.

    Shapes: x, z [batch, seqlen, nheads * headdim]; delta [batch, seqlen,
    nheads]; B, C [batch, seqlen, d_state]; A, delta_bias [nheads]; D
    [nheads * headdim]; h0 [batch, nheads * headdim, d_state].  Returns (out,
    h_final) as float64 arrays.  Heads are independent and split across host
    threads.
    """
    lib = lib or load()
    x, delta, z, B, C, A = map(_f64, (x, delta, z, B, C, A))
    D, delta_bias, h0 = _f64(D), _f64(delta_bias), _f64(h0)
    batch, seqlen, d_inner = x.shape
    d_state = B.shape[-1]
    assert d_inner % nheads == 0 and A.shape == (nheads,)
    assert delta.shape == (batch, seqlen, nheads) and z.shape == x.shape
    headdim = d_inner // nheads
    out = np.empty_like(x)
    h_final = np.empty((batch, d_inner, d_state), dtype=np.float64)

    def run(lo, hi):
        if lib.oracle_ssd_scan_f64(batch, seqlen, nheads, headdim, d_state, lo, hi, _ptr(x),
                                   _ptr(delta), _ptr(z), _ptr(B), _ptr(C), _ptr(A), _ptr(D),
                                   _ptr(delta_bias), int(bool(delta_softplus)), _ptr(h0),
                                   _ptr(out), _ptr(h_final)) != 0:
            raise ValueError("oracle_ssd_scan_f64 rejected its arguments")

    threads = max(1, min(int(threads), nheads))
    if threads == 1:
        run(0, nheads)
    else:
        bounds = np.linspace(0, nheads, threads + 1).astype(np.int64)
        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(lambda i: run(int(bounds[i]), int(bounds[i + 1])), range(threads)))
    return out, h_final
