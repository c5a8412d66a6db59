"""B200-native Mamba-1 selective scan (S6): Python binding of the C ABI.

The calls, with the names of the C entry points:

* ``jamba_ssm_scan``          -- prefill scan over whole sequences, returning the
  gated output and (for the decode cache) the final state;
* ``jamba_ssm_state_update``  -- one-token decode step, state updated in place;
* ``jamba_ssm_scan_bwd``      -- the scan's backward pass (gradients of every
  input, for training);
* ``jamba_ssm_ssd_scan``      -- the scalar-identity (Mamba-2) variant of the
  scan: one decay per head and token;
* ``jamba_ssm_x_proj``        -- the projection of the scan's input to dt_low, B
  and C with their RMSNorms (libjamba_ssm_proj.so);
* ``jamba_ssm_dt_proj``       -- the low-rank product that produces the scan's
  raw Delta from dt_low (libjamba_ssm_proj.so).

Every step of the computation runs in the CUDA kernels of the libraries; this
module only checks tensor metadata, allocates outputs with PyTorch when the
caller does not pass them, and hands raw device pointers and the current CUDA
stream to the library.  There is no CPU fallback: without the built library or
without a CUDA device every call raises.
"""
from __future__ import annotations

import torch

from . import _lib
from ._lib import JambaSSMError

__all__ = ["jamba_ssm_scan", "jamba_ssm_state_update", "jamba_ssm_get_status", "scan_plan",
           "jamba_ssm_scan_workspace_size", "jamba_ssm_scan_ckpt_size", "jamba_ssm_scan_bwd",
           "jamba_ssm_scan_bwd_workspace_size", "jamba_ssm_ssd_scan",
           "jamba_ssm_x_proj", "jamba_ssm_dt_proj", "jamba_ssm_proj_get_status",
           "JambaSSMError"]

_IO = {torch.bfloat16: _lib.BF16, torch.float32: _lib.F32}


def _ptr(t):
    return None if t is None else t.data_ptr()


def _check(t, name, shape, dtype, device):
    if t is None:
        return
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if t.dtype != dtype:
        raise TypeError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _stream(stream, device):
    if stream is None:
        return torch.cuda.current_stream(device).cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _workspace(ws, device):
    """(pointer, bytes) of an optional workspace tensor (the call's status word)."""
    if ws is None:
        return None, 0
    if not isinstance(ws, torch.Tensor) or ws.device != device or not ws.is_contiguous():
        raise ValueError("workspace must be a contiguous tensor on the device of the inputs")
    return ws.data_ptr(), ws.numel() * ws.element_size()


def _scan_params(x, delta, z, B, C, A, D, delta_bias, delta_softplus, h0, out, h_final,
                 variant, debug_flags, timeout_cycles, cu_seqlens=None, state_indices=None,
                 workspace=None, ckpt=None):
    if x.dtype not in _IO:
        raise TypeError(f"x must be bfloat16 or float32, got {x.dtype}")
    d_state = A.shape[-1]
    dev = x.device
    io = x.dtype
    if cu_seqlens is not None:
        # packed layout: [total_tokens, d_inner], sequences delimited by cu_seqlens
        total, d_inner = x.shape
        _check(cu_seqlens, "cu_seqlens", (cu_seqlens.numel(),), torch.int32, dev)
        batch, seqlen = cu_seqlens.numel() - 1, 0
        act, bc = (total, d_inner), (total, d_state)
    else:
        batch, seqlen, d_inner = x.shape
        total = 0
        act, bc = (batch, seqlen, d_inner), (batch, seqlen, d_state)
    for t, n, s in ((x, "x", act), (delta, "delta", act), (z, "z", act), (B, "B", bc),
                    (C, "C", bc), (out, "out", act)):
        _check(t, n, s, io, dev)
    _check(A, "A", (d_inner, d_state), torch.float32, dev)
    _check(D, "D", (d_inner,), torch.float32, dev)
    _check(delta_bias, "delta_bias", (d_inner,), torch.float32, dev)
    num_slots = 0
    if state_indices is not None:
        _check(state_indices, "state_indices", (batch,), torch.int32, dev)
        caches = [t for t in (h0, h_final) if t is not None]
        num_slots = caches[0].shape[0] if caches else 1
    state_shape = (num_slots if state_indices is not None else batch, d_inner, d_state)
    _check(h0, "h0", state_shape, torch.float32, dev)
    _check(h_final, "h_final", state_shape, torch.float32, dev)
    ws, ws_bytes = _workspace(workspace, dev)
    if ckpt is not None:
        _check(ckpt, "ckpt", (batch, (seqlen + 15) // 16, d_inner, d_state), torch.float32, dev)
    return _lib.new_scan_params(
        batch=batch, seqlen=seqlen, d_inner=d_inner, d_state=d_state, io_dtype=_IO[io],
        delta_softplus=int(bool(delta_softplus)), x=_ptr(x), delta=_ptr(delta), z=_ptr(z),
        B=_ptr(B), C=_ptr(C), A=_ptr(A), D=_ptr(D), delta_bias=_ptr(delta_bias), h0=_ptr(h0),
        out=_ptr(out), h_final=_ptr(h_final), kernel_variant=int(variant),
        debug_flags=int(debug_flags), timeout_cycles=int(timeout_cycles),
        cu_seqlens=_ptr(cu_seqlens), total_tokens=int(total),
        state_indices=_ptr(state_indices), num_slots=int(num_slots), workspace=ws,
        workspace_bytes=ws_bytes, ckpt=_ptr(ckpt))


def jamba_ssm_scan(x, delta, z, B, C, A, D=None, delta_bias=None, delta_softplus=True,
                   h0=None, out=None, h_final=None, return_final_state=True, stream=None,
                   variant: int = 0, debug_flags: int = 0, timeout_cycles: int = 0,
                   cu_seqlens=None, state_indices=None, workspace=None, ckpt=None):
    """Prefill S6 scan.  Shapes: x, delta, z [batch, seqlen, d_inner] (bf16 or
    fp32), B, C [batch, seqlen, d_state] (same dtype), A [d_inner, d_state]
    fp32, D and delta_bias [d_inner] fp32 or None, h0 [batch, d_inner, d_state]
    fp32 or None.  Returns (out, h_final); h_final is None when
    return_final_state is False and no buffer was passed.

    Serving layouts: with ``cu_seqlens`` (int32 [batch + 1] on the device) the
    activations are packed [total_tokens, d_inner] / [total_tokens, d_state]
    and sequence b is rows cu_seqlens[b]:cu_seqlens[b+1].  With
    ``state_indices`` (int32 [batch]) h0 / h_final are [num_slots, d_inner,
    d_state] caches and sequence b uses row state_indices[b] (negative: zero
    initial state, nothing written); pass h_final explicitly in that case.

    ``workspace``: an optional zero-filled device tensor of at least
    ``jamba_ssm_scan_workspace_size(...)`` bytes that holds this call's status
    word (read with ``jamba_ssm_get_status(workspace=...)``).

    ``ckpt``: an optional fp32 device tensor [batch, ceil(seqlen / 16),
    d_inner, d_state] that receives the state before every 16th step, for a
    ``jamba_ssm_scan_bwd`` on the same inputs to take (batched layout only)."""
    if out is None:
        out = torch.empty_like(x)
    if h_final is None and return_final_state and state_indices is None:
        batch = cu_seqlens.numel() - 1 if cu_seqlens is not None else x.shape[0]
        h_final = torch.empty(batch, x.shape[-1], A.shape[-1], dtype=torch.float32,
                              device=x.device)
    p = _scan_params(x, delta, z, B, C, A, D, delta_bias, delta_softplus, h0, out, h_final,
                     variant, debug_flags, timeout_cycles, cu_seqlens, state_indices, workspace,
                     ckpt)
    st = _lib.call_scan(p, _stream(stream, x.device))
    if st != _lib.OK:
        raise JambaSSMError(st, "jamba_ssm_scan")
    return out, h_final


def jamba_ssm_scan_ckpt_size(batch: int, seqlen: int, d_inner: int, d_state: int) -> int:
    """Bytes of the checkpoints jamba_ssm_scan stores when given ``ckpt``."""
    return _lib.scan_ckpt_size(int(batch), int(seqlen), int(d_inner), int(d_state))


def jamba_ssm_scan_bwd_workspace_size(batch: int, seqlen: int, d_inner: int,
                                      d_state: int) -> int:
    """Bytes of the workspace the backward pass needs (0: d_state unsupported)."""
    return _lib.scan_bwd_workspace_size(int(batch), int(seqlen), int(d_inner), int(d_state))


def jamba_ssm_scan_bwd(x, delta, z, B, C, A, dout, D=None, delta_bias=None,
                       delta_softplus=True, h0=None, dh_final=None, workspace=None,
                       stream=None, debug_flags: int = 0, timeout_cycles: int = 0, ckpt=None):
    """Backward pass of jamba_ssm_scan: the gradients of a loss with respect to
    every input, given dout = dL/dout [batch, seqlen, d_inner] (the dtype of x)
    and optionally dh_final = dL/dh_final [batch, d_inner, d_state] fp32.

    Returns a dict: dx, ddelta, dz [batch, seqlen, d_inner] and dB, dC [batch,
    seqlen, d_state] in x's dtype; dA [d_inner, d_state], dD, ddelta_bias
    [d_inner] fp32 (summed over the batch); dh0 [batch, d_inner, d_state] fp32.
    ``workspace``: a device tensor of at least
    ``jamba_ssm_scan_bwd_workspace_size(...)`` bytes whose first 16 bytes are
    zero (allocated here when None; its status word is read with
    ``jamba_ssm_get_status(workspace=...)``).
    ``ckpt``: the checkpoints a ``jamba_ssm_scan(..., ckpt=...)`` on the same
    inputs stored; the backward then skips its own checkpoint pass."""
    if x.dtype not in _IO:
        raise TypeError(f"x must be bfloat16 or float32, got {x.dtype}")
    batch, seqlen, d_inner = x.shape
    d_state = A.shape[-1]
    dev, io = x.device, x.dtype
    act, bc = (batch, seqlen, d_inner), (batch, seqlen, d_state)
    for t, n, s in ((x, "x", act), (delta, "delta", act), (z, "z", act), (B, "B", bc),
                    (C, "C", bc), (dout, "dout", act)):
        _check(t, n, s, io, dev)
    _check(A, "A", (d_inner, d_state), torch.float32, dev)
    _check(D, "D", (d_inner,), torch.float32, dev)
    _check(delta_bias, "delta_bias", (d_inner,), torch.float32, dev)
    _check(h0, "h0", (batch, d_inner, d_state), torch.float32, dev)
    _check(dh_final, "dh_final", (batch, d_inner, d_state), torch.float32, dev)
    if ckpt is not None:
        _check(ckpt, "ckpt", (batch, (seqlen + 15) // 16, d_inner, d_state), torch.float32, dev)
    if workspace is None:
        need = jamba_ssm_scan_bwd_workspace_size(batch, seqlen, d_inner, d_state)
        workspace = torch.zeros(max(need, _lib.STATUS_BYTES), dtype=torch.uint8, device=dev)
    ws, ws_bytes = _workspace(workspace, dev)
    g = dict(dx=torch.empty_like(x), ddelta=torch.empty_like(x), dz=torch.empty_like(x),
             dB=torch.empty_like(B), dC=torch.empty_like(C),
             dA=torch.empty(d_inner, d_state, dtype=torch.float32, device=dev),
             dD=torch.empty(d_inner, dtype=torch.float32, device=dev),
             ddelta_bias=torch.empty(d_inner, dtype=torch.float32, device=dev),
             dh0=torch.empty(batch, d_inner, d_state, dtype=torch.float32, device=dev))
    p = _lib.new_scan_bwd_params(
        batch=batch, seqlen=seqlen, d_inner=d_inner, d_state=d_state, io_dtype=_IO[io],
        delta_softplus=int(bool(delta_softplus)), x=_ptr(x), delta=_ptr(delta), z=_ptr(z),
        B=_ptr(B), C=_ptr(C), A=_ptr(A), D=_ptr(D), delta_bias=_ptr(delta_bias), h0=_ptr(h0),
        dout=_ptr(dout), dh_final=_ptr(dh_final),
        **{k: _ptr(v) for k, v in g.items()},
        workspace=ws, workspace_bytes=ws_bytes, debug_flags=int(debug_flags),
        timeout_cycles=int(timeout_cycles), ckpt=_ptr(ckpt))
    st = _lib.call_scan_bwd(p, _stream(stream, dev))
    if st != _lib.OK:
        raise JambaSSMError(st, "jamba_ssm_scan_bwd")
    return g


def jamba_ssm_ssd_scan(x, delta, z, B, C, A, D=None, delta_bias=None, delta_softplus=True,
                       h0=None, out=None, h_final=None, return_final_state=True, stream=None,
                       debug_flags: int = 0, timeout_cycles: int = 0, workspace=None):
    """Scan of the scalar-identity (Mamba-2) variant.  x, z [batch, seqlen,
    nheads * headdim]; delta [batch, seqlen, nheads] (one step size per head);
    B, C [batch, seqlen, d_state]; A, delta_bias [nheads] fp32; D [nheads *
    headdim] fp32; h0 [batch, nheads * headdim, d_state] fp32.  Returns (out,
    h_final)."""
    if x.dtype not in _IO:
        raise TypeError(f"x must be bfloat16 or float32, got {x.dtype}")
    batch, seqlen, d_inner = x.shape
    nheads = A.shape[0]
    d_state = B.shape[-1]
    if nheads < 1 or d_inner % nheads:
        raise ValueError("d_inner must be a multiple of the number of heads")
    dev, io = x.device, x.dtype
    if out is None:
        out = torch.empty_like(x)
    if h_final is None and return_final_state:
        h_final = torch.empty(batch, d_inner, d_state, dtype=torch.float32, device=dev)
    for t, n, sh in ((x, "x", (batch, seqlen, d_inner)), (z, "z", (batch, seqlen, d_inner)),
                     (out, "out", (batch, seqlen, d_inner)),
                     (delta, "delta", (batch, seqlen, nheads)),
                     (B, "B", (batch, seqlen, d_state)), (C, "C", (batch, seqlen, d_state))):
        _check(t, n, sh, io, dev)
    _check(A, "A", (nheads,), torch.float32, dev)
    _check(delta_bias, "delta_bias", (nheads,), torch.float32, dev)
    _check(D, "D", (d_inner,), torch.float32, dev)
    _check(h0, "h0", (batch, d_inner, d_state), torch.float32, dev)
    _check(h_final, "h_final", (batch, d_inner, d_state), torch.float32, dev)
    ws, ws_bytes = _workspace(workspace, dev)
    p = _lib.new_ssd_params(
        batch=batch, seqlen=seqlen, nheads=nheads, headdim=d_inner // nheads, d_state=d_state,
        io_dtype=_IO[io], delta_softplus=int(bool(delta_softplus)), x=_ptr(x), delta=_ptr(delta),
        z=_ptr(z), B=_ptr(B), C=_ptr(C), A=_ptr(A), D=_ptr(D), delta_bias=_ptr(delta_bias),
        h0=_ptr(h0), out=_ptr(out), h_final=_ptr(h_final), workspace=ws, workspace_bytes=ws_bytes,
        debug_flags=int(debug_flags), timeout_cycles=int(timeout_cycles))
    st = _lib.call_ssd(p, _stream(stream, dev))
    if st != _lib.OK:
        raise JambaSSMError(st, "jamba_ssm_ssd_scan")
    return out, h_final


def scan_plan(x, A, B=None, variant: int = 0):
    """Launch shape the library picks for a scan of x's shape (no launch)."""
    batch, seqlen, d_inner = x.shape
    p = _lib.new_scan_params(batch=batch, seqlen=seqlen, d_inner=d_inner, d_state=A.shape[-1],
                             io_dtype=_IO[x.dtype], x=16, delta=16, z=16, B=16, C=16, A=16,
                             out=1 << 40, kernel_variant=int(variant))
    return _lib.scan_plan(p)


def jamba_ssm_state_update(state, x, delta, z, B, C, A, D=None, delta_bias=None,
                           delta_softplus=True, out=None, stream=None, state_indices=None,
                           debug_flags: int = 0, timeout_cycles: int = 0, workspace=None):
    """One decode step; `state` [batch, d_inner, d_state] fp32 is updated in
    place.  x, delta, z [batch, d_inner]; B, C [batch, d_state].  Returns out
    [batch, d_inner].  With ``state_indices`` (int32 [batch] on the device)
    `state` is a [num_slots, d_inner, d_state] cache and request b updates row
    state_indices[b]; a negative index skips the request (its out row is left
    as it was)."""
    if x.dtype not in _IO:
        raise TypeError(f"x must be bfloat16 or float32, got {x.dtype}")
    batch, d_inner = x.shape
    d_state = A.shape[-1]
    dev, io = x.device, x.dtype
    if out is None:
        out = torch.empty_like(x)
    for t, n, s in ((x, "x", (batch, d_inner)), (delta, "delta", (batch, d_inner)),
                    (z, "z", (batch, d_inner)), (B, "B", (batch, d_state)),
                    (C, "C", (batch, d_state)), (out, "out", (batch, d_inner))):
        _check(t, n, s, io, dev)
    num_slots = 0
    if state_indices is not None:
        _check(state_indices, "state_indices", (batch,), torch.int32, dev)
        num_slots = state.shape[0]
    _check(state, "state", (num_slots if state_indices is not None else batch, d_inner, d_state),
           torch.float32, dev)
    _check(A, "A", (d_inner, d_state), torch.float32, dev)
    _check(D, "D", (d_inner,), torch.float32, dev)
    _check(delta_bias, "delta_bias", (d_inner,), torch.float32, dev)
    ws, ws_bytes = _workspace(workspace, dev)
    p = _lib.new_state_update_params(
        batch=batch, d_inner=d_inner, d_state=d_state, io_dtype=_IO[io],
        delta_softplus=int(bool(delta_softplus)), state=_ptr(state), x=_ptr(x),
        delta=_ptr(delta), z=_ptr(z), B=_ptr(B), C=_ptr(C), A=_ptr(A), D=_ptr(D),
        delta_bias=_ptr(delta_bias), out=_ptr(out), state_indices=_ptr(state_indices),
        num_slots=int(num_slots), debug_flags=int(debug_flags),
        timeout_cycles=int(timeout_cycles), workspace=ws, workspace_bytes=ws_bytes)
    st = _lib.call_state_update(p, _stream(stream, dev))
    if st != _lib.OK:
        raise JambaSSMError(st, "jamba_ssm_state_update")
    return out


def jamba_ssm_get_status(stream=None, device=None, workspace=None) -> int:
    """Synchronize the stream and read-and-clear a status word: the
    workspace's, or the device's word of the library when none is given."""
    dev = torch.device(device) if device is not None else torch.device("cuda",
                                                                        torch.cuda.current_device())
    ws, _ = _workspace(workspace, workspace.device if workspace is not None else dev)
    return _lib.get_status(_stream(stream, dev), ws or 0)


def jamba_ssm_scan_workspace_size(batch: int, seqlen: int, d_inner: int, d_state: int) -> int:
    """Bytes of the optional workspace of a scan (its status block)."""
    return _lib.scan_workspace_size(int(batch), int(seqlen), int(d_inner), int(d_state))


def jamba_ssm_x_proj(u, W_x, w_dt=None, w_B=None, w_C=None, eps=1e-6, d_state=16,
                     k_split=0, timeout_cycles=0, stream=None, debug_flags=0):
    """[dt_low | B | C] = u @ W_x.T, each part RMS-normalised with its weight
    (None: not normalised).

    u: [..., d_inner] bf16; W_x: [dt_rank + 2 d_state, d_inner] bf16; weights
    fp32.  Returns (dt_low_hi, dt_low_lo, B, C): the two bf16 planes of dt_low
    [..., dt_rank] and B, C [..., d_state] bf16.
    """
    dev = u.device
    if dev.type != "cuda":
        raise ValueError("jamba_ssm_x_proj needs CUDA tensors; there is no CPU path")
    rows, d_inner = W_x.shape
    dt_rank = rows - 2 * d_state
    lead = tuple(u.shape[:-1])
    _check(u, "u", lead + (d_inner,), torch.bfloat16, dev)
    _check(W_x, "W_x", (rows, d_inner), torch.bfloat16, dev)
    _check(w_dt, "w_dt", (dt_rank,), torch.float32, dev)
    _check(w_B, "w_B", (d_state,), torch.float32, dev)
    _check(w_C, "w_C", (d_state,), torch.float32, dev)
    hi, lo = (torch.empty(lead + (dt_rank,), dtype=torch.bfloat16, device=dev) for _ in range(2))
    B, C = (torch.empty(lead + (d_state,), dtype=torch.bfloat16, device=dev) for _ in range(2))
    ntok = 1
    for n in lead:
        ntok *= n
    p = _lib.new_x_proj_params(ntok=ntok, d_inner=d_inner, dt_rank=dt_rank, d_state=d_state,
                               u=_ptr(u), W_x=_ptr(W_x), w_dt=_ptr(w_dt), w_B=_ptr(w_B),
                               w_C=_ptr(w_C), eps=float(eps), k_split=int(k_split),
                               dt_low_hi=_ptr(hi), dt_low_lo=_ptr(lo), B=_ptr(B), C=_ptr(C),
                               timeout_cycles=int(timeout_cycles), debug_flags=int(debug_flags))
    st = _lib.call_x_proj(p, _stream(stream, dev))
    if st != _lib.OK:
        raise JambaSSMError(st, "jamba_ssm_x_proj",
                            cuda_error=_lib.proj_lib().jamba_ssm_proj_last_cuda_error())
    return hi, lo, B, C


def jamba_ssm_dt_proj(dt_low_hi, W_dt, dt_low_lo=None, out=None, timeout_cycles=0, stream=None,
                      debug_flags=0):
    """delta = (dt_low_hi + dt_low_lo) @ W_dt.T in fp32, rounded once to bf16.

    dt_low_hi / dt_low_lo: [..., dt_rank] bf16, the two planes of the fp32
    dt_low (lo may be None); W_dt: [d_inner, dt_rank] bf16.  Returns delta
    [..., d_inner] bf16 (written into ``out`` when given).
    """
    dev = dt_low_hi.device
    if dev.type != "cuda":
        raise ValueError("jamba_ssm_dt_proj needs CUDA tensors; there is no CPU path")
    d_inner, dt_rank = W_dt.shape
    lead = tuple(dt_low_hi.shape[:-1])
    _check(dt_low_hi, "dt_low_hi", lead + (dt_rank,), torch.bfloat16, dev)
    _check(dt_low_lo, "dt_low_lo", lead + (dt_rank,), torch.bfloat16, dev)
    _check(W_dt, "W_dt", (d_inner, dt_rank), torch.bfloat16, dev)
    if out is None:
        out = torch.empty(lead + (d_inner,), dtype=torch.bfloat16, device=dev)
    _check(out, "out", lead + (d_inner,), torch.bfloat16, dev)
    ntok = 1
    for n in lead:
        ntok *= n
    p = _lib.new_dt_proj_params(ntok=ntok, d_inner=d_inner, dt_rank=dt_rank,
                                dt_low_hi=_ptr(dt_low_hi), dt_low_lo=_ptr(dt_low_lo),
                                W_dt=_ptr(W_dt), delta=_ptr(out),
                                timeout_cycles=int(timeout_cycles), debug_flags=int(debug_flags))
    st = _lib.call_dt_proj(p, _stream(stream, dev))
    if st != _lib.OK:
        raise JambaSSMError(st, "jamba_ssm_dt_proj",
                            cuda_error=_lib.proj_lib().jamba_ssm_proj_last_cuda_error())
    return out


def jamba_ssm_proj_get_status(stream=None, device=None):
    """Wait for the stream and return (and clear) the projection library's
    device-side status (0 = ok)."""
    dev = torch.device(device) if device is not None else torch.device("cuda",
                                                                        torch.cuda.current_device())
    return _lib.proj_get_status(_stream(stream, dev))
