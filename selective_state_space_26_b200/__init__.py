"""B200-native Mamba-1 selective scan (S6): Python binding of the C ABI.

Two calls, with the names of the C entry points:

* ``jamba_ssm_scan``          -- prefill scan over whole sequences, returning the
  gated output and (for the decode cache) the final state;
* ``jamba_ssm_state_update``  -- one-token decode step, state updated in place.

Every step of the computation runs in the CUDA kernels of libjamba_ssm.so; this
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


def _scan_params(x, delta, z, B, C, A, D, delta_bias, delta_softplus, h0, out, h_final,
                 variant, debug_flags, timeout_cycles):
    if x.dtype not in _IO:
        raise TypeError(f"x must be bfloat16 or float32, got {x.dtype}")
    batch, seqlen, d_inner = x.shape
    d_state = A.shape[-1]
    dev = x.device
    io = x.dtype
    for t, n, s in ((x, "x", (batch, seqlen, d_inner)), (delta, "delta", (batch, seqlen, d_inner)),
                    (z, "z", (batch, seqlen, d_inner)), (B, "B", (batch, seqlen, d_state)),
                    (C, "C", (batch, seqlen, d_state)), (out, "out", (batch, seqlen, d_inner))):
        _check(t, n, s, io, dev)
    _check(A, "A", (d_inner, d_state), torch.float32, dev)
    _check(D, "D", (d_inner,), torch.float32, dev)
    _check(delta_bias, "delta_bias", (d_inner,), torch.float32, dev)
    _check(h0, "h0", (batch, d_inner, d_state), torch.float32, dev)
    _check(h_final, "h_final", (batch, d_inner, d_state), torch.float32, dev)
    return _lib.new_scan_params(
        batch=batch, seqlen=seqlen, d_inner=d_inner, d_state=d_state, io_dtype=_IO[io],
        delta_softplus=int(bool(delta_softplus)), x=_ptr(x), delta=_ptr(delta), z=_ptr(z),
        B=_ptr(B), C=_ptr(C), A=_ptr(A), D=_ptr(D), delta_bias=_ptr(delta_bias), h0=_ptr(h0),
        out=_ptr(out), h_final=_ptr(h_final), kernel_variant=int(variant),
        debug_flags=int(debug_flags), timeout_cycles=int(timeout_cycles))


def jamba_ssm_scan(x, delta, z, B, C, A, D=None, delta_bias=None, delta_softplus=True,
                   h0=None, out=None, h_final=None, return_final_state=True, stream=None,
                   variant: int = 0, debug_flags: int = 0, timeout_cycles: int = 0):
    """Prefill S6 scan.  Shapes: x, delta, z [batch, seqlen, d_inner] (bf16 or
    fp32), B, C [batch, seqlen, d_state] (same dtype), A [d_inner, d_state]
    fp32, D and delta_bias [d_inner] fp32 or None, h0 [batch, d_inner, d_state]
    fp32 or None.  Returns (out, h_final); h_final is None when
    return_final_state is False and no buffer was passed."""
    if out is None:
        out = torch.empty_like(x)
    if h_final is None and return_final_state:
        h_final = torch.empty(x.shape[0], x.shape[2], A.shape[-1], dtype=torch.float32,
                              device=x.device)
    p = _scan_params(x, delta, z, B, C, A, D, delta_bias, delta_softplus, h0, out, h_final,
                     variant, debug_flags, timeout_cycles)
    st = _lib.call_scan(p, _stream(stream, x.device))
    if st != _lib.OK:
        raise JambaSSMError(st, "jamba_ssm_scan")
    return out, h_final


def scan_plan(x, A, B=None, variant: int = 0):
    """Launch shape the library picks for a scan of x's shape (no launch)."""
    batch, seqlen, d_inner = x.shape
    p = _lib.new_scan_params(batch=batch, seqlen=seqlen, d_inner=d_inner, d_state=A.shape[-1],
                             io_dtype=_IO[x.dtype], x=16, delta=16, z=16, B=16, C=16, A=16,
                             out=1 << 40, kernel_variant=int(variant))
    return _lib.scan_plan(p)


def jamba_ssm_state_update(state, x, delta, z, B, C, A, D=None, delta_bias=None,
                           delta_softplus=True, out=None, stream=None):
    """One decode step; `state` [batch, d_inner, d_state] fp32 is updated in
    place.  x, delta, z [batch, d_inner]; B, C [batch, d_state].  Returns out
    [batch, d_inner]."""
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
    _check(state, "state", (batch, d_inner, d_state), torch.float32, dev)
    _check(A, "A", (d_inner, d_state), torch.float32, dev)
    _check(D, "D", (d_inner,), torch.float32, dev)
    _check(delta_bias, "delta_bias", (d_inner,), torch.float32, dev)
    p = _lib.new_state_update_params(
        batch=batch, d_inner=d_inner, d_state=d_state, io_dtype=_IO[io],
        delta_softplus=int(bool(delta_softplus)), state=_ptr(state), x=_ptr(x),
        delta=_ptr(delta), z=_ptr(z), B=_ptr(B), C=_ptr(C), A=_ptr(A), D=_ptr(D),
        delta_bias=_ptr(delta_bias), out=_ptr(out))
    st = _lib.call_state_update(p, _stream(stream, dev))
    if st != _lib.OK:
        raise JambaSSMError(st, "jamba_ssm_state_update")
    return out


def jamba_ssm_get_status(stream=None, device=None) -> int:
    """Synchronize the stream and read-and-clear the device status word."""
    dev = torch.device(device) if device is not None else torch.device("cuda",
                                                                        torch.cuda.current_device())
    return _lib.get_status(_stream(stream, dev))
