"""The backward pass for callers that cannot allocate device memory
(jamba_ssm_scan_bwd_noalloc, needs a B200).

Some callers cannot call cudaMalloc where they run the backward pass -- a
plug-in whose host framework owns every device allocation, or a path where the
allocator's implicit device synchronisation is not acceptable.  This entry
point takes its scratch from a fixed array the library keeps on every device.
The test calls it through the C ABI (ctypes, no Python wrapper) twice in a row,
with different sizes, and checks each result against the usual entry point,
jamba_ssm_scan_bwd with a caller workspace, under the comparison rules the
other GPU tests use (tests/parity.py).  It lives in a file that pytest collects
last and needs nothing from the other tests, so it passes alone in a fresh
process as well as after them."""
import ctypes

import pytest
import torch

from selective_state_space_26_b200 import (_lib, jamba_ssm_get_status, jamba_ssm_scan_bwd,
                                           jamba_ssm_scan_bwd_workspace_size, synth)
from tests.parity import compare_out, compare_state

pytestmark = pytest.mark.gpu
IO_GRADS = ("dx", "ddelta", "dz", "dB", "dC")
F32_GRADS = ("dA", "dD", "ddelta_bias", "dh0")
SCRATCH_BYTES = 64 * 1024 * 1024  # JAMBA_SSM_BWD_NOALLOC_SCRATCH_BYTES


def _case(batch, seqlen, d_inner, d_state, dtype, seed):
    dev = torch.device("cuda", 0)
    inp = synth.scan_inputs(batch, seqlen, d_inner, d_state, dtype, seed=seed, device=dev,
                            h0_std=0.5, A_kind="random")
    g = torch.Generator(device=dev)
    g.manual_seed(seed + 1)
    dout = torch.randn(inp.x.shape, generator=g, device=dev).to(dtype)
    dh = torch.randn(batch, d_inner, d_state, generator=g, device=dev)
    return inp, dout, dh


def _params(inp, dout, dh, grads, **kw):
    b, l, d = inp.x.shape
    n = inp.A.shape[1]
    ptr = lambda t: None if t is None else t.data_ptr()  # noqa: E731
    fields = dict(batch=b, seqlen=l, d_inner=d, d_state=n,
                  io_dtype=_lib.BF16 if inp.x.dtype == torch.bfloat16 else _lib.F32,
                  delta_softplus=1, x=ptr(inp.x), delta=ptr(inp.delta), z=ptr(inp.z),
                  B=ptr(inp.B), C=ptr(inp.C), A=ptr(inp.A), D=ptr(inp.D),
                  delta_bias=ptr(inp.delta_bias), h0=ptr(inp.h0), dout=ptr(dout),
                  dh_final=ptr(dh), **{k: ptr(v) for k, v in grads.items()})
    fields.update(kw)
    return _lib.new_scan_bwd_params(**fields)


def _noalloc(inp, dout, dh):
    """One call of jamba_ssm_scan_bwd_noalloc through the C ABI."""
    dev = inp.x.device
    x = inp.x
    b, l, d = x.shape
    n = inp.A.shape[1]
    grads = dict(dx=torch.empty_like(x), ddelta=torch.empty_like(x), dz=torch.empty_like(x),
                 dB=torch.empty_like(inp.B), dC=torch.empty_like(inp.C),
                 dA=torch.empty(d, n, device=dev), dD=torch.empty(d, device=dev),
                 ddelta_bias=torch.empty(d, device=dev), dh0=torch.empty(b, d, n, device=dev))
    p = _params(inp, dout, dh, grads)
    stream = ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)
    st = _lib.lib().jamba_ssm_scan_bwd_noalloc(ctypes.byref(p), stream)
    assert st == _lib.OK, _lib.status_string(st)
    torch.cuda.synchronize()
    return grads


def _same_as_workspace_path(got, inp, dout, dh, what):
    ref = jamba_ssm_scan_bwd(inp.x, inp.delta, inp.z, inp.B, inp.C, inp.A, dout, D=inp.D,
                             delta_bias=inp.delta_bias, h0=inp.h0, dh_final=dh)
    torch.cuda.synchronize()
    for k in IO_GRADS:
        m = compare_out(got[k], ref[k].double(), inp.x.dtype)
        assert m["ok"], (what, k, m)
    for k in F32_GRADS:
        m = compare_state(got[k], ref[k], inp.x.dtype)
        assert m["ok"], (what, k, m)


def test_backward_without_a_workspace_matches_the_workspace_path():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    assert jamba_ssm_get_status() == _lib.OK
    # call 1: two sequences, several tiles and a ragged end, bf16
    a = _case(2, 203, 200, 16, torch.bfloat16, seed=91)
    _same_as_workspace_path(_noalloc(*a), *a, "first call")
    # call 2, straight after, on other sizes and dtype: the array holds call
    # 1's contents, which must not leak into this result
    b = _case(1, 150, 196, 8, torch.float32, seed=92)
    assert jamba_ssm_scan_bwd_workspace_size(1, 150, 196, 8) <= SCRATCH_BYTES
    _same_as_workspace_path(_noalloc(*b), *b, "second call")
    assert jamba_ssm_get_status() == _lib.OK


def test_backward_without_a_workspace_rejects_what_it_cannot_hold():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    a = _case(1, 16, 64, 16, torch.bfloat16, seed=93)
    L = _lib.lib()
    # sizes whose scratch exceeds the fixed array: a clear error, nothing enqueued
    big = _params(*a, {}, seqlen=1 << 20, d_inner=8192)
    assert jamba_ssm_scan_bwd_workspace_size(1, 1 << 20, 8192, 16) > SCRATCH_BYTES
    assert L.jamba_ssm_scan_bwd_noalloc(ctypes.byref(big), None) == _lib.ERR_WORKSPACE
    # a caller workspace is not taken by this call
    ws = _params(*a, {}, workspace=0x10000, workspace_bytes=1 << 20)
    assert L.jamba_ssm_scan_bwd_noalloc(ctypes.byref(ws), None) == _lib.ERR_INVALID_ARG
    # a state size the backward does not take
    bad = _params(*a, {}, d_state=3)
    assert L.jamba_ssm_scan_bwd_noalloc(ctypes.byref(bad), None) == _lib.ERR_UNSUPPORTED
