"""Parity of the small-state kernels (d_state 1, 2 and 4 with bf16 I/O, 1 and 2
with fp32 I/O: B / C rows shorter than a 16-byte TMA row) and of the decode
update at d_state 1 and 2 with the fp64 oracle, through the C ABI; and the
status word kept in a caller's workspace (needs a B200)."""
import os

import pytest
import torch

import oracle
from selective_state_space_26_b200 import (_lib, jamba_ssm_get_status, jamba_ssm_scan,
                                           jamba_ssm_scan_workspace_size,
                                           jamba_ssm_state_update, scan_plan, synth)
from tests.parity import assert_out, assert_state

pytestmark = pytest.mark.gpu
THREADS = max(1, min(32, os.cpu_count() or 1))
SMALL = [(torch.bfloat16, 1), (torch.bfloat16, 2), (torch.bfloat16, 4),
         (torch.float32, 1), (torch.float32, 2)]


def _dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda", 0)


def _oracle(inp, h0=None):
    return oracle.scan(inp.x, inp.delta, inp.z, inp.B, inp.C, inp.A, D=inp.D,
                       delta_bias=inp.delta_bias, delta_softplus=inp.delta_softplus,
                       h0=inp.h0 if h0 is None else h0, threads=THREADS)


@pytest.mark.parametrize("dtype,n", SMALL)
@pytest.mark.parametrize("seqlen", [1, 17, 203])
def test_small_state_scan(dtype, n, seqlen):
    """Ragged lengths (partial register blocks of 8 steps and odd block
    counts), a ragged channel block, random A and a nonzero initial state."""
    dev = _dev()
    d = 200 if dtype == torch.bfloat16 else 196
    inp = synth.scan_inputs(3, seqlen, d, n, dtype, seed=41 + n, device=dev, h0_std=0.5,
                            A_kind="random")
    ref, ref_h = _oracle(inp)
    out, hf = jamba_ssm_scan(inp.x, inp.delta, inp.z, inp.B, inp.C, inp.A, D=inp.D,
                             delta_bias=inp.delta_bias, h0=inp.h0)
    torch.cuda.synchronize()
    assert_out(out, ref, dtype, f"small state {dtype} N={n} L={seqlen}")
    assert_state(hf, ref_h, dtype, f"small state {dtype} N={n} L={seqlen}")
    plan = scan_plan(inp.x, inp.A)
    assert plan["variant"] == 0 and plan["lanes_per_channel"] == 1


def test_small_state_no_softplus_and_empty():
    dev = _dev()
    inp = synth.scan_inputs(2, 40, 64, 2, torch.bfloat16, seed=5, device=dev, h0_std=1.0)
    inp.delta.zero_()
    inp.delta_bias.zero_()
    inp.delta_softplus = False
    out, hf = jamba_ssm_scan(inp.x, inp.delta, inp.z, inp.B, inp.C, inp.A, D=inp.D,
                             delta_bias=inp.delta_bias, delta_softplus=False, h0=inp.h0)
    torch.cuda.synchronize()
    assert torch.equal(hf, inp.h0)  # Delta = 0: the state is untouched
    ref, _ = _oracle(inp)
    assert_out(out, ref, torch.bfloat16, "Delta=0, N=2")
    e = synth.scan_inputs(2, 0, 64, 4, torch.bfloat16, seed=5, device=dev, h0_std=1.0)
    hf = torch.full((2, 64, 4), float("nan"), device=dev)
    jamba_ssm_scan(e.x, e.delta, e.z, e.B, e.C, e.A, h0=e.h0, h_final=hf)
    torch.cuda.synchronize()
    assert torch.equal(hf, e.h0)


def test_small_state_split_is_bitwise_whole():
    dev = _dev()
    inp = synth.scan_inputs(2, 100, 64, 4, torch.bfloat16, seed=6, device=dev, h0_std=0.3)
    whole, hw = jamba_ssm_scan(inp.x, inp.delta, inp.z, inp.B, inp.C, inp.A, D=inp.D,
                               delta_bias=inp.delta_bias, h0=inp.h0)
    cut = 37
    part = lambda t, s: t[:, s].contiguous()  # noqa: E731
    o1, h1 = jamba_ssm_scan(*(part(t, slice(0, cut)) for t in (inp.x, inp.delta, inp.z, inp.B,
                                                                inp.C)),
                            inp.A, D=inp.D, delta_bias=inp.delta_bias, h0=inp.h0)
    o2, h2 = jamba_ssm_scan(*(part(t, slice(cut, None)) for t in (inp.x, inp.delta, inp.z,
                                                                   inp.B, inp.C)),
                            inp.A, D=inp.D, delta_bias=inp.delta_bias, h0=h1)
    torch.cuda.synchronize()
    assert torch.equal(torch.cat([o1, o2], 1), whole) and torch.equal(h2, hw)


@pytest.mark.parametrize("dtype,n", SMALL)
def test_small_state_packed_and_slots(dtype, n):
    """Packed variable-length sequences (one empty) through state-cache slots,
    one of them negative (no cached state, nothing written)."""
    dev = _dev()
    lens = [23, 0, 9, 40]
    d = 64
    tot = sum(lens)
    full = synth.scan_inputs(len(lens), max(lens), d, n, dtype, seed=77, device=dev,
                             h0_std=0.5, A_kind="random")
    cat = lambda t: torch.cat([t[b, :m] for b, m in enumerate(lens)]).contiguous()  # noqa: E731
    cu = torch.tensor([0] + list(torch.tensor(lens).cumsum(0)), dtype=torch.int32, device=dev)
    slots = torch.tensor([5, 0, -1, 2], dtype=torch.int32, device=dev)
    cache = torch.randn(6, d, n, device=dev)
    h0c = cache.clone()
    out = torch.empty(tot, d, dtype=dtype, device=dev)
    jamba_ssm_scan(cat(full.x), cat(full.delta), cat(full.z), cat(full.B), cat(full.C), full.A,
                   D=full.D, delta_bias=full.delta_bias, h0=cache, h_final=cache, out=out,
                   cu_seqlens=cu, state_indices=slots)
    torch.cuda.synchronize()
    assert tot == cu[-1].item()
    row = 0
    for b, m in enumerate(lens):
        s = int(slots[b])
        h0 = h0c[s:s + 1] if s >= 0 else torch.zeros(1, d, n, device=dev)
        one = synth.ScanInputs(full.x[b:b + 1, :m], full.delta[b:b + 1, :m], full.z[b:b + 1, :m],
                               full.B[b:b + 1, :m], full.C[b:b + 1, :m], full.A, full.D,
                               full.delta_bias, h0)
        ref, ref_h = _oracle(one)
        if m:
            assert_out(out[row:row + m], ref[0], dtype, f"packed seq {b}")
        if s >= 0:
            assert_state(cache[s], ref_h[0], dtype, f"slot {s}")
        row += m
    untouched = [r for r in range(6) if r not in (5, 0, 2)]
    assert torch.equal(cache[untouched], h0c[untouched])


@pytest.mark.parametrize("dtype,n", [(torch.bfloat16, 1), (torch.bfloat16, 2),
                                     (torch.float32, 1), (torch.float32, 2),
                                     (torch.bfloat16, 4)])
def test_small_state_decode_steps(dtype, n):
    """Eight chained decode steps at d_state 1 and 2 (and bf16 4, the plain
    kernel) equal the oracle's chained steps; slots with padding skip."""
    dev = _dev()
    batch, d = 5, 72
    A = synth.make_A(d, n, "random", seed=3).to(dev)
    Dv = torch.ones(d, device=dev)
    bias = synth.dt_bias_for(d, 3).to(dev)
    st = synth.decode_state(batch, d, n, 9, device=dev)
    ref_st = st.cpu()
    for k in range(8):
        s = synth.decode_step(batch, d, n, k, 3, dtype, dev)
        o = jamba_ssm_state_update(st, s.x, s.delta, s.z, s.B, s.C, A, D=Dv, delta_bias=bias)
        torch.cuda.synchronize()
        ref_o, ref_st = oracle.state_update(ref_st, s.x, s.delta, s.z, s.B, s.C, A, D=Dv,
                                            delta_bias=bias)
        assert_out(o, ref_o, dtype, f"decode step {k}")
        assert_state(st, ref_st, dtype, f"decode step {k}")
    # slots: request 1 is padding (-1), the rest map to rows of a cache of 8
    cache = torch.randn(8, d, n, device=dev)
    before = cache.clone()
    slots = torch.tensor([7, -1, 0, 3, 4], dtype=torch.int32, device=dev)
    s = synth.decode_step(batch, d, n, 99, 3, dtype, dev)
    out = torch.full((batch, d), 7.0, dtype=dtype, device=dev)
    jamba_ssm_state_update(cache, s.x, s.delta, s.z, s.B, s.C, A, D=Dv, delta_bias=bias,
                           out=out, state_indices=slots)
    torch.cuda.synchronize()
    ref_o, ref_c = oracle.state_update_slots(before, s.x, s.delta, s.z, s.B, s.C, A,
                                             slots.cpu(), D=Dv, delta_bias=bias)
    assert torch.all(out[1] == 7.0)
    keep = [0, 2, 3, 4]
    assert_out(out[keep], ref_o[keep], dtype, "decode through slots")
    assert_state(cache, ref_c, dtype, "decode through slots")


def test_status_word_in_workspace():
    """A call given a workspace records its device-side condition (a withheld
    tile's timeout) there, not in the library's word; get_status on the
    workspace reads and clears it; workspace_size is the status block."""
    dev = _dev()
    assert jamba_ssm_scan_workspace_size(1, 200, 128, 16) == _lib.STATUS_BYTES
    ws = torch.zeros(_lib.STATUS_BYTES, dtype=torch.uint8, device=dev)
    inp = synth.scan_inputs(1, 200, 128, 16, torch.bfloat16, seed=16, device=dev)
    assert jamba_ssm_get_status() == _lib.OK
    jamba_ssm_scan(inp.x, inp.delta, inp.z, inp.B, inp.C, inp.A, D=inp.D,
                   delta_bias=inp.delta_bias, debug_flags=1, timeout_cycles=2_000_000,
                   workspace=ws)
    assert jamba_ssm_get_status() == _lib.OK  # the library's word saw nothing
    assert jamba_ssm_get_status(workspace=ws) == _lib.ERR_TIMEOUT
    assert jamba_ssm_get_status(workspace=ws) == _lib.OK  # read and cleared
    assert not torch.any(ws)
    # a clean call with the workspace is correct and leaves it clear
    out, hf = jamba_ssm_scan(inp.x, inp.delta, inp.z, inp.B, inp.C, inp.A, D=inp.D,
                             delta_bias=inp.delta_bias, workspace=ws)
    assert jamba_ssm_get_status(workspace=ws) == _lib.OK
    ref, ref_h = _oracle(inp)
    assert_out(out, ref, torch.bfloat16, "with a workspace")
    # a bad slot of a decode call given the workspace is recorded there
    st = torch.zeros(2, 64, 16, device=dev)
    s = synth.decode_step(2, 64, 16, 0, 1, torch.bfloat16, dev)
    jamba_ssm_state_update(st, s.x, s.delta, s.z, s.B, s.C, inp.A[:64].contiguous(),
                           state_indices=torch.tensor([0, 9], dtype=torch.int32, device=dev),
                           workspace=ws)
    assert jamba_ssm_get_status() == _lib.OK
    assert jamba_ssm_get_status(workspace=ws) == _lib.ERR_INVALID_ARG
