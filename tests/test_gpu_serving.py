"""Serving layouts of the two entry points (needs a B200), against the fp64
oracle run sequence by sequence and request by request:

* packed variable-length prefill: activations [total_tokens, d_inner], one
  sequence per cu_seqlens range, empty sequences included;
* state-cache slots: h0 / h_final (prefill) and the decode state addressed by
  state_indices into a cache with more rows than the batch, negative indices
  as padding, an out-of-range index reported through the status word.
"""
import numpy as np
import pytest
import torch

import oracle
from selective_state_space_26_b200 import (jamba_ssm_get_status, jamba_ssm_scan,
                                           jamba_ssm_state_update, synth)
from selective_state_space_26_b200 import _lib
from tests.parity import assert_out, assert_state
from tests.test_gpu_scan import THREADS, variants_for

pytestmark = pytest.mark.gpu


def _dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda", 0)


def _pack(inp, lengths, dev):
    """Sequence b = the first lengths[b] steps of batch row b, concatenated."""
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    cat = lambda t: torch.cat([t[b, :L] for b, L in enumerate(lengths)]).contiguous()
    return (torch.tensor(cu, device=dev), cat(inp.x), cat(inp.delta), cat(inp.z), cat(inp.B),
            cat(inp.C))


def _oracle_seq(inp, b, L, h0=None):
    """Oracle scan of sequence b over its first L steps (h0: [d_inner, d_state])."""
    if L == 0:
        hf = np.zeros(inp.A.shape, dtype=np.float64) if h0 is None else h0.double().cpu().numpy()
        return np.zeros((0, inp.x.shape[-1])), hf
    sl = lambda t: t[b:b + 1, :L]
    out, hf = oracle.scan(sl(inp.x), sl(inp.delta), sl(inp.z), sl(inp.B), sl(inp.C), inp.A,
                          D=inp.D, delta_bias=inp.delta_bias, delta_softplus=True,
                          h0=None if h0 is None else h0[None], threads=THREADS)
    return out[0], hf[0]


LENGTHS = [0, 1, 63, 64, 65, 200, 17, 128]


@pytest.mark.parametrize("dtype,n", [(torch.bfloat16, 16), (torch.bfloat16, 8),
                                     (torch.float32, 16), (torch.float32, 4)])
def test_packed_sequences_match_oracle(dtype, n):
    dev = _dev()
    d_inner = 200 if dtype == torch.bfloat16 else 196
    inp = synth.scan_inputs(len(LENGTHS), max(LENGTHS), d_inner, n, dtype, seed=31, device=dev,
                            h0_std=0.5, A_kind="random")
    cu, x, dt, z, B, C = _pack(inp, LENGTHS, dev)
    refs = [_oracle_seq(inp, b, L, inp.h0[b]) for b, L in enumerate(LENGTHS)]
    for v in [0] + variants_for(dtype, n):
        out, hf = jamba_ssm_scan(x, dt, z, B, C, inp.A, D=inp.D, delta_bias=inp.delta_bias,
                                 h0=inp.h0, cu_seqlens=cu, variant=v)
        torch.cuda.synchronize()
        for b, L in enumerate(LENGTHS):
            o0 = int(cu[b])
            if L:
                assert_out(out[o0:o0 + L], refs[b][0], dtype, f"variant {v} seq {b} (L={L})")
            assert_state(hf[b], refs[b][1], dtype, f"variant {v} seq {b} (L={L})")


def test_packed_equal_lengths_is_bitwise_the_batched_scan():
    dev = _dev()
    inp = synth.scan_inputs(3, 150, 136, 16, torch.bfloat16, seed=5, device=dev, h0_std=0.3)
    cu, x, dt, z, B, C = _pack(inp, [150, 150, 150], dev)
    for v in [0] + variants_for(torch.bfloat16, 16):
        ob, hb = jamba_ssm_scan(inp.x, inp.delta, inp.z, inp.B, inp.C, inp.A, D=inp.D,
                                delta_bias=inp.delta_bias, h0=inp.h0, variant=v)
        op, hp = jamba_ssm_scan(x, dt, z, B, C, inp.A, D=inp.D, delta_bias=inp.delta_bias,
                                h0=inp.h0, cu_seqlens=cu, variant=v)
        torch.cuda.synchronize()
        assert torch.equal(op, ob.reshape(-1, 136)), f"variant {v}"
        assert torch.equal(hp, hb), f"variant {v}"


def test_packed_prefill_into_a_state_cache():
    """h0 / h_final rows picked by state_indices from a 12-row cache, resumed in
    place; a negative index starts from zero and writes no state."""
    dev = _dev()
    lengths = [40, 0, 130, 64, 7]
    slots = [7, 2, -1, 11, 0]
    inp = synth.scan_inputs(len(lengths), max(lengths), 128, 16, torch.bfloat16, seed=8,
                            device=dev, A_kind="random")
    cu, x, dt, z, B, C = _pack(inp, lengths, dev)
    cache = synth.decode_state(12, 128, 16, seed=9, device=dev, std=0.5)
    before = cache.clone()
    idx = torch.tensor(slots, dtype=torch.int32, device=dev)
    out, _ = jamba_ssm_scan(x, dt, z, B, C, inp.A, D=inp.D, delta_bias=inp.delta_bias, h0=cache,
                            h_final=cache, cu_seqlens=cu, state_indices=idx)
    torch.cuda.synchronize()
    for b, (L, s) in enumerate(zip(lengths, slots)):
        ref_o, ref_h = _oracle_seq(inp, b, L, before[s] if s >= 0 else None)
        o0 = int(cu[b])
        if L:
            assert_out(out[o0:o0 + L], ref_o, torch.bfloat16, f"seq {b}")
        if s >= 0:
            assert_state(cache[s], ref_h, torch.bfloat16, f"seq {b}")
    untouched = [r for r in range(12) if r not in slots]
    assert torch.equal(cache[untouched], before[untouched])


def test_packed_all_empty_copies_states():
    dev = _dev()
    cache = synth.decode_state(6, 64, 16, seed=2, device=dev)
    final = torch.full_like(cache, float("nan"))
    idx = torch.tensor([4, -1, 1], dtype=torch.int32, device=dev)
    cu = torch.zeros(4, dtype=torch.int32, device=dev)
    x = torch.empty(0, 64, dtype=torch.bfloat16, device=dev)
    bc = torch.empty(0, 16, dtype=torch.bfloat16, device=dev)
    A = synth.make_A(64, 16).to(dev)
    jamba_ssm_scan(x, x, x, bc, bc, A, h0=cache, h_final=final, cu_seqlens=cu, state_indices=idx)
    torch.cuda.synchronize()
    assert torch.equal(final[[4, 1]], cache[[4, 1]])
    assert torch.isnan(final[[0, 2, 3, 5]]).all()


@pytest.mark.parametrize("dtype,n,d_inner", [(torch.bfloat16, 16, 136), (torch.bfloat16, 4, 40),
                                             (torch.float32, 16, 36)])
def test_decode_through_state_slots(dtype, n, d_inner):
    """Requests update cache rows state_indices[b]; the padded request (-1)
    leaves its out row and every other cache row untouched.  (bf16 with
    d_state 4 takes the plain-load kernel, the others the bulk-copy one.)"""
    dev = _dev()
    slots = [3, 9, -1, 0, 7, 4]
    cache = synth.decode_state(10, d_inner, n, seed=4, device=dev)
    A = synth.make_A(d_inner, n, "random", 4).to(dev)
    D = torch.ones(d_inner, device=dev)
    bias = synth.dt_bias_for(d_inner, 4).to(dev)
    idx = torch.tensor(slots, dtype=torch.int32, device=dev)
    init = cache.clone()
    ref = cache.double().cpu().numpy()  # fp64 chain of the live rows
    live = [b for b, r in enumerate(slots) if r >= 0]
    rows = [slots[b] for b in live]
    for step in range(3):
        s = synth.decode_step(len(slots), d_inner, n, step, 4, dtype, dev)
        out = torch.full((len(slots), d_inner), 7.0, dtype=dtype, device=dev)
        jamba_ssm_state_update(cache, s.x, s.delta, s.z, s.B, s.C, A, D=D, delta_bias=bias,
                               out=out, state_indices=idx)
        torch.cuda.synchronize()
        ref_out, new = oracle.state_update(ref[rows], s.x[live], s.delta[live], s.z[live],
                                           s.B[live], s.C[live], A, D=D, delta_bias=bias)
        ref[rows] = new
        assert_out(out[live], ref_out, dtype, f"step {step}")
        assert_state(cache[rows], new, dtype, f"step {step}")
        assert (out[2] == 7.0).all(), "the padded request's out row was written"
        untouched = [r for r in range(10) if r not in slots]
        assert torch.equal(cache[untouched], init[untouched])


def test_prefill_then_decode_through_the_cache():
    """A continuous batch: packed prefill writes each sequence's final state
    into its slot, decode steps continue from the slots; the outputs and
    states equal the oracle's scan of the whole sequences."""
    dev = _dev()
    lengths, slots, steps = [50, 0, 130], [4, 1, 2], 3
    d_inner, n = 64, 16
    total = [L + steps for L in lengths]
    inp = synth.scan_inputs(3, max(total), d_inner, n, torch.bfloat16, seed=12, device=dev,
                            A_kind="random")
    cu, x, dt, z, B, C = _pack(inp, lengths, dev)
    cache = torch.zeros(6, d_inner, n, device=dev)
    idx = torch.tensor(slots, dtype=torch.int32, device=dev)
    jamba_ssm_scan(x, dt, z, B, C, inp.A, D=inp.D, delta_bias=inp.delta_bias, h_final=cache,
                   cu_seqlens=cu, state_indices=idx)
    outs = []
    for k in range(steps):
        pick = lambda t: torch.stack([t[b, lengths[b] + k] for b in range(3)]).contiguous()
        outs.append(jamba_ssm_state_update(cache, pick(inp.x), pick(inp.delta), pick(inp.z),
                                           pick(inp.B), pick(inp.C), inp.A, D=inp.D,
                                           delta_bias=inp.delta_bias, state_indices=idx))
    torch.cuda.synchronize()
    for b in range(3):
        ref_o, ref_h = _oracle_seq(inp, b, total[b])
        got = torch.stack([o[b] for o in outs])
        assert_out(got, ref_o[lengths[b]:], torch.bfloat16, f"seq {b}")
        assert_state(cache[slots[b]], ref_h, torch.bfloat16, f"seq {b}")


def test_out_of_range_slot_is_reported_and_skipped():
    dev = _dev()
    jamba_ssm_get_status()
    cache = synth.decode_state(4, 64, 16, seed=1, device=dev)
    before = cache.clone()
    s = synth.decode_step(2, 64, 16, 0, 1, torch.bfloat16, dev)
    A = synth.make_A(64, 16).to(dev)
    out = torch.full((2, 64), 3.0, dtype=torch.bfloat16, device=dev)
    idx = torch.tensor([1, 4], dtype=torch.int32, device=dev)  # 4 is past the 4-row cache
    jamba_ssm_state_update(cache, s.x, s.delta, s.z, s.B, s.C, A, out=out, state_indices=idx)
    assert jamba_ssm_get_status() == _lib.ERR_INVALID_ARG
    assert jamba_ssm_get_status() == _lib.OK  # read and cleared
    assert (out[1] == 3.0).all()
    assert torch.equal(cache[[0, 2, 3]], before[[0, 2, 3]])
    assert not torch.equal(cache[1], before[1])
    # prefill: the out-of-range sequence starts from zero and writes no state
    inp = synth.scan_inputs(2, 20, 64, 16, torch.bfloat16, seed=3, device=dev)
    cache2 = torch.zeros(4, 64, 16, device=dev)
    jamba_ssm_scan(inp.x, inp.delta, inp.z, inp.B, inp.C, inp.A, h_final=cache2,
                   state_indices=torch.tensor([9, 2], dtype=torch.int32, device=dev))
    assert jamba_ssm_get_status() == _lib.ERR_INVALID_ARG
    assert (cache2[[0, 1, 3]] == 0).all() and (cache2[2] != 0).any()


def test_batched_layout_with_state_slots():
    """The batched [batch, seqlen, d_inner] layout with h0 / h_final in a
    cache: the serving kernel, checked against the oracle per sequence."""
    dev = _dev()
    slots = [5, -1, 0]
    inp = synth.scan_inputs(3, 90, 136, 16, torch.bfloat16, seed=14, device=dev,
                            A_kind="random")
    cache = synth.decode_state(6, 136, 16, seed=15, device=dev, std=0.4)
    final = torch.zeros_like(cache)
    idx = torch.tensor(slots, dtype=torch.int32, device=dev)
    out, _ = jamba_ssm_scan(inp.x, inp.delta, inp.z, inp.B, inp.C, inp.A, D=inp.D,
                            delta_bias=inp.delta_bias, h0=cache, h_final=final,
                            state_indices=idx)
    torch.cuda.synchronize()
    for b, s in enumerate(slots):
        ref_o, ref_h = _oracle_seq(inp, b, 90, cache[s] if s >= 0 else None)
        assert_out(out[b], ref_o, torch.bfloat16, f"seq {b}")
        if s >= 0:
            assert_state(final[s], ref_h, torch.bfloat16, f"seq {b}")
    assert (final[[1, 2, 3, 4]] == 0).all()


def test_serving_kernel_bounded_wait_times_out_and_reports():
    """The serving kernel's waits are bounded too: with each task's first tile
    withheld (test hook) the call records TIMEOUT, and the next call is correct."""
    dev = _dev()
    lengths = [70, 0, 33]
    inp = synth.scan_inputs(3, 70, 128, 16, torch.bfloat16, seed=17, device=dev)
    cu, x, dt, z, B, C = _pack(inp, lengths, dev)
    assert jamba_ssm_get_status() == _lib.OK
    jamba_ssm_scan(x, dt, z, B, C, inp.A, D=inp.D, delta_bias=inp.delta_bias, cu_seqlens=cu,
                   debug_flags=1, timeout_cycles=2_000_000)
    assert jamba_ssm_get_status() == _lib.ERR_TIMEOUT
    assert jamba_ssm_get_status() == _lib.OK
    out, hf = jamba_ssm_scan(x, dt, z, B, C, inp.A, D=inp.D, delta_bias=inp.delta_bias,
                             cu_seqlens=cu)
    torch.cuda.synchronize()
    for b, L in enumerate(lengths):
        ref_o, ref_h = _oracle_seq(inp, b, L)
        o0 = int(cu[b])
        if L:
            assert_out(out[o0:o0 + L], ref_o, torch.bfloat16, f"seq {b}")
        assert_state(hf[b], ref_h, torch.bfloat16, f"seq {b}")
