"""Parity of the CUDA decode state update with the fp64 oracle (needs a B200)."""
import pytest
import torch

import oracle
from selective_state_space_26_b200 import jamba_ssm_scan, jamba_ssm_state_update, synth
from tests.parity import assert_out, assert_state, rel_l2

pytestmark = pytest.mark.gpu


def _dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda", 0)


def _params(d_inner, d_state, seed, dev, A_kind="mamba"):
    return (synth.make_A(d_inner, d_state, A_kind, seed).to(dev),
            torch.ones(d_inner, device=dev), synth.dt_bias_for(d_inner, seed).to(dev))


@pytest.mark.parametrize("dtype,n", [(torch.bfloat16, 16), (torch.bfloat16, 8),
                                     (torch.bfloat16, 4), (torch.float32, 16),
                                     (torch.float32, 4)])
def test_steps_match_oracle(dtype, n):
    dev = _dev()
    batch, d_inner = 5, 136
    A, D, bias = _params(d_inner, n, 21, dev, "random")
    st = synth.decode_state(batch, d_inner, n, seed=21, device=dev)
    ref_st = st.clone()
    for step in range(6):
        s = synth.decode_step(batch, d_inner, n, step, 21, dtype, dev)
        out = jamba_ssm_state_update(st, s.x, s.delta, s.z, s.B, s.C, A, D=D, delta_bias=bias)
        torch.cuda.synchronize()
        ref_out, ref_st = oracle.state_update(ref_st, s.x, s.delta, s.z, s.B, s.C, A, D=D,
                                              delta_bias=bias)
        assert_out(out, ref_out, dtype, f"step {step}")
        assert_state(st, ref_st, dtype, f"step {step}")


def test_decode_steps_equal_scan():
    """L calls of the decode update reproduce one prefill scan of length L."""
    dev = _dev()
    inp = synth.scan_inputs(3, 40, 128, 16, torch.bfloat16, seed=22, device=dev, h0_std=0.1)
    out_scan, h_scan = jamba_ssm_scan(inp.x, inp.delta, inp.z, inp.B, inp.C, inp.A, D=inp.D,
                                      delta_bias=inp.delta_bias, h0=inp.h0)
    st = inp.h0.clone()
    outs = []
    for t in range(40):
        outs.append(jamba_ssm_state_update(st, inp.x[:, t].contiguous(), inp.delta[:, t].contiguous(),
                                           inp.z[:, t].contiguous(), inp.B[:, t].contiguous(),
                                           inp.C[:, t].contiguous(), inp.A, D=inp.D,
                                           delta_bias=inp.delta_bias))
    torch.cuda.synchronize()
    o = torch.stack(outs, dim=1)
    # same inputs, same fp32 formulas; only the order of the C.h sum differs
    assert rel_l2(st, h_scan) < 1e-6
    diff = (o.float() - out_scan.float()).abs()
    assert float(diff.max()) <= 2 * float(out_scan.float().abs().max()) * 2 ** -8


def test_odd_sizes_and_ragged_grid():
    dev = _dev()
    batch, d_inner, n = 3, 37, 16  # total lanes not a multiple of the block
    A, D, bias = _params(d_inner, n, 23, dev)
    st = synth.decode_state(batch, d_inner, n, seed=23, device=dev)
    ref_st = st.clone()
    s = synth.decode_step(batch, d_inner, n, 0, 23, torch.bfloat16, dev)
    out = jamba_ssm_state_update(st, s.x, s.delta, s.z, s.B, s.C, A, D=D, delta_bias=bias)
    torch.cuda.synchronize()
    ref_out, ref_st = oracle.state_update(ref_st, s.x, s.delta, s.z, s.B, s.C, A, D=D,
                                          delta_bias=bias)
    assert_out(out, ref_out, torch.bfloat16)
    assert_state(st, ref_st, torch.bfloat16)


def test_bounded_wait_times_out_and_reports():
    """The bulk-copy decode kernel's waits are bounded: with each CTA's first
    load withheld (test hook) the call records TIMEOUT and leaves; the context
    stays usable and the next call matches the oracle."""
    from selective_state_space_26_b200 import _lib, jamba_ssm_get_status
    dev = _dev()
    A, D, bias = _params(128, 16, 3, dev)
    st = synth.decode_state(40, 128, 16, seed=3, device=dev)
    s = synth.decode_step(40, 128, 16, 0, 3, torch.bfloat16, dev)
    assert jamba_ssm_get_status() == _lib.OK
    work = st.clone()
    jamba_ssm_state_update(work, s.x, s.delta, s.z, s.B, s.C, A, D=D, delta_bias=bias,
                           debug_flags=1, timeout_cycles=2_000_000)
    assert jamba_ssm_get_status() == _lib.ERR_TIMEOUT
    assert jamba_ssm_get_status() == _lib.OK
    work = st.clone()
    out = jamba_ssm_state_update(work, s.x, s.delta, s.z, s.B, s.C, A, D=D, delta_bias=bias)
    torch.cuda.synchronize()
    ref_out, ref_st = oracle.state_update(st, s.x, s.delta, s.z, s.B, s.C, A, D=D, delta_bias=bias)
    assert_out(out, ref_out, torch.bfloat16, "after timeout")
    assert_state(work, ref_st, torch.bfloat16, "after timeout")
