"""Parity of the CUDA prefill scan with the fp64 oracle (needs a B200).

Every case runs through the C ABI (the Python binding only marshals pointers)
on seeded synthetic inputs, copies the very same input tensors to the host for
the oracle, and applies the comparison rules of tests/parity.py.
"""
import os

import pytest
import torch

import oracle
from selective_state_space_26_b200 import (JambaSSMError, jamba_ssm_get_status, jamba_ssm_scan,
                                           scan_plan, synth)
from selective_state_space_26_b200 import _lib
from tests.parity import assert_out, assert_state

pytestmark = pytest.mark.gpu
THREADS = max(1, min(32, os.cpu_count() or 1))


def _dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda", 0)


def run_gpu(inp, variant=0, h0=None, out=None, h_final=None):
    out, hf = jamba_ssm_scan(inp.x, inp.delta, inp.z, inp.B, inp.C, inp.A, D=inp.D,
                             delta_bias=inp.delta_bias, delta_softplus=inp.delta_softplus,
                             h0=inp.h0 if h0 is None else h0, out=out, h_final=h_final,
                             variant=variant)
    torch.cuda.synchronize()
    return out, hf


def run_oracle(inp, channels=None):
    sel = slice(None) if channels is None else channels
    h0 = None if inp.h0 is None else inp.h0[:, sel]
    return oracle.scan(inp.x[:, :, sel], inp.delta[:, :, sel], inp.z[:, :, sel], inp.B, inp.C,
                       inp.A[sel], D=inp.D[sel], delta_bias=inp.delta_bias[sel],
                       delta_softplus=inp.delta_softplus, h0=h0, threads=THREADS)


def variants_for(dtype, n):
    out = []
    k = 1
    while True:
        info = _lib.variant_info(k)
        if info is None:
            return out
        if info["io_dtype"] == (_lib.BF16 if dtype == torch.bfloat16 else _lib.F32) and \
                info["d_state"] == n:
            out.append(k)
        k += 1


def test_tiny_fp32_workload_matches_oracle():
    dev = _dev()
    w = synth.WORKLOADS["s6_tiny_fp32_b1_l64_d16_n4"]
    inp = synth.workload_inputs(w, device=dev)
    out, hf = run_gpu(inp)
    ref, ref_h = run_oracle(inp)
    assert_out(out, ref, torch.float32, "tiny fp32")
    assert_state(hf, ref_h, torch.float32, "tiny fp32")


@pytest.mark.parametrize("dtype,n", [(torch.bfloat16, 16), (torch.bfloat16, 8),
                                     (torch.float32, 16), (torch.float32, 8),
                                     (torch.float32, 4)])
def test_every_variant_ragged_tiles(dtype, n):
    """Several time tiles plus a ragged tail, a ragged channel group, two
    sequences, a random (unstructured) A and a nonzero initial state."""
    dev = _dev()
    inp = synth.scan_inputs(2, 203, 200 if dtype == torch.bfloat16 else 196, n, dtype,
                            seed=101, device=dev, h0_std=0.5, A_kind="random")
    ref, ref_h = run_oracle(inp)
    vs = variants_for(dtype, n)
    assert vs, "no variant built for this dtype / d_state"
    for v in [0] + vs:
        out, hf = run_gpu(inp, variant=v)
        assert_out(out, ref, dtype, f"variant {v}")
        assert_state(hf, ref_h, dtype, f"variant {v}")


@pytest.mark.parametrize("seqlen", [1, 2, 63, 64, 65, 129])
def test_short_and_boundary_lengths(seqlen):
    dev = _dev()
    inp = synth.scan_inputs(3, seqlen, 136, 16, torch.bfloat16, seed=7, device=dev, h0_std=0.2)
    ref, ref_h = run_oracle(inp)
    for v in [0] + variants_for(torch.bfloat16, 16):
        out, hf = run_gpu(inp, variant=v)
        assert_out(out, ref, torch.bfloat16, f"L={seqlen} variant {v}")
        assert_state(hf, ref_h, torch.bfloat16, f"L={seqlen} variant {v}")


def test_empty_inputs():
    dev = _dev()
    inp = synth.scan_inputs(2, 0, 64, 16, torch.bfloat16, seed=3, device=dev, h0_std=1.0)
    hf = torch.full((2, 64, 16), float("nan"), device=dev)
    run_gpu(inp, h_final=hf)
    assert torch.equal(hf, inp.h0)
    inp0 = synth.scan_inputs(2, 0, 64, 16, torch.bfloat16, seed=3, device=dev)
    run_gpu(inp0, h_final=hf)
    assert not torch.any(hf)
    inpb = synth.scan_inputs(0, 16, 64, 16, torch.bfloat16, seed=3, device=dev)
    out, hfb = run_gpu(inpb)
    assert out.numel() == 0 and hfb.numel() == 0


def test_smaller_than_one_channel_tile():
    dev = _dev()
    inp = synth.scan_inputs(1, 70, 8, 16, torch.bfloat16, seed=5, device=dev)
    ref, ref_h = run_oracle(inp)
    for v in [0] + variants_for(torch.bfloat16, 16):
        out, hf = run_gpu(inp, variant=v)
        assert_out(out, ref, torch.bfloat16, f"d_inner=8 variant {v}")
        assert_state(hf, ref_h, torch.bfloat16, f"d_inner=8 variant {v}")


def test_delta_zero_limit_and_no_softplus():
    dev = _dev()
    inp = synth.scan_inputs(2, 77, 64, 16, torch.bfloat16, seed=9, device=dev, h0_std=1.0)
    inp.delta.zero_()
    inp.delta_bias.zero_()
    inp.delta_softplus = False
    out, hf = run_gpu(inp)
    assert torch.equal(hf, inp.h0)  # Abar = 1, Bbar x = 0: state untouched, bit for bit
    ref, _ = run_oracle(inp)
    assert_out(out, ref, torch.bfloat16, "Delta=0")


def test_split_scan_is_bitwise_whole_scan():
    """Chunked prefill: scan(L1) then scan(L2, h0 = h_final) == scan(L1 + L2)."""
    dev = _dev()
    inp = synth.scan_inputs(2, 300, 256, 16, torch.bfloat16, seed=11, device=dev, h0_std=0.3)
    whole, hw = run_gpu(inp)
    for cut in (1, 64, 100):
        a = synth.ScanInputs(inp.x[:, :cut].contiguous(), inp.delta[:, :cut].contiguous(),
                             inp.z[:, :cut].contiguous(), inp.B[:, :cut].contiguous(),
                             inp.C[:, :cut].contiguous(), inp.A, inp.D, inp.delta_bias, inp.h0)
        b = synth.ScanInputs(inp.x[:, cut:].contiguous(), inp.delta[:, cut:].contiguous(),
                             inp.z[:, cut:].contiguous(), inp.B[:, cut:].contiguous(),
                             inp.C[:, cut:].contiguous(), inp.A, inp.D, inp.delta_bias, None)
        o1, h1 = run_gpu(a)
        o2, h2 = run_gpu(b, h0=h1)
        assert torch.equal(torch.cat([o1, o2], dim=1), whole), cut
        assert torch.equal(h2, hw), cut


def test_resume_in_place():
    dev = _dev()
    inp = synth.scan_inputs(1, 50, 64, 16, torch.bfloat16, seed=12, device=dev, h0_std=0.3)
    _, expect = run_gpu(inp)
    st = inp.h0.clone()
    run_gpu(inp, h0=st, h_final=st)
    assert torch.equal(st, expect)


def test_deterministic():
    dev = _dev()
    inp = synth.scan_inputs(2, 150, 256, 16, torch.bfloat16, seed=13, device=dev)
    o1, h1 = run_gpu(inp)
    o2, h2 = run_gpu(inp)
    assert torch.equal(o1, o2) and torch.equal(h1, h2)


def test_large_activation_range():
    """Activations 1e3-1e4 (the pages report layer outputs up to ~4e6 before
    the activation penalty): nothing overflows in the fp32 path."""
    dev = _dev()
    inp = synth.scan_inputs(1, 130, 64, 16, torch.bfloat16, seed=14, device=dev)
    inp.x.mul_(2048.0)
    ref, ref_h = run_oracle(inp)
    out, hf = run_gpu(inp)
    assert torch.isfinite(out.float()).all()
    assert_out(out / 2048.0, ref / 2048.0, torch.bfloat16, "x scaled by 2048")
    assert_state(hf, ref_h, torch.bfloat16, "x scaled by 2048")


def test_argument_errors_do_not_launch():
    dev = _dev()
    inp = synth.scan_inputs(1, 16, 64, 16, torch.bfloat16, seed=15, device=dev)
    with pytest.raises(JambaSSMError) as e:  # out overlaps x
        jamba_ssm_scan(inp.x, inp.delta, inp.z, inp.B, inp.C, inp.A, out=inp.x)
    assert e.value.status == _lib.ERR_INVALID_ARG
    with pytest.raises(JambaSSMError) as e:  # variant built for another d_state
        jamba_ssm_scan(inp.x, inp.delta, inp.z, inp.B, inp.C, inp.A,
                       variant=variants_for(torch.bfloat16, 8)[0])
    assert e.value.status == _lib.ERR_UNSUPPORTED
    buf = torch.zeros(16 * 64 + 8, dtype=torch.bfloat16, device=dev)
    x8 = buf[1:1 + 16 * 64].view(1, 16, 64)  # 2-byte offset: not 16-byte aligned
    with pytest.raises(JambaSSMError) as e:
        jamba_ssm_scan(x8, inp.delta, inp.z, inp.B, inp.C, inp.A)
    assert e.value.status == _lib.ERR_MISALIGNED
    assert jamba_ssm_get_status() == _lib.OK


def test_bounded_wait_times_out_and_reports():
    """A tile load that never arrives (withheld on purpose) makes the bounded
    mbarrier wait run out: the kernel records TIMEOUT and returns; the context
    stays usable and the next call is correct."""
    dev = _dev()
    inp = synth.scan_inputs(1, 200, 128, 16, torch.bfloat16, seed=16, device=dev)
    assert jamba_ssm_get_status() == _lib.OK
    jamba_ssm_scan(inp.x, inp.delta, inp.z, inp.B, inp.C, inp.A, D=inp.D,
                   delta_bias=inp.delta_bias, debug_flags=1, timeout_cycles=2_000_000)
    assert jamba_ssm_get_status() == _lib.ERR_TIMEOUT
    assert jamba_ssm_get_status() == _lib.OK  # read-and-clear
    ref, _ = run_oracle(inp)
    out, _ = run_gpu(inp)
    assert_out(out, ref, torch.bfloat16, "after timeout")


def test_sync_check_environment_returns_device_conditions():
    """With JAMBA_SSM_SYNC_CHECK=1 a call waits for its kernel and returns the
    device-side condition it recorded (here a withheld tile's timeout) as its
    own status; a clean call returns OK.  Run in a child process because the
    variable is read once per process."""
    _dev()
    import subprocess
    import sys
    code = (
        "import torch\n"
        "from selective_state_space_26_b200 import synth, jamba_ssm_scan, JambaSSMError, _lib\n"
        "dev = torch.device('cuda', 0)\n"
        "inp = synth.scan_inputs(1, 100, 128, 16, torch.bfloat16, seed=3, device=dev)\n"
        "args = (inp.x, inp.delta, inp.z, inp.B, inp.C, inp.A)\n"
        "try:\n"
        "    jamba_ssm_scan(*args, debug_flags=1, timeout_cycles=2_000_000)\n"
        "    print('NO-ERROR')\n"
        "except JambaSSMError as e:\n"
        "    print('STATUS', e.status)\n"
        "jamba_ssm_scan(*args)\n"
        "print('CLEAN-OK')\n")
    env = dict(os.environ, JAMBA_SSM_SYNC_CHECK="1")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "-c", code], cwd=root, env=env, capture_output=True,
                       text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    assert f"STATUS {_lib.ERR_TIMEOUT}" in r.stdout, r.stdout
    assert "CLEAN-OK" in r.stdout, r.stdout


def test_launch_shape_for_jamba_layers():
    """The cost model picks narrow CTAs for one sequence, so its 8192 channels
    cover the SMs, and the cheapest per-step variant once the batch fills them."""
    dev = _dev()
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    A = torch.empty(8192, 16, device=dev)
    one = torch.empty(1, 4096, 8192, dtype=torch.bfloat16, device=dev)
    plan = scan_plan(one, A)
    assert plan["channels_per_cta"] == 56 and plan["lanes_per_channel"] == 4
    assert plan["grid"] == min(sms, 147) and plan["tasks"] == 147
    many = torch.empty(16, 64, 8192, dtype=torch.bfloat16, device=dev)
    plan = scan_plan(many, A)
    assert plan["channels_per_cta"] == 128 and plan["lanes_per_channel"] == 2
    assert plan["grid"] == sms and plan["tasks"] == 16 * 64
