"""Parity of the CUDA backward scan (training) with the fp64 oracle's scan_bwd
(needs a B200).

Every gradient is compared element by element on the same seeded inputs:
gradients of the bf16 (or fp32) inputs -- dx, ddelta, dz, dB, dC -- in the I/O
dtype under the layer's output rule (tests/parity.py); the fp32 gradients of
the parameters and of the initial state -- dA, dD, ddelta_bias, dh0 -- under
the rule for the fp32 state (rel-L2 <= 1e-4 with bf16 inputs, <= 1e-5 with fp32
inputs): the inputs are identical on both sides, so only fp32 rounding inside
the kernels differs, as for the forward's final state."""
import numpy as np
import pytest
import torch

import oracle
from selective_state_space_26_b200 import (_lib, jamba_ssm_get_status, jamba_ssm_scan,
                                           jamba_ssm_scan_bwd, jamba_ssm_scan_bwd_workspace_size,
                                           scan_plan, synth)
from tests.parity import assert_out, assert_state

pytestmark = pytest.mark.gpu
IO_GRADS = ("dx", "ddelta", "dz", "dB", "dC")
F32_GRADS = ("dA", "dD", "ddelta_bias", "dh0")


def _dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda", 0)


def _case(batch, seqlen, d_inner, d_state, dtype, seed, softplus=True, dh=True):
    dev = _dev()
    inp = synth.scan_inputs(batch, seqlen, d_inner, d_state, dtype, seed=seed, device=dev,
                            h0_std=0.5, A_kind="random")
    inp.delta_softplus = softplus
    if not softplus:  # Delta = delta + bias must stay positive and small
        inp.delta.copy_((inp.delta.float().abs() * 0.05).to(dtype))
        inp.delta_bias.fill_(0.01)
    g = torch.Generator(device=dev)
    g.manual_seed(seed + 7)
    dout = torch.randn(inp.x.shape, generator=g, device=dev).to(dtype)
    dh_final = torch.randn(batch, d_inner, d_state, generator=g, device=dev) if dh else None
    return inp, dout, dh_final


def _run(inp, dout, dh_final, **kw):
    out = jamba_ssm_scan_bwd(inp.x, inp.delta, inp.z, inp.B, inp.C, inp.A, dout, D=inp.D,
                             delta_bias=inp.delta_bias, delta_softplus=inp.delta_softplus,
                             h0=inp.h0, dh_final=dh_final, **kw)
    torch.cuda.synchronize()
    return out


def _oracle(inp, dout, dh_final):
    return oracle.scan_bwd(inp.x, inp.delta, inp.z, inp.B, inp.C, inp.A, dout, D=inp.D,
                           delta_bias=inp.delta_bias, delta_softplus=inp.delta_softplus,
                           h0=inp.h0, dh_final=dh_final)


def _compare(got, ref, dtype, what):
    for k in IO_GRADS:
        assert_out(got[k], ref[k], dtype, f"{what}: {k}")
    for k in F32_GRADS:
        assert_state(got[k], ref[k], dtype, f"{what}: {k}")


@pytest.mark.parametrize("dtype,n", [(torch.bfloat16, 16), (torch.bfloat16, 8),
                                     (torch.float32, 16), (torch.float32, 8),
                                     (torch.float32, 4)])
def test_backward_matches_oracle_ragged(dtype, n):
    """Several tiles, a partial last tile and a partial last 16-step segment
    (203 = 3 x 64 + 11 steps), a ragged channel group, two sequences (dA, dD and
    ddelta_bias are sums over them), random A, nonzero h0 and dL/dh_final."""
    d = 200 if dtype == torch.bfloat16 else 196
    inp, dout, dh = _case(2, 203, d, n, dtype, seed=61)
    _compare(_run(inp, dout, dh), _oracle(inp, dout, dh), dtype, f"bwd {dtype} N={n}")


@pytest.mark.parametrize("seqlen", [1, 15, 16, 17, 64, 65])
def test_backward_boundary_lengths(seqlen):
    inp, dout, dh = _case(1, seqlen, 112, 16, torch.bfloat16, seed=62 + seqlen)
    _compare(_run(inp, dout, dh), _oracle(inp, dout, dh), torch.bfloat16, f"L={seqlen}")


def test_backward_without_softplus_and_without_dh_final():
    inp, dout, _ = _case(2, 100, 64, 16, torch.bfloat16, seed=63, softplus=False)
    _compare(_run(inp, dout, None), _oracle(inp, dout, None), torch.bfloat16, "no softplus")


def test_backward_is_deterministic():
    """Every sum is taken in a fixed order (no atomics): the same bits twice."""
    inp, dout, dh = _case(2, 150, 256, 16, torch.bfloat16, seed=64)
    a = _run(inp, dout, dh)
    b = _run(inp, dout, dh)
    for k in a:
        assert torch.equal(a[k], b[k]), k


def test_backward_empty_sequence():
    inp, dout, dh = _case(2, 0, 64, 16, torch.bfloat16, seed=65)
    g = _run(inp, dout, dh)
    assert not torch.any(g["dA"]) and not torch.any(g["dD"]) and not torch.any(g["ddelta_bias"])
    assert torch.equal(g["dh0"], dh)


def test_backward_matches_autograd_of_the_forward_directional():
    """A directional check through the CUDA forward itself: the layer is
    linear in x (Delta, B, C, z do not depend on it), so with L = <dout,
    scan(x)>, <dL/dx, e> = (L(x + e) - L(x - e)) / 2 for any direction e, up to
    rounding; fp32 I/O on both sides."""
    dev = _dev()
    inp, dout, _ = _case(1, 80, 64, 16, torch.float32, seed=66, dh=False)
    g = _run(inp, dout, None)
    gen = torch.Generator(device=dev)
    gen.manual_seed(5)
    e = torch.randn(inp.x.shape, generator=gen, device=dev)
    s = 1.0

    def loss(xv):
        out, _ = jamba_ssm_scan(xv, inp.delta, inp.z, inp.B, inp.C, inp.A, D=inp.D,
                                delta_bias=inp.delta_bias, h0=inp.h0)
        return float((out.double() * dout.double()).sum())
    fd = (loss(inp.x + s * e) - loss(inp.x - s * e)) / (2 * s)
    an = float((g["dx"].double() * e.double()).sum())
    assert abs(fd - an) <= 1e-3 * max(1.0, abs(an)), (fd, an)


def test_backward_full_size_jamba_layer():
    """Jamba's layer, batch 1 x 4096 steps x d_inner 8192 x d_state 16, the
    launch the benchmark times: every gradient against the oracle."""
    inp, dout, dh = _case(1, 4096, 8192, 16, torch.bfloat16, seed=67)
    _compare(_run(inp, dout, dh), _oracle(inp, dout, dh), torch.bfloat16, "full size")


def test_backward_workspace_size_and_errors():
    dev = _dev()
    need = jamba_ssm_scan_bwd_workspace_size(1, 100, 64, 16)
    assert need > _lib.STATUS_BYTES
    assert jamba_ssm_scan_bwd_workspace_size(1, 100, 64, 3) == 0
    inp, dout, dh = _case(1, 100, 64, 16, torch.bfloat16, seed=68)
    small = torch.zeros(need - 256, dtype=torch.uint8, device=dev)
    with pytest.raises(Exception) as e:
        _run(inp, dout, dh, workspace=small)
    assert getattr(e.value, "status", None) == _lib.ERR_WORKSPACE


def test_backward_bounded_wait_times_out_and_reports():
    """A withheld tile makes the backward kernel's bounded waits run out: the
    status word of the workspace reads TIMEOUT, the context stays usable and
    the next call is correct."""
    dev = _dev()
    inp, dout, dh = _case(1, 200, 112, 16, torch.bfloat16, seed=69)
    ws = torch.zeros(jamba_ssm_scan_bwd_workspace_size(1, 200, 112, 16), dtype=torch.uint8,
                     device=dev)
    _run(inp, dout, dh, workspace=ws, debug_flags=1, timeout_cycles=2_000_000)
    assert jamba_ssm_get_status(workspace=ws) == _lib.ERR_TIMEOUT
    assert jamba_ssm_get_status(workspace=ws) == _lib.OK
    _compare(_run(inp, dout, dh, workspace=ws), _oracle(inp, dout, dh), torch.bfloat16,
             "after a timeout")
    assert jamba_ssm_get_status(workspace=ws) == _lib.OK


# ------------------------------------------ checkpoints stored by the forward
def _ckpt(inp):
    b, L, d = inp.x.shape
    return torch.full((b, (L + 15) // 16, d, inp.A.shape[-1]), float("nan"),
                      dtype=torch.float32, device=inp.x.device)


@pytest.mark.parametrize("dtype,n", [(torch.bfloat16, 16), (torch.bfloat16, 8),
                                     (torch.float32, 16), (torch.float32, 4)])
def test_forward_checkpoints_are_the_oracle_states_and_change_nothing(dtype, n):
    """jamba_ssm_scan with ckpt: out and h_final are the same bits as without;
    entry [b, k] is the state before step 16 k, which the oracle gives as the
    final state of the first 16 k steps (entry 0 is h0)."""
    d = 200 if dtype == torch.bfloat16 else 196
    inp, _, _ = _case(2, 203, d, n, dtype, seed=67)
    kw = dict(D=inp.D, delta_bias=inp.delta_bias, delta_softplus=inp.delta_softplus, h0=inp.h0)
    out0, hf0 = jamba_ssm_scan(inp.x, inp.delta, inp.z, inp.B, inp.C, inp.A, **kw)
    ck = _ckpt(inp)
    out1, hf1 = jamba_ssm_scan(inp.x, inp.delta, inp.z, inp.B, inp.C, inp.A, ckpt=ck, **kw)
    torch.cuda.synchronize()
    assert jamba_ssm_get_status() == _lib.OK
    assert torch.equal(out0, out1) and torch.equal(hf0, hf1)
    assert not torch.isnan(ck).any(), "a checkpoint was not written"
    refs = [inp.h0.cpu().double().numpy()]
    for k in range(1, ck.shape[1]):
        t = 16 * k
        sl = lambda v: v[:, :t].contiguous()  # noqa: E731
        _, hk = oracle.scan(sl(inp.x), sl(inp.delta), sl(inp.z), sl(inp.B), sl(inp.C), inp.A,
                            D=inp.D, delta_bias=inp.delta_bias,
                            delta_softplus=inp.delta_softplus, h0=inp.h0)
        refs.append(hk)
    ref = np.stack(refs, axis=1)
    assert_state(ck, ref, dtype, f"checkpoints {dtype} N={n}")


@pytest.mark.parametrize("dtype,n", [(torch.bfloat16, 16), (torch.float32, 8)])
def test_backward_takes_the_forward_checkpoints(dtype, n):
    """jamba_ssm_scan_bwd given the forward's checkpoints skips its own pass and
    returns the same bits."""
    d = 200 if dtype == torch.bfloat16 else 196
    inp, dout, dh = _case(2, 203, d, n, dtype, seed=68)
    ck = _ckpt(inp)
    jamba_ssm_scan(inp.x, inp.delta, inp.z, inp.B, inp.C, inp.A, D=inp.D,
                   delta_bias=inp.delta_bias, delta_softplus=inp.delta_softplus, h0=inp.h0,
                   ckpt=ck)
    a = _run(inp, dout, dh)
    b = _run(inp, dout, dh, ckpt=ck)
    assert jamba_ssm_get_status() == _lib.OK
    for k in IO_GRADS + F32_GRADS:
        assert torch.equal(a[k], b[k]), k


def test_training_step_at_the_headline_size():
    """Forward with checkpoints then backward with them, at Jamba's layer (one
    sequence of 4096 tokens, d_inner 8192, d_state 16): the same gradients, bit
    for bit, as the backward that makes its own checkpoints."""
    dev = _dev()
    w = synth.WORKLOADS["s6_prefill_bf16_b1_l4096_d8192_n16"]
    inp = synth.workload_inputs(w, device=dev)
    g = torch.Generator(device=dev)
    g.manual_seed(69)
    dout = torch.randn(inp.x.shape, generator=g, device=dev).to(w.dtype)
    ck = _ckpt(inp)
    out, hf = jamba_ssm_scan(inp.x, inp.delta, inp.z, inp.B, inp.C, inp.A, D=inp.D,
                             delta_bias=inp.delta_bias, ckpt=ck)
    out0, hf0 = jamba_ssm_scan(inp.x, inp.delta, inp.z, inp.B, inp.C, inp.A, D=inp.D,
                               delta_bias=inp.delta_bias)
    torch.cuda.synchronize()
    assert torch.equal(out, out0) and torch.equal(hf, hf0)
    kw = dict(D=inp.D, delta_bias=inp.delta_bias)
    a = jamba_ssm_scan_bwd(inp.x, inp.delta, inp.z, inp.B, inp.C, inp.A, dout, **kw)
    b = jamba_ssm_scan_bwd(inp.x, inp.delta, inp.z, inp.B, inp.C, inp.A, dout, ckpt=ck, **kw)
    torch.cuda.synchronize()
    assert jamba_ssm_get_status() == _lib.OK
    for k in IO_GRADS + F32_GRADS:
        assert torch.equal(a[k], b[k]), k


@pytest.mark.parametrize("variant", [1, 2, 5, 7, 8, 9, 10])
def test_forward_checkpoints_on_every_variant_that_stores_them(variant):
    """Each launch shape with a checkpoint-storing forward, forced: the output is
    the same bits as that variant's plain forward, and the checkpoints are the
    oracle's states (the 2-lane variants are the library's choice at batch >= 2
    and are not reached by the shapes above)."""
    info = _lib.variant_info(variant)
    dtype = torch.bfloat16 if info["io_dtype"] == _lib.BF16 else torch.float32
    n = info["d_state"]
    inp, _, _ = _case(2, 150, 256, n, dtype, seed=70 + variant)
    kw = dict(D=inp.D, delta_bias=inp.delta_bias, delta_softplus=inp.delta_softplus, h0=inp.h0,
              variant=variant)
    out0, hf0 = jamba_ssm_scan(inp.x, inp.delta, inp.z, inp.B, inp.C, inp.A, **kw)
    ck = _ckpt(inp)
    out1, hf1 = jamba_ssm_scan(inp.x, inp.delta, inp.z, inp.B, inp.C, inp.A, ckpt=ck, **kw)
    torch.cuda.synchronize()
    assert jamba_ssm_get_status() == _lib.OK
    assert torch.equal(out0, out1) and torch.equal(hf0, hf1)
    refs = [inp.h0.cpu().double().numpy()]
    for k in range(1, ck.shape[1]):
        sl = lambda v: v[:, :16 * k].contiguous()  # noqa: E731
        refs.append(oracle.scan(sl(inp.x), sl(inp.delta), sl(inp.z), sl(inp.B), sl(inp.C),
                                inp.A, D=inp.D, delta_bias=inp.delta_bias,
                                delta_softplus=inp.delta_softplus, h0=inp.h0)[1])
    assert_state(ck, np.stack(refs, axis=1), dtype, f"checkpoints, variant {variant}")


def test_backward_many_sequences_takes_the_two_lane_checkpoint_pass():
    """32 sequences of 1024 channels: the cost model picks the 2-lane variant
    for the backward's checkpoint pass (and for a forward storing checkpoints),
    with two tasks per persistent CTA; the gradients match the oracle and the
    forward's checkpoints give the same bits."""
    inp, dout, dh = _case(32, 70, 1024, 16, torch.bfloat16, seed=79)
    plan = scan_plan(inp.x, inp.A)
    assert plan["lanes_per_channel"] == 2, plan
    got = _run(inp, dout, dh)
    _compare(got, _oracle(inp, dout, dh), torch.bfloat16, "bwd, 16 sequences")
    ck = _ckpt(inp)
    jamba_ssm_scan(inp.x, inp.delta, inp.z, inp.B, inp.C, inp.A, D=inp.D,
                   delta_bias=inp.delta_bias, delta_softplus=inp.delta_softplus, h0=inp.h0,
                   ckpt=ck)
    again = _run(inp, dout, dh, ckpt=ck)
    for k in IO_GRADS + F32_GRADS:
        assert torch.equal(got[k], again[k]), k
