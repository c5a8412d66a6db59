"""Parity of the scalar-identity (Mamba-2) scan kernel with the fp64 oracle's
ssd_scan (needs a B200), under the layer's comparison rules (tests/parity.py),
and its agreement with the diagonal scan kernel when the diagonal scan's
parameters are tied across each head."""
import os

import pytest
import torch

import oracle
from selective_state_space_26_b200 import (_lib, jamba_ssm_get_status, jamba_ssm_scan,
                                           jamba_ssm_ssd_scan, synth)
from tests.parity import BF16_REL_L2, assert_out, assert_state, compare_out, rel_l2

pytestmark = pytest.mark.gpu
THREADS = max(1, min(32, os.cpu_count() or 1))


def _dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda", 0)


def _gpu(inp, **kw):
    out, hf = jamba_ssm_ssd_scan(inp.x, inp.delta, inp.z, inp.B, inp.C, inp.A, D=inp.D,
                                 delta_bias=inp.delta_bias, delta_softplus=inp.delta_softplus,
                                 h0=inp.h0, **kw)
    torch.cuda.synchronize()
    if not kw.get("debug_flags", 0) & 1:  # no wait ran out
        assert jamba_ssm_get_status() == _lib.OK
    return out, hf


def _oracle(inp):
    return oracle.ssd_scan(inp.x, inp.delta, inp.z, inp.B, inp.C, inp.A, inp.A.shape[0],
                           D=inp.D, delta_bias=inp.delta_bias, delta_softplus=inp.delta_softplus,
                           h0=inp.h0, threads=THREADS)


@pytest.mark.parametrize("dtype,n", [(torch.bfloat16, 16), (torch.bfloat16, 8),
                                     (torch.float32, 16), (torch.float32, 8)])
def test_ssd_matches_oracle_ragged(dtype, n):
    """Several 64-step tiles and a ragged tail, 8 heads of 64 channels (two
    CTAs per head), two sequences, a nonzero initial state."""
    dev = _dev()
    inp = synth.ssd_inputs(2, 203, 8, 64, n, dtype, seed=71, device=dev, h0_std=0.5)
    out, hf = _gpu(inp)
    ref, ref_h = _oracle(inp)
    assert_out(out, ref, dtype, f"ssd {dtype} N={n}")
    assert_state(hf, ref_h, dtype, f"ssd {dtype} N={n}")


@pytest.mark.parametrize("seqlen", [1, 63, 64, 65])
def test_ssd_boundary_lengths_and_heads_of_32(seqlen):
    dev = _dev()
    inp = synth.ssd_inputs(1, seqlen, 16, 32, 16, torch.bfloat16, seed=72, device=dev, h0_std=0.3)
    out, hf = _gpu(inp)
    ref, ref_h = _oracle(inp)
    assert_out(out, ref, torch.bfloat16, f"L={seqlen}")
    assert_state(hf, ref_h, torch.bfloat16, f"L={seqlen}")


def test_ssd_without_softplus_split_and_empty():
    dev = _dev()
    inp = synth.ssd_inputs(1, 150, 8, 32, 16, torch.bfloat16, seed=73, device=dev, h0_std=0.3)
    inp.delta.copy_((inp.delta.float().abs() * 0.05).to(torch.bfloat16))
    inp.delta_bias.fill_(0.01)
    inp.delta_softplus = False
    out, hf = _gpu(inp)
    ref, ref_h = _oracle(inp)
    assert_out(out, ref, torch.bfloat16, "no softplus")
    # chunked: the first 70 steps, then the rest from their final state, is the whole scan
    cut = 70
    part = lambda t, sl: t[:, sl].contiguous()  # noqa: E731
    a = synth.SsdInputs(*(part(getattr(inp, k), slice(0, cut)) for k in ("x", "delta", "z", "B", "C")),
                        inp.A, inp.D, inp.delta_bias, inp.h0, False)
    o1, h1 = _gpu(a)
    b = synth.SsdInputs(*(part(getattr(inp, k), slice(cut, None)) for k in ("x", "delta", "z", "B", "C")),
                        inp.A, inp.D, inp.delta_bias, h1, False)
    o2, h2 = _gpu(b)
    assert torch.equal(torch.cat([o1, o2], 1), out) and torch.equal(h2, hf)
    e = synth.ssd_inputs(1, 0, 8, 32, 16, torch.bfloat16, seed=74, device=dev, h0_std=1.0)
    _, he = _gpu(e)
    assert torch.equal(he, e.h0)


def test_ssd_agrees_with_the_diagonal_kernel_on_tied_parameters():
    """The diagonal scan with A[d, n] = A[head(d)] and Delta[t, d] = Delta[t,
    head(d)] is the same map; the two kernels agree under the bf16 rule."""
    dev = _dev()
    H, P, N = 8, 64, 16
    inp = synth.ssd_inputs(1, 130, H, P, N, torch.bfloat16, seed=75, device=dev, h0_std=0.2)
    out, hf = _gpu(inp)
    head = torch.arange(H * P, device=dev) // P
    A_diag = inp.A[head][:, None].expand(H * P, N).contiguous()
    out_d, hf_d = jamba_ssm_scan(inp.x, inp.delta[:, :, head].contiguous(), inp.z, inp.B, inp.C,
                                 A_diag, D=inp.D, delta_bias=inp.delta_bias[head].contiguous(),
                                 h0=inp.h0)
    torch.cuda.synchronize()
    m = compare_out(out, out_d.double(), torch.bfloat16)
    assert m["ok"], m
    assert_state(hf, hf_d, torch.bfloat16, "tied parameters")


def test_ssd_full_size_jamba_width():
    """Jamba's layer width as 128 heads of 64 channels, d_state 16, 4096
    tokens: every output against the oracle."""
    dev = _dev()
    inp = synth.ssd_inputs(1, 4096, 128, 64, 16, torch.bfloat16, seed=76, device=dev)
    out, hf = _gpu(inp)
    ref, ref_h = _oracle(inp)
    assert_out(out, ref, torch.bfloat16, "ssd full size")
    assert_state(hf, ref_h, torch.bfloat16, "ssd full size")


def test_ssd_deterministic_and_timeout():
    dev = _dev()
    inp = synth.ssd_inputs(2, 140, 8, 32, 16, torch.bfloat16, seed=77, device=dev)
    a = _gpu(inp)
    b = _gpu(inp)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
    assert jamba_ssm_get_status() == _lib.OK
    _gpu(inp, debug_flags=1, timeout_cycles=2_000_000)
    assert jamba_ssm_get_status() == _lib.ERR_TIMEOUT
    assert jamba_ssm_get_status() == _lib.OK
    c = _gpu(inp)
    assert torch.equal(c[0], a[0])


# ---------------------------------------------------------------- chunked form
# bf16 I/O with d_state 16 and headdim 64 runs the chunked tensor-core kernel
# (128-token chunks); bit 1 of debug_flags forces the per-step kernel.

@pytest.mark.parametrize("batch,seqlen,h0_std", [(1, 1, 0.0), (2, 127, 0.5), (1, 128, 0.3),
                                                 (3, 129, 0.0), (2, 515, 0.4)])
def test_ssd_chunked_lengths_against_oracle(batch, seqlen, h0_std):
    """One token, a chunk short by one, exactly one chunk, one past it, and
    several chunks with a ragged tail; several sequences (one CTA per sequence
    and head), with and without an initial state."""
    dev = _dev()
    inp = synth.ssd_inputs(batch, seqlen, 8, 64, 16, torch.bfloat16, seed=80 + seqlen, device=dev,
                           h0_std=h0_std)
    out, hf = _gpu(inp)
    ref, ref_h = _oracle(inp)
    assert_out(out, ref, torch.bfloat16, f"chunked L={seqlen}")
    assert_state(hf, ref_h, torch.bfloat16, f"chunked L={seqlen}")


def test_ssd_chunked_and_per_step_kernels_agree():
    """The two kernels compute one map: each within the bf16 rule of the
    oracle and of each other, softplus on and off, 16 heads."""
    dev = _dev()
    for sp in (True, False):
        inp = synth.ssd_inputs(2, 300, 16, 64, 16, torch.bfloat16, seed=88, device=dev, h0_std=0.3)
        if not sp:  # Delta = delta + bias itself: keep it positive
            inp.delta.copy_((inp.delta.float().abs() * 0.05).to(torch.bfloat16))
            inp.delta_bias.fill_(0.01)
            inp.delta_softplus = False
        out_c, hf_c = _gpu(inp)
        out_s, hf_s = _gpu(inp, debug_flags=2)
        ref, ref_h = _oracle(inp)
        assert_out(out_c, ref, torch.bfloat16, f"chunked softplus={sp}")
        assert_out(out_s, ref, torch.bfloat16, f"per-step softplus={sp}")
        assert_state(hf_c, ref_h, torch.bfloat16, f"chunked softplus={sp}")
        # two bf16 results: the max-excess rule needs an exact reference, so
        # between the kernels only the rel-L2 part applies
        assert rel_l2(out_c, out_s) <= BF16_REL_L2
        assert_state(hf_c, hf_s, torch.bfloat16, "chunked vs per-step")


def test_ssd_chunked_strong_decay_and_split():
    """Steps large enough that e^{s_t - s_j} underflows inside a chunk (A down
    to -16, Delta near 1), and the sequence cut at a point that is not a chunk
    boundary and resumed from its final state: the concatenation is the whole
    scan up to fp32 rounding order."""
    dev = _dev()
    inp = synth.ssd_inputs(1, 400, 8, 64, 16, torch.bfloat16, seed=89, device=dev, h0_std=0.2)
    inp.A.copy_(-torch.linspace(0.5, 16.0, 8, device=dev))
    inp.delta_bias.fill_(0.5)
    out, hf = _gpu(inp)
    ref, ref_h = _oracle(inp)
    assert_out(out, ref, torch.bfloat16, "strong decay")
    assert_state(hf, ref_h, torch.bfloat16, "strong decay")
    cut = 200
    part = lambda t, sl: t[:, sl].contiguous()  # noqa: E731
    a = synth.SsdInputs(*(part(getattr(inp, k), slice(0, cut)) for k in ("x", "delta", "z", "B", "C")),
                        inp.A, inp.D, inp.delta_bias, inp.h0, True)
    o1, h1 = _gpu(a)
    b = synth.SsdInputs(*(part(getattr(inp, k), slice(cut, None)) for k in ("x", "delta", "z", "B", "C")),
                        inp.A, inp.D, inp.delta_bias, h1, True)
    o2, h2 = _gpu(b)
    assert_out(torch.cat([o1, o2], 1), ref, torch.bfloat16, "split at 200")
    assert_state(h2, ref_h, torch.bfloat16, "split at 200")


def test_ssd_chunked_deterministic_and_timeout():
    dev = _dev()
    inp = synth.ssd_inputs(2, 300, 8, 64, 16, torch.bfloat16, seed=90, device=dev)
    a = _gpu(inp)
    b = _gpu(inp)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
    assert jamba_ssm_get_status() == _lib.OK
    _gpu(inp, debug_flags=1, timeout_cycles=2_000_000)
    assert jamba_ssm_get_status() == _lib.ERR_TIMEOUT
    assert jamba_ssm_get_status() == _lib.OK
    c = _gpu(inp)
    assert torch.equal(c[0], a[0]) and torch.equal(c[1], a[1])


def test_ssd_chunked_degenerate_decays():
    """A = 0 on some heads (no decay: the state only accumulates, sigma stays
    at 0), and softplus off with Delta exactly 0 on whole stretches of tokens
    (the state and the decay sums do not move there), over exactly two chunks."""
    dev = _dev()
    inp = synth.ssd_inputs(1, 256, 8, 64, 16, torch.bfloat16, seed=91, device=dev, h0_std=0.3)
    inp.A[::2] = 0.0
    d = (inp.delta.float().abs() * 0.02).to(torch.bfloat16)
    d[:, 40:90] = 0.0
    d[:, 200:230] = 0.0
    inp.delta.copy_(d)
    inp.delta_bias.zero_()
    inp.delta_softplus = False
    out, hf = _gpu(inp)
    ref, ref_h = _oracle(inp)
    assert_out(out, ref, torch.bfloat16, "degenerate decays")
    assert_state(hf, ref_h, torch.bfloat16, "degenerate decays")


def test_ssd_chunked_more_ctas_than_sms():
    """4 sequences x 48 heads: 192 CTAs of one (sequence, head) each, more than
    the SMs, so the chunked kernel runs in two waves; sequences of 300 steps
    from different initial states."""
    dev = _dev()
    inp = synth.ssd_inputs(4, 300, 48, 64, 16, torch.bfloat16, seed=92, device=dev, h0_std=0.4)
    out, hf = _gpu(inp)
    ref, ref_h = _oracle(inp)
    assert_out(out, ref, torch.bfloat16, "two waves")
    assert_state(hf, ref_h, torch.bfloat16, "two waves")


def test_ssd_chunked_in_place_state_and_optional_inputs():
    """The chunked kernel with the state updated in place (h_final is h0), no
    skip term (D absent) and no bias; then the same call without a final state
    at all (the output alone)."""
    dev = _dev()
    inp = synth.ssd_inputs(2, 260, 8, 64, 16, torch.bfloat16, seed=93, device=dev, h0_std=0.4)
    ref, ref_h = oracle.ssd_scan(inp.x, inp.delta, inp.z, inp.B, inp.C, inp.A, 8, D=None,
                                 delta_bias=None, h0=inp.h0, threads=THREADS)
    h = inp.h0.clone()
    out, hf = jamba_ssm_ssd_scan(inp.x, inp.delta, inp.z, inp.B, inp.C, inp.A, h0=h, h_final=h)
    torch.cuda.synchronize()
    assert jamba_ssm_get_status() == _lib.OK
    assert hf.data_ptr() == h.data_ptr()
    assert_out(out, ref, torch.bfloat16, "in place")
    assert_state(h, ref_h, torch.bfloat16, "in place")
    out2, hf2 = jamba_ssm_ssd_scan(inp.x, inp.delta, inp.z, inp.B, inp.C, inp.A, h0=inp.h0,
                                   return_final_state=False)
    torch.cuda.synchronize()
    assert jamba_ssm_get_status() == _lib.OK
    assert hf2 is None and torch.equal(out2, out)


@pytest.mark.parametrize("headdim", [128, 192])
def test_ssd_chunked_wider_heads(headdim):
    """Heads of 128 and 192 channels run the chunked kernel as 2 or 3 CTAs per
    head, each a 64-channel slice repeating the head's per-token work."""
    dev = _dev()
    inp = synth.ssd_inputs(2, 300, 8, headdim, 16, torch.bfloat16, seed=94 + headdim, device=dev,
                           h0_std=0.3)
    out, hf = _gpu(inp)
    ref, ref_h = _oracle(inp)
    assert_out(out, ref, torch.bfloat16, f"headdim {headdim}")
    assert_state(hf, ref_h, torch.bfloat16, f"headdim {headdim}")
    out_s, _ = _gpu(inp, debug_flags=2)
    assert rel_l2(out, out_s) <= BF16_REL_L2
