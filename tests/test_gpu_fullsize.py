"""Parity at the full workload sizes, in the launch configuration the benchmark
times (the library's automatic variant choice), against the fp64 oracle on all
outputs (4K prefill) or on sampled channels over every step and sequence (256K
and batched 16K prefill), and on sampled requests over all 128 decode steps.
Channels are independent recurrences, so a sampled channel's oracle result is
exact, not an approximation.
"""
import os

import numpy as np
import pytest
import torch

import oracle
from selective_state_space_26_b200 import jamba_ssm_scan, jamba_ssm_state_update, synth
from tests.parity import assert_out, assert_state

pytestmark = pytest.mark.gpu
THREADS = max(1, min(64, os.cpu_count() or 1))


def _dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda", 0)


def sample_channels(d_inner, k_random=24, seed=0):
    """Both edges of every 64-channel block boundary near the ends, plus random ones."""
    edge = [0, 1, 7, 8, 15, 16, 31, 32, 63, 64, 127, 128, d_inner // 2, d_inner - 129,
            d_inner - 65, d_inner - 64, d_inner - 2, d_inner - 1]
    rnd = np.random.default_rng(seed).choice(d_inner, k_random, replace=False).tolist()
    return sorted(set(c for c in edge + rnd if 0 <= c < d_inner))


def _oracle_on_channels(inp, ch):
    idx = torch.tensor(ch, device=inp.x.device)
    sel = lambda t: t.index_select(2, idx)  # noqa: E731
    return oracle.scan(sel(inp.x), sel(inp.delta), sel(inp.z), inp.B, inp.C,
                       inp.A.index_select(0, idx), D=inp.D.index_select(0, idx),
                       delta_bias=inp.delta_bias.index_select(0, idx), threads=THREADS), idx


def test_prefill_4k_all_outputs():
    dev = _dev()
    w = synth.WORKLOADS["s6_prefill_bf16_b1_l4096_d8192_n16"]
    inp = synth.workload_inputs(w, device=dev)
    out, hf = jamba_ssm_scan(inp.x, inp.delta, inp.z, inp.B, inp.C, inp.A, D=inp.D,
                             delta_bias=inp.delta_bias)
    torch.cuda.synchronize()
    ref, ref_h = oracle.scan(inp.x, inp.delta, inp.z, inp.B, inp.C, inp.A, D=inp.D,
                             delta_bias=inp.delta_bias, threads=THREADS)
    m = assert_out(out, ref, torch.bfloat16, w.name)
    assert_state(hf, ref_h, torch.bfloat16, w.name)
    print(w.name, m)


@pytest.mark.parametrize("name", ["s6_prefill_bf16_b1_l262144_d8192_n16",
                                  "s6_prefill_bf16_b16_l16384_d8192_n16"])
def test_prefill_long_sampled_channels(name):
    dev = _dev()
    w = synth.WORKLOADS[name]
    inp = synth.workload_inputs(w, device=dev)
    out, hf = jamba_ssm_scan(inp.x, inp.delta, inp.z, inp.B, inp.C, inp.A, D=inp.D,
                             delta_bias=inp.delta_bias)
    torch.cuda.synchronize()
    ch = sample_channels(w.d_inner, seed=w.seed)
    (ref, ref_h), idx = _oracle_on_channels(inp, ch)
    m = assert_out(out.index_select(2, idx), ref, torch.bfloat16, name)
    assert_state(hf.index_select(1, idx), ref_h, torch.bfloat16, name)
    print(name, len(ch), "channels", m)
    del inp, out, hf
    torch.cuda.empty_cache()


def test_decode_256_requests_128_steps_sampled_requests():
    dev = _dev()
    w = synth.WORKLOADS["s6_decode_bf16_b256_d8192_n16_x128"]
    A = synth.make_A(w.d_inner, w.d_state).to(dev)
    D = torch.ones(w.d_inner, device=dev)
    bias = synth.dt_bias_for(w.d_inner, w.seed).to(dev)
    st = synth.decode_state(w.batch, w.d_inner, w.d_state, w.seed, device=dev)
    req = torch.tensor([0, 1, 77, 128, 254, 255], device=dev)
    ref_st = st.index_select(0, req).cpu()
    worst = {}
    for step in range(w.seqlen):
        s = synth.decode_step(w.batch, w.d_inner, w.d_state, step, w.seed, w.dtype, dev)
        out = jamba_ssm_state_update(st, s.x, s.delta, s.z, s.B, s.C, A, D=D, delta_bias=bias)
        pick = lambda t: t.index_select(0, req)  # noqa: E731
        ref_out, ref_st = oracle.state_update(ref_st, pick(s.x), pick(s.delta), pick(s.z),
                                              pick(s.B), pick(s.C), A, D=D, delta_bias=bias)
        m = assert_out(pick(out), ref_out, torch.bfloat16, f"decode step {step}")
        worst = max(worst, m, key=lambda d: d.get("rel_l2", 0.0)) if worst else m
    torch.cuda.synchronize()
    assert_state(st.index_select(0, req), ref_st, torch.bfloat16, "decode final state")
    print("decode worst step", worst)
