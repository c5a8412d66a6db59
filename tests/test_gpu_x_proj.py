"""Parity of the tensor-core x_proj kernel ([dt_low | B | C] = W_x u with the
three RMSNorms, split over d_inner across a thread-block cluster) with the fp64
oracle, the composed projection -> scan against the oracle's composition, and
the bounded-wait timeout paths of both projection kernels (needs a B200).

dt_low is an fp32 quantity delivered as two bf16 planes: hi + lo is compared
with the oracle's dt_low under the fp32 rule (rel-L2 <= 1e-5).  B and C are
bf16 outputs and take the bf16 rule of tests/parity.py."""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import oracle
from selective_state_space_26_b200 import (_lib, jamba_ssm_dt_proj,
                                           jamba_ssm_proj_get_status, jamba_ssm_scan,
                                           jamba_ssm_x_proj, synth)
from tests.parity import assert_out, round_bf16, to_np

pytestmark = pytest.mark.gpu
R, N = 256, 16


def _dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda", 0)


def _oracle(inp, rows=None, norms=True):
    u = to_np(inp.u) if rows is None else to_np(inp.u)[rows]
    d_inner = u.shape[-1]
    W_dt = np.zeros((d_inner, R))  # dt_low is compared directly; Delta is not needed here
    _, B, C, dt_low = oracle.project(u, to_np(inp.W_x), W_dt, N,
                                     w_dt=inp.w_dt if norms else None,
                                     w_B=inp.w_B if norms else None,
                                     w_C=inp.w_C if norms else None, threads=8,
                                     return_dt_low=True)
    return dt_low, B, C


def _check(hi, lo, B, C, ref, what):
    dt_low, rB, rC = ref
    assert_out(hi.float() + lo.float(), dt_low, torch.float32, f"{what}: dt_low")
    assert_out(B, rB, torch.bfloat16, f"{what}: B")
    assert_out(C, rC, torch.bfloat16, f"{what}: C")


def _run(inp, k_split, norms=True, **kw):
    out = jamba_ssm_x_proj(inp.u, inp.W_x, w_dt=inp.w_dt if norms else None,
                           w_B=inp.w_B if norms else None, w_C=inp.w_C if norms else None,
                           k_split=k_split, **kw)
    assert jamba_ssm_proj_get_status() == 0
    return out


def test_x_proj_one_cta_per_tile_first():
    """k_split = 1 (no cluster reduction): the tcgen05 path alone, on a ragged
    token count (128 + 72) and a ragged K (d_inner 776: 12 full 64-wide blocks
    and 8 zero-filled columns)."""
    dev = _dev()
    inp = synth.x_proj_inputs(200, 776, R, N, seed=51, device=dev)
    _check(*_run(inp, 1), _oracle(inp), "k_split 1")


@pytest.mark.parametrize("k_split", [2, 4, 8])
def test_x_proj_cluster_split(k_split):
    """The d_inner reduction through distributed shared memory; at 8 the last
    CTA of each cluster gets an empty K slice (13 blocks over 8 CTAs)."""
    dev = _dev()
    inp = synth.x_proj_inputs(200, 776, R, N, seed=52, device=dev)
    _check(*_run(inp, k_split), _oracle(inp), f"k_split {k_split}")


def test_x_proj_without_norms_and_tiny():
    dev = _dev()
    inp = synth.x_proj_inputs(200, 512, R, N, seed=53, device=dev)
    _check(*_run(inp, 4, norms=False), _oracle(inp, norms=False), "no norms")
    one = synth.x_proj_inputs(1, 8, R, N, seed=54, device=dev)
    _check(*_run(one, 0), _oracle(one), "1 token, d_inner 8")


def test_x_proj_full_size_sampled_rows():
    """4096 tokens x d_inner 8192 (Jamba's layer) at the library's own split:
    the first token tile and a seeded sample of rows from the others."""
    dev = _dev()
    inp = synth.x_proj_inputs(4096, 8192, R, N, seed=55, device=dev)
    hi, lo, B, C = _run(inp, 0)
    rng = np.random.default_rng(55)
    rows = np.concatenate([np.arange(128), np.sort(rng.choice(np.arange(128, 4096), 64,
                                                              replace=False))])
    idx = torch.as_tensor(rows, device=dev)
    _check(hi[idx], lo[idx], B[idx], C[idx], _oracle(inp, rows=rows), "full size")


def test_x_proj_is_deterministic():
    """The cluster reduction adds the K slices in a fixed order: same bits."""
    dev = _dev()
    inp = synth.x_proj_inputs(300, 1024, R, N, seed=56, device=dev)
    a = _run(inp, 4)
    b = _run(inp, 4)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_projection_then_scan_matches_the_oracle_composition():
    """x_proj -> dt_proj -> scan through the three C entry points, against
    oracle.project followed by oracle.scan.  The scan's ABI carries Delta_raw,
    B and C in bf16, so the oracle composition rounds them once (RNE) at that
    interface, exactly where the library's data path does."""
    dev = _dev()
    L, D = 200, 512
    xp = synth.x_proj_inputs(L, D, R, N, seed=57, device=dev)
    dp = synth.dt_proj_inputs(1, D, R, seed=57, device=dev)  # for W_dt only
    sc = synth.scan_inputs(1, L, D, N, torch.bfloat16, seed=57, device=dev, A_kind="random")
    hi, lo, B, C = jamba_ssm_x_proj(xp.u, xp.W_x, w_dt=xp.w_dt, w_B=xp.w_B, w_C=xp.w_C)
    delta = jamba_ssm_dt_proj(hi, dp.W_dt, dt_low_lo=lo)
    out, hf = jamba_ssm_scan(xp.u.view(1, L, D), delta.view(1, L, D), sc.z, B.view(1, L, N),
                             C.view(1, L, N), sc.A, D=sc.D, delta_bias=sc.delta_bias)
    torch.cuda.synchronize()
    assert jamba_ssm_proj_get_status() == 0
    r_delta, r_B, r_C = oracle.project(to_np(xp.u), to_np(xp.W_x), to_np(dp.W_dt), N,
                                       w_dt=xp.w_dt, w_B=xp.w_B, w_C=xp.w_C, threads=8)
    ref, ref_h = oracle.scan(to_np(xp.u)[None], round_bf16(r_delta)[None], sc.z,
                             round_bf16(r_B)[None], round_bf16(r_C)[None], sc.A, D=sc.D,
                             delta_bias=sc.delta_bias, threads=8)
    assert_out(delta, r_delta, torch.bfloat16, "composed: Delta_raw")
    assert_out(out, ref, torch.bfloat16, "composed: layer output")


@pytest.mark.parametrize("dt_rank", [256, 320])
def test_dt_proj_bounded_wait_times_out_and_reports(dt_rank):
    """A withheld operand block makes the MMA thread's bounded wait run out:
    TIMEOUT is recorded, the CTAs drain their loads and write nothing, the
    context stays usable and the next call is correct.  dt_rank 256 runs the
    persistent kernel, 320 the one-tile kernel."""
    dev = _dev()
    inp = synth.dt_proj_inputs(300, 776, dt_rank, seed=58, device=dev)
    assert jamba_ssm_proj_get_status() == 0
    out = torch.full((300, 776), 7.0, dtype=torch.bfloat16, device=dev)
    jamba_ssm_dt_proj(inp.hi, inp.W_dt, dt_low_lo=inp.lo, out=out, debug_flags=1,
                      timeout_cycles=2_000_000)
    assert jamba_ssm_proj_get_status() == _lib.ERR_TIMEOUT
    assert jamba_ssm_proj_get_status() == 0  # read and cleared
    assert torch.all(out == 7.0), "a timed-out tile was written"
    good = jamba_ssm_dt_proj(inp.hi, inp.W_dt, dt_low_lo=inp.lo)
    assert jamba_ssm_proj_get_status() == 0
    assert_out(good, oracle.dt_proj(to_np(inp.hi) + to_np(inp.lo), to_np(inp.W_dt), threads=8),
               torch.bfloat16, "dt_proj after a timeout")


@pytest.mark.parametrize("k_split", [1, 4])
def test_x_proj_bounded_wait_times_out_and_reports(k_split):
    dev = _dev()
    inp = synth.x_proj_inputs(200, 776, R, N, seed=59, device=dev)
    assert jamba_ssm_proj_get_status() == 0
    jamba_ssm_x_proj(inp.u, inp.W_x, w_dt=inp.w_dt, w_B=inp.w_B, w_C=inp.w_C, k_split=k_split,
                     debug_flags=1, timeout_cycles=2_000_000)
    assert jamba_ssm_proj_get_status() == _lib.ERR_TIMEOUT
    assert jamba_ssm_proj_get_status() == 0
    _check(*_run(inp, k_split), _oracle(inp), f"x_proj after a timeout, k_split {k_split}")


def test_proj_sync_check_environment_returns_device_conditions():
    """With JAMBA_SSM_SYNC_CHECK=1 the projection calls wait for their kernel
    and return its device-side condition themselves (child process: the
    variable is read once per process)."""
    _dev()
    code = (
        "import torch\n"
        "from selective_state_space_26_b200 import synth, jamba_ssm_x_proj, jamba_ssm_dt_proj, "
        "JambaSSMError\n"
        "dev = torch.device('cuda', 0)\n"
        "x = synth.x_proj_inputs(200, 512, 256, 16, seed=3, device=dev)\n"
        "d = synth.dt_proj_inputs(200, 512, 256, seed=3, device=dev)\n"
        "for f, a in ((jamba_ssm_x_proj, (x.u, x.W_x)), (jamba_ssm_dt_proj, (d.hi, d.W_dt))):\n"
        "    try:\n"
        "        f(*a, debug_flags=1, timeout_cycles=2_000_000)\n"
        "        print('NO-ERROR')\n"
        "    except JambaSSMError as e:\n"
        "        print('STATUS', e.status)\n"
        "    f(*a)\n"
        "print('CLEAN-OK')\n")
    env = dict(os.environ, JAMBA_SSM_SYNC_CHECK="1")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "-c", code], cwd=root, env=env, capture_output=True,
                       text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.count(f"STATUS {_lib.ERR_TIMEOUT}") == 2, r.stdout
    assert "CLEAN-OK" in r.stdout, r.stdout
