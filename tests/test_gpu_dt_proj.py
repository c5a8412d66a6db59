"""Parity of the tensor-core dt_proj kernel (the low-rank product that produces
the scan's raw Delta) with the fp64 oracle (needs a B200).

The oracle is given hi + lo, the exact value the kernel's two bf16 planes
represent, so the comparison sees only the kernel's own arithmetic (fp32
accumulation, one bf16 rounding) under the layer's bf16 rule."""
import numpy as np
import pytest
import torch

import oracle
from selective_state_space_26_b200 import jamba_ssm_dt_proj, jamba_ssm_proj_get_status, synth
from tests.parity import assert_out, to_np

pytestmark = pytest.mark.gpu


def _dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda", 0)


def _ref(inp, rows=None, lo=True):
    hi = to_np(inp.hi)
    a = hi + to_np(inp.lo) if lo else hi
    if rows is not None:
        a = a[rows]
    return oracle.dt_proj(a, to_np(inp.W_dt), threads=8)


# token counts and widths that leave ragged tiles on every axis: 300 tokens =
# 2 full 128-token tiles + 44; 776 channels = 6 full 128-channel tiles + 8;
# dt_rank 200 = 3 full 64-wide K blocks + 8 (zero-filled by TMA).  Ranks up to
# 256 run the persistent kernel (planes resident, W_dt through a 3-stage
# ring); 320 runs the one-tile kernel's 2-stage ring through two and a half
# passes
@pytest.mark.parametrize("ntok,d_inner,dt_rank", [(300, 776, 256), (300, 776, 200),
                                                  (1, 8, 8), (128, 256, 64), (257, 512, 320)])
def test_dt_proj_matches_oracle(ntok, d_inner, dt_rank):
    dev = _dev()
    inp = synth.dt_proj_inputs(ntok, d_inner, dt_rank, seed=31, device=dev)
    out = jamba_ssm_dt_proj(inp.hi, inp.W_dt, dt_low_lo=inp.lo)
    assert jamba_ssm_proj_get_status() == 0
    assert_out(out, _ref(inp), torch.bfloat16, f"dt_proj {ntok}x{d_inner}x{dt_rank}")


def test_dt_proj_hi_plane_only():
    dev = _dev()
    inp = synth.dt_proj_inputs(300, 776, 256, seed=32, device=dev)
    out = jamba_ssm_dt_proj(inp.hi, inp.W_dt)
    assert jamba_ssm_proj_get_status() == 0
    assert_out(out, _ref(inp, lo=False), torch.bfloat16, "dt_proj hi only")


def test_dt_proj_writes_only_its_rows_and_columns():
    dev = _dev()
    inp = synth.dt_proj_inputs(130, 264, 64, seed=33, device=dev)
    big = torch.full((131, 264), 7.0, dtype=torch.bfloat16, device=dev)
    jamba_ssm_dt_proj(inp.hi, inp.W_dt, dt_low_lo=inp.lo, out=big[:130])
    torch.cuda.synchronize()
    assert torch.all(big[130] == 7.0), "a row past ntok was written"
    assert_out(big[:130], _ref(inp), torch.bfloat16, "dt_proj in a larger buffer")


def test_dt_proj_empty_batch():
    dev = _dev()
    inp = synth.dt_proj_inputs(1, 256, 256, seed=34, device=dev)
    out = jamba_ssm_dt_proj(inp.hi[:0], inp.W_dt, dt_low_lo=inp.lo[:0])
    assert out.shape == (0, 256)
    assert jamba_ssm_proj_get_status() == 0


def test_dt_proj_full_size_sampled_rows():
    """4096 tokens x d_inner 8192 x dt_rank 256 (Jamba's sizes), the launch the
    timing uses; the oracle checks the first token tile and a seeded sample of
    rows from every other tile."""
    dev = _dev()
    inp = synth.dt_proj_inputs(4096, 8192, 256, seed=35, device=dev)
    out = jamba_ssm_dt_proj(inp.hi, inp.W_dt, dt_low_lo=inp.lo)
    assert jamba_ssm_proj_get_status() == 0
    rng = np.random.default_rng(35)
    rows = np.concatenate([np.arange(128), np.sort(rng.choice(np.arange(128, 4096), 96,
                                                              replace=False))])
    got = out[torch.as_tensor(rows, device=dev)]
    assert_out(got, _ref(inp, rows=rows), torch.bfloat16, "dt_proj full size")


def test_dt_proj_is_deterministic():
    """A fixed MMA order and no atomics: two launches give the same bits."""
    dev = _dev()
    inp = synth.dt_proj_inputs(300, 776, 256, seed=36, device=dev)
    a = jamba_ssm_dt_proj(inp.hi, inp.W_dt, dt_low_lo=inp.lo)
    b = jamba_ssm_dt_proj(inp.hi, inp.W_dt, dt_low_lo=inp.lo)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_dt_proj_persistent_walks_token_blocks():
    """Several items per CTA, ranges that start inside a token block and cross
    into the next (the planes are reloaded after the block's MMAs), both TMEM
    accumulators in turn, and a ragged last token block: every output."""
    dev = _dev()
    inp = synth.dt_proj_inputs(2000, 4096, 256, seed=34, device=dev)
    out = jamba_ssm_dt_proj(inp.hi, inp.W_dt, dt_low_lo=inp.lo)
    torch.cuda.synchronize()
    assert jamba_ssm_proj_get_status() == 0
    assert_out(out, _ref(inp), torch.bfloat16, "dt_proj 2000 x 4096 x 256")
