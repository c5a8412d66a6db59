"""Comparison rules between the CUDA path and the fp64 oracle.

Tolerances (stated for the S6 layer: rel-L2 <= 1e-3 and max-abs <= 2e-2 on
bf16 outputs, <= 1e-5 relative in fp32 mode), read so that a perfect kernel
passes: correctly rounding the exact result to bf16 already moves it by up to
half a bf16 ulp (|out| reaches ~17 at Jamba's sizes, where half an ulp is
0.03), so

  bf16 outputs:  rel-L2(gpu, bf16_RNE(oracle))                       <= 1e-3
                 max_i max(0, |gpu_i - oracle_i| - ulp_bf16(oracle_i)/2)  <= 2e-2
  fp32 outputs:  rel-L2(gpu, oracle)                                 <= 1e-5
                 max |gpu - oracle| <= 1e-5 * max(1, max |oracle|)
  fp32 final state: rel-L2 <= 1e-5 (fp32 I/O) or 1e-4 (bf16 I/O; same inputs,
                 only fp32 rounding inside the recurrence differs).
"""
from __future__ import annotations

import numpy as np
import torch

BF16_REL_L2 = 1e-3
BF16_MAX_EXCESS = 2e-2
F32_REL = 1e-5
STATE_REL_L2 = {torch.bfloat16: 1e-4, torch.float32: 1e-5}


def to_np(t) -> np.ndarray:
    if isinstance(t, torch.Tensor):
        return t.detach().to("cpu", torch.float64).numpy()
    return np.asarray(t, dtype=np.float64)


def round_bf16(a: np.ndarray) -> np.ndarray:
    """Round float64 values to the nearest bfloat16 (ties to even), in one
    step: bf16 keeps 8 significant bits, and np.rint rounds half to even."""
    a = np.asarray(a, dtype=np.float64)
    m, e = np.frexp(a)  # a = m * 2**e, 0.5 <= |m| < 1
    return np.ldexp(np.rint(m * 256.0) / 256.0, e)


def ulp_bf16(a: np.ndarray) -> np.ndarray:
    """Spacing of bfloat16 numbers at |a| (normal range)."""
    _, e = np.frexp(np.asarray(a, dtype=np.float64))
    return np.ldexp(1.0, e - 8)


def rel_l2(a, b) -> float:
    a, b = to_np(a), to_np(b)
    den = float(np.linalg.norm(b))
    num = float(np.linalg.norm(a - b))
    return num / den if den > 0 else num


def compare_out(gpu, ref, dtype) -> dict:
    """Metrics of gpu output vs the unrounded fp64 oracle `ref`."""
    g, r = to_np(gpu), to_np(ref)
    m = {"raw_rel_l2": rel_l2(g, r), "raw_max_abs": float(np.max(np.abs(g - r))) if r.size else 0.0}
    if dtype == torch.bfloat16:
        rb = round_bf16(r)
        m["rel_l2"] = rel_l2(g, rb)
        excess = np.abs(g - r) - 0.5 * ulp_bf16(r)
        m["max_excess"] = float(np.max(np.maximum(excess, 0.0))) if r.size else 0.0
        m["ok"] = m["rel_l2"] <= BF16_REL_L2 and m["max_excess"] <= BF16_MAX_EXCESS
    else:
        m["rel_l2"] = m["raw_rel_l2"]
        lim = F32_REL * max(1.0, float(np.max(np.abs(r))) if r.size else 1.0)
        m["max_excess"] = max(0.0, m["raw_max_abs"] - lim)
        m["ok"] = m["rel_l2"] <= F32_REL and m["raw_max_abs"] <= lim
    return m


def compare_state(gpu, ref, dtype) -> dict:
    e = rel_l2(gpu, ref)
    return {"state_rel_l2": e, "ok": e <= STATE_REL_L2[dtype]}


def assert_out(gpu, ref, dtype, what=""):
    m = compare_out(gpu, ref, dtype)
    assert m["ok"], f"{what} output parity failed: {m}"
    return m


def assert_state(gpu, ref, dtype, what=""):
    m = compare_state(gpu, ref, dtype)
    assert m["ok"], f"{what} state parity failed: {m}"
    return m
