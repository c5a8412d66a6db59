"""Throughput of the special-function unit on the B200 (needs a GPU): the
per-SM rate behind the scan's MUFU roofline (16 exp2 or reciprocal operations
per SM per clock).  Builds tests/c/mufu_rate.cu with nvcc and runs it."""
import os
import subprocess

import pytest
import torch

pytestmark = pytest.mark.gpu
HERE = os.path.dirname(os.path.abspath(__file__))


def test_mufu_ops_per_clock_per_sm(tmp_path):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    exe = tmp_path / "mufu_rate"
    subprocess.run(["/usr/local/cuda/bin/nvcc", "-gencode", "arch=compute_100a,code=sm_100a",
                    "-O3", "-o", str(exe), os.path.join(HERE, "c", "mufu_rate.cu")], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120, check=True)
    f = out.stdout.split()
    vals = dict(zip(f[0::2], f[1::2]))
    print("mufu_rate:", out.stdout.strip())
    ex2, rcp = float(vals["ex2"]), float(vals["rcp"])
    # the roofline's 16 per SM per clock, within the timing's resolution
    assert 15.0 <= ex2 <= 16.5, out.stdout
    assert 15.0 <= rcp <= 16.5, out.stdout
