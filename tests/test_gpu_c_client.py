"""The boundary is a C ABI: plain C programs (tests/c/abi_client.c and
tests/c/ssd_client.c, gcc + the CUDA runtime, no Python or torch in the
process) call jamba_ssm_scan and jamba_ssm_state_update on fp32 data, and
jamba_ssm_ssd_scan on bf16 data, and their results match the oracle."""
import os
import subprocess

import numpy as np
import pytest
import torch

import oracle
from selective_state_space_26_b200 import _lib, build, synth
from tests.parity import assert_out, assert_state

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")


def test_plain_c_client_matches_oracle(tmp_path):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    exe = tmp_path / "abi_client"
    libdir = os.path.dirname(_lib.LIB_PATH)
    subprocess.run(["gcc", "-O1", "-o", str(exe), os.path.join(ROOT, "tests", "c", "abi_client.c"),
                    "-I", os.path.join(ROOT, "include"), "-I", os.path.join(CUDA, "include"),
                    "-L", libdir, "-ljamba_ssm", "-L", os.path.join(CUDA, "lib64"), "-lcudart",
                    f"-Wl,-rpath,{libdir}", f"-Wl,-rpath,{os.path.join(CUDA, 'lib64')}"],
                   check=True)
    b, l, d, n = 2, 150, 68, 16
    inp = synth.scan_inputs(b, l, d, n, torch.float32, seed=19, A_kind="random")
    tok = synth.decode_step(b, d, n, 0, 19, torch.float32)
    f = tmp_path / "in.bin"
    with open(f, "wb") as fh:
        fh.write(np.array([b, l, d, n], dtype=np.int64).tobytes())
        for t in (inp.x, inp.delta, inp.z, inp.B, inp.C, inp.A, inp.D, inp.delta_bias,
                  tok.x, tok.delta, tok.z, tok.B, tok.C):
            fh.write(t.numpy().astype(np.float32).tobytes())
    o = tmp_path / "out.bin"
    r = subprocess.run([str(exe), str(f), str(o)], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, (r.returncode, r.stderr)
    raw = np.fromfile(o, dtype=np.float32)
    sizes = [b * l * d, b * d * n, b * d, b * d * n]
    parts = np.split(raw, np.cumsum(sizes)[:-1])
    out, hf = parts[0].reshape(b, l, d), parts[1].reshape(b, d, n)
    out1, st1 = parts[2].reshape(b, d), parts[3].reshape(b, d, n)
    ref, ref_h = oracle.scan(inp.x, inp.delta, inp.z, inp.B, inp.C, inp.A, D=inp.D,
                             delta_bias=inp.delta_bias)
    assert_out(out, ref, torch.float32, "C client scan")
    assert_state(hf, ref_h, torch.float32, "C client scan")
    ref1, ref_st1 = oracle.state_update(ref_h, tok.x, tok.delta, tok.z, tok.B, tok.C, inp.A,
                                        D=inp.D, delta_bias=inp.delta_bias)
    assert_out(out1, ref1, torch.float32, "C client decode")
    assert_state(st1, ref_st1, torch.float32, "C client decode")


def test_plain_c_client_ssd_matches_oracle(tmp_path):
    """jamba_ssm_ssd_scan from a plain C program on bf16 data with d_state 16
    and heads of 64 (the chunked tensor-core kernel), two sequences over three
    chunks with a ragged last one and a nonzero initial state."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    exe = tmp_path / "ssd_client"
    libdir = os.path.dirname(_lib.LIB_PATH)
    subprocess.run(["gcc", "-O1", "-o", str(exe), os.path.join(ROOT, "tests", "c", "ssd_client.c"),
                    "-I", os.path.join(ROOT, "include"), "-I", os.path.join(CUDA, "include"),
                    "-L", libdir, "-ljamba_ssm", "-L", os.path.join(CUDA, "lib64"), "-lcudart",
                    f"-Wl,-rpath,{libdir}", f"-Wl,-rpath,{os.path.join(CUDA, 'lib64')}"],
                   check=True)
    b, l, h, p, n = 2, 300, 8, 64, 16
    inp = synth.ssd_inputs(b, l, h, p, n, torch.bfloat16, seed=23, h0_std=0.3)
    bits = lambda t: t.contiguous().view(torch.int16).numpy().tobytes()  # noqa: E731
    f = tmp_path / "in.bin"
    with open(f, "wb") as fh:
        fh.write(np.array([b, l, h, p, n], dtype=np.int64).tobytes())
        for t in (inp.x, inp.z, inp.delta, inp.B, inp.C):
            fh.write(bits(t))
        for t in (inp.A, inp.D, inp.delta_bias, inp.h0):
            fh.write(t.numpy().astype(np.float32).tobytes())
    o = tmp_path / "out.bin"
    r = subprocess.run([str(exe), str(f), str(o)], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, (r.returncode, r.stderr)
    raw = o.read_bytes()
    nout = b * l * h * p
    out = torch.frombuffer(bytearray(raw[:2 * nout]), dtype=torch.int16).view(torch.bfloat16)
    hf = np.frombuffer(raw[2 * nout:], dtype=np.float32).reshape(b, h * p, n)
    ref, ref_h = oracle.ssd_scan(inp.x, inp.delta, inp.z, inp.B, inp.C, inp.A, h, D=inp.D,
                                 delta_bias=inp.delta_bias, h0=inp.h0)
    assert_out(out.reshape(b, l, h * p), ref, torch.bfloat16, "C client ssd")
    assert_state(hf, ref_h, torch.bfloat16, "C client ssd")
