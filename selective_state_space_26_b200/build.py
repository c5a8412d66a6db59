"""Build the CUDA libraries in-tree for sm_100a with nvcc: libjamba_ssm.so
(the scan and the decode update) and libjamba_ssm_proj.so (the projection that
feeds the scan)."""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
SRC = os.path.join(PKG, "csrc", "jamba_ssm.cu")
LIB = os.path.join(PKG, "libjamba_ssm.so")
PROJ_SRC = os.path.join(PKG, "csrc", "jamba_ssm_proj.cu")
PROJ_LIB = os.path.join(PKG, "libjamba_ssm_proj.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


def sources():
    d = os.path.join(PKG, "csrc")
    return [os.path.join(d, f) for f in sorted(os.listdir(d)) if f.endswith((".cu", ".cuh"))]


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    inc = os.path.join(ROOT, "include")
    deps = sources() + [os.path.join(inc, h) for h in os.listdir(inc) if h.endswith(".h")]
    return all(os.path.getmtime(s) <= t for s in deps)


def _nvcc(src: str, out: str, verbose: bool) -> None:
    # Hidden visibility: each library keeps its own kernels and device status
    # word; only the extern "C" entry points marked for export are visible.
    cmd = [NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo",
           "-std=c++17", "-Xcompiler", "-fPIC", "-shared", "-cudart", "static",
           "-I", os.path.join(ROOT, "include"), "-o", out, src]
    if out == PROJ_LIB:
        cmd[cmd.index("-fPIC")] = "-fPIC,-fvisibility=hidden"
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.run(cmd, check=True)


def build(verbose: bool = False, force: bool = False) -> str:
    for src, out in ((SRC, LIB), (PROJ_SRC, PROJ_LIB)):
        if force or not up_to_date(out):
            _nvcc(src, out, verbose)
    return LIB


if __name__ == "__main__":
    build(verbose="-v" in sys.argv, force=True)
    print(LIB)
    print(PROJ_LIB)
