"""Host-side logic of the multi-GPU bench path, run as gloo ranks on the CPU:
the max-over-ranks timing, the whole-job throughput of independent replicas,
the per-rank sequence offsets (each replica scans its own seeded sequences),
and the reference arm under torchrun (rank 0 alone prints one line)."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from selective_state_space_26_b200 import synth  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r reports (r + 1, 10 - r): the max must come back on every rank
        got = bench.max_over_ranks([rank + 1.0, 10.0 - rank], world, torch.device("cpu"))
        w = synth.WORKLOADS["s6_tiny_fp32_b1_l64_d16_n4"]
        off = bench.replica_seq_offset(rank, w.batch)
        inp = synth.workload_inputs(w, device="cpu", seq_offset=off)
        q.put((rank, got, off, inp.x.clone(), inp.B.clone()))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_gloo_two_ranks_max_and_replica_shards():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q))
             for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(world):
        rank, got, off, x, B = q.get(timeout=120)
        res[rank] = (got, off, x, B)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in range(world):
        assert res[r][0] == [float(world), 10.0]
    assert res[0][1] == 0 and res[1][1] == 1
    # the two replicas scan different sequences ...
    assert not torch.equal(res[0][2], res[1][2])
    # ... which are exactly sequences 0 and 1 of one batch-2 draw of the stream
    w = synth.WORKLOADS["s6_tiny_fp32_b1_l64_d16_n4"]
    both = synth.scan_inputs(2, w.seqlen, w.d_inner, w.d_state, w.dtype, w.seed, "cpu")
    for r in range(world):
        assert torch.equal(res[r][2][0], both.x[r])
        assert torch.equal(res[r][3][0], both.B[r])


def test_job_throughput_is_weak_scaling_sum():
    assert bench.job_tokens_per_s(4097, 1, 0.5) == pytest.approx(8194.0)
    assert bench.job_tokens_per_s(4097, 8, 0.5) == pytest.approx(8 * 8194.0)
    assert bench.max_over_ranks([1.5, 2.5], 1, torch.device("cpu")) == [1.5, 2.5]


def test_reference_arm_under_torchrun_prints_one_line():
    env = dict(os.environ)
    env.pop("CUDA_VISIBLE_DEVICES", None)
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), "bench.py",
           "--impl", "reference", "--gpus", "2", "--steps", "2", "--warmup", "3",
           "--workload", "s6_tiny_fp32_b1_l64_d16_n4", "--ref-seconds", "2"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=300, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["steps"] == 2
    assert d["cpu_baseline"]["kind"] == "oracle"
    assert d["e2e"]["h2d_bytes_per_step"] == 0


def test_traffic_record_follows_the_kernel_device_sources(tmp_path, monkeypatch):
    """roofline.traffic is reported only while the recorded DRAM counters were
    taken on the current device code of the timed kernel (its header and every
    header that includes, directly or not) and, for the scan, on the same
    launch shape: a header in that closure changes the hash, a file outside
    it does not, and another launch shape drops the record."""
    csrc = tmp_path / "selective_state_space_26_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "k.cuh").write_text('#include "a.cuh"\n#include <cuda.h>\n')
    (csrc / "a.cuh").write_text('#include "b.cuh"\nint a;\n')
    (csrc / "b.cuh").write_text("int b;\n")
    (csrc / "host.cu").write_text('#include "k.cuh"\nint host;\n')
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setitem(bench.KERNEL_HEADER, "k", "k.cuh")
    h0 = bench.kernel_source_hash("k")
    (csrc / "host.cu").write_text('#include "k.cuh"\nint host2;\n')
    (csrc / "unrelated.cuh").write_text("int u;\n")
    assert bench.kernel_source_hash("k") == h0
    (csrc / "b.cuh").write_text("int b2;\n")  # included indirectly
    h1 = bench.kernel_source_hash("k")
    assert h1 != h0
    prof = tmp_path / "profiles"
    prof.mkdir()
    launch = bench.plan_launch({"variant": 2, "grid": 147, "channels_per_cta": 56})
    (prof / "dram_traffic.json").write_text(json.dumps(
        {"k": {"w": {"bytes_per_launch": 123, "source_hash": h1, "launch": launch}}}))
    assert bench.recorded_traffic("k", "w") == 123.0
    assert bench.recorded_traffic("k", "w", launch) == 123.0
    other = bench.plan_launch({"variant": 1, "grid": 64, "channels_per_cta": 128})
    assert bench.recorded_traffic("k", "w", other) is None
    (csrc / "a.cuh").write_text('#include "b.cuh"\nint a2;\n')
    assert bench.recorded_traffic("k", "w") is None

