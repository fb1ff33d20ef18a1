"""Multi-process paths of the benchmark, on the CPU.

With N GPUs the benchmark runs N independent replicas (the (batch, head)
units need no exchange), so its only cross-rank logic is the timing: every
rank times its own replica and the job reports the slowest.  These tests run
that logic on world-size-2 gloo process groups, and check that the reference
arm launched under torchrun prints one line from rank 0 while the other rank
exits without work.
"""
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


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, values, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        out[rank] = bench.max_over_ranks(values[rank], dist, torch.device("cpu"))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("values", [[1.5, 0.25], [0.25, 1.5], [2.0, 2.0]])
def test_max_over_ranks_two_gloo_ranks(values):
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        port = _free_port()
        procs = [ctx.Process(target=_rank_main, args=(r, 2, port, values, out)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
        assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
        assert out[0] == out[1] == max(values)


def test_max_over_ranks_without_a_group_is_identity():
    import bench
    assert bench.max_over_ranks(3.25) == 3.25


def test_reference_arm_under_torchrun_prints_once():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3", "--config", "c0"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "tokens/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["e2e"]["h2d_bytes_per_step"] == 0


@pytest.mark.parametrize("op", ["step", "conv", "bwd", "conv_bwd"])
def test_reference_arm_of_the_other_ops(op):
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--op", op, "--steps", "1",
           "--warmup", "3", "--step-batch", "8"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["cpu_baseline"]["kind"] == "oracle"
