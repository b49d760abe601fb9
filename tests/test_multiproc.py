"""The multi-process path of the benchmark on the CPU (gloo, world size 2):
the path shards into independent (sequence, KV head) units, so N GPUs run N
replicas with no data-path collective; what crosses ranks is the barrier and
the max-over-ranks step time, and only rank 0 prints."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    import bench
    r, w, _ = bench.setup_dist(world)
    try:
        assert (r, w) == (rank, world)
        assert torch.distributed.get_backend() == "gloo"
        bench.barrier(w)
        t = bench.max_over_ranks(1.0 + 2.5 * rank, w)  # each rank's step time
        out[rank] = t
        bench.barrier(w)
    finally:
        torch.distributed.destroy_process_group()


@pytest.mark.skipif(torch.cuda.is_available(), reason="the gloo path is the host-only one")
def test_max_over_ranks_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        mp.start_processes(_rank_main, args=(2, free_port(), out), nprocs=2, join=True, start_method="spawn")
        assert dict(out) == {0: 3.5, 1: 3.5}  # every rank times the slowest rank


@pytest.mark.skipif(torch.cuda.is_available(), reason="the gloo path is the host-only one")
def test_reference_arm_under_torchrun_prints_once():
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(free_port()), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--workload", "tiny_fp32_t2048", "--steps", "3", "--warmup", "2"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout  # rank 0 alone prints
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["config"]["workload"] == "tiny_fp32_t2048" and d["higher_is_better"] is True
    assert (d["steps"], d["warmup"]) == (3, 2)  # the driver's --steps / --warmup, not clamped
    assert abs(d["value"] * d["ms_per_step"] - 1000.0) < 1e-6 * 1000.0  # whole steps, measured
