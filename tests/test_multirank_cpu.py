"""N > 1 host path of bench.py on CPU: gloo ranks, world size 2.

The decode path shards over (slot, head) units with no exchange step, so a
multi-GPU run is N replicas.  What the ranks share is the timing protocol:
barrier, per-rank seed, max-over-ranks time and the whole-job aggregate.
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


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        my_ms = 10.0 + 5.0 * rank                       # rank 1 is the slow one
        worst = bench.reduce_max(my_ms, world, torch.device("cpu"))
        dist.barrier()
        out[rank] = (worst, bench.rank_seed(0, rank),
                     bench.job_tokens_per_s(256, 256, 4, world, worst))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_aggregate_gloo():
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    assert out[0][0] == out[1][0] == 15.0                  # every rank sees the slowest time
    assert out[0][1] != out[1][1]                          # replicas draw different inputs
    expect = 256 * 256 * 4 * world / 0.015                 # all ranks' tokens / slowest time
    assert abs(out[0][2] - expect) < 1e-6 * expect and out[0][2] == out[1][2]


def test_reduce_max_single_rank_is_identity():
    import bench
    assert bench.reduce_max(3.5, 1, torch.device("cpu")) == 3.5


def test_reference_arm_under_torchrun_prints_once():
    """The CPU reference arm launched like the driver does for N = 2: rank 0
    prints exactly one JSON line, rank 1 exits 0 without work."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2", "--steps", "1",
           "--warmup", "0", "--B", "2", "--H", "2", "--dk", "64"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"


@pytest.mark.parametrize("world", [1, 2, 4])
def test_job_aggregate_scales_with_replicas(world):
    import bench
    one = bench.job_tokens_per_s(128, 256, 10, 1, 20.0)
    assert bench.job_tokens_per_s(128, 256, 10, world, 20.0) == pytest.approx(world * one)


def test_cpu_baseline_uses_every_core_and_reports_one_core():
    """cpu_baseline runs the oracle on spawned worker processes (one per core)
    and on one core alone, over the same per-worker sample."""
    import argparse

    import bench
    a = argparse.Namespace(op="gdn", B=4, H=4, d=64, M=4, tokens=8, seed=0)
    cb = bench.cpu_baseline(a)
    cores = min(bench.host_cores(), bench.ORACLE_MAX_WORKERS)
    assert cb["kind"] == "oracle" and cb["cores"] == cores and cb["value"] > 0
    assert cb["cpu_model"] and cb["single_core"]["value"] > 0
    assert f"{cores} worker process(es)" in cb["sample"]
    assert cb["sample"].split(",", 1)[1] == cb["single_core"]["sample"].split(",", 1)[1]
