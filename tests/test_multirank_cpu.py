"""Replica bookkeeping of bench.py over two gloo ranks on the CPU.

The layer has no cross-GPU step: with N > 1 every rank runs its own replica and the only
collectives are the timing reductions.  These tests run those reductions, the whole-job
throughput arithmetic and the reference arm's rank handling as two CPU processes."""
import json
import os
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402



def _worker(rank, world, init_file, q):
    import datetime
    # rendezvous through a file in the test's own temporary directory (no port to race for)
    dist.init_process_group("gloo", init_method="file://" + init_file, rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        # rank r "measured" (r + 1) * 10 ms: the job time is the slowest rank's
        ms = bench.max_over_ranks(10.0 * (rank + 1), world, torch.device("cpu"))
        e2e = bench.max_over_ranks(3.0 if rank == 0 else 7.5, world, torch.device("cpu"))
        val = bench.whole_job_tokens_per_s(world, 256, 4, ms)
        q.put((rank, ms, e2e, val))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world2(tmp_path):
    world, init_file = 2, str(tmp_path / "rendezvous")
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, init_file, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ms, e2e, val in out:
        assert ms == 20.0 and e2e == 7.5
        # 2 replicas x 256 tokens x 4 steps in 20 ms
        assert val == pytest.approx(2 * 256 * 4 / 0.020)


def test_max_over_ranks_single_rank_is_identity():
    assert bench.max_over_ranks(1.25, 1, None) == 1.25


def _reference_arm(rank: int):
    env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank))
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
                           "tiny", "--gpus", "2", "--steps", "3", "--warmup", "3"],
                          env=env, capture_output=True, text=True, timeout=300)


def test_reference_arm_rank1_exits_without_work():
    r = _reference_arm(1)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


def test_reference_arm_rank0_prints_one_line():
    r = _reference_arm(0)
    assert r.returncode == 0, r.stderr
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["steps"] == 3
    assert line["cpu_baseline"]["kind"] == "oracle" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["value"] == line["value"]
