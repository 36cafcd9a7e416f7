"""Host logic of bench.py's multi-GPU (replica) path, on CPU with two gloo
ranks: every rank gets the slowest rank's time, the whole-job throughput
counts all ranks' bytes, and the reference arm runs on rank 0 only."""
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


def _rank_main(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = 10.0 + 5.0 * rank                      # rank 1 is the slow one
        got = bench.max_over_ranks(ms, world, "cpu")
        dist.barrier()
        got2 = bench.max_over_ranks(3.0 - rank, world, "cpu")
        out[rank] = (got, got2)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    world, port = 2, 29511
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert res[0] == res[1] == (15.0, 3.0)


def test_max_over_ranks_single_rank_is_identity():
    assert bench.max_over_ranks(7.5, 1) == 7.5


def test_whole_job_gbs_counts_all_ranks():
    one = bench.whole_job_gbs(1, bench.LAYERS * bench.WEIGHT_BYTES, 10, 5.0)
    two = bench.whole_job_gbs(2, bench.LAYERS * bench.WEIGHT_BYTES, 10, 5.0)
    assert two == pytest.approx(2 * one)
    assert one == pytest.approx(bench.LAYERS * bench.WEIGHT_BYTES * 10 / 5.0e6)


def test_reference_arm_runs_on_rank_zero_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "3"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0
    assert r.stdout.strip() == ""


def test_reference_arm_line_on_rank_zero():
    """Rank 0 of the reference arm prints one JSON line with the contract's keys:
    the oracle timed on the host, its e2e equal to its value with no copies."""
    import json
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "2",
                        "--warmup", "3"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
              "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference" and d["steps"] == 2 and d["warmup"] >= 3
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["value"] == d["value"] and d["e2e"]["h2d_bytes_per_step"] == 0
    assert d["e2e"]["d2h_bytes_per_step"] == 0 and d["value"] > 0
