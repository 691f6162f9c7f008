"""The multi-rank host logic of bench.py on CPU (gloo, world size 2).

The decode path does not shard: every rank is an independent replica, and
the only exchange is the timing, the slowest rank's time over all ranks.
These tests run that exchange on two gloo ranks, and the reference arm under
torchrun with two ranks (rank 0 alone runs and prints)."""
import json
import os
import socket
import subprocess
import sys
import tempfile

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_worker(rank, world, port, outdir):
    import datetime

    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        ms = 10.0 + 5.0 * rank          # rank 1 is the slower one
        m = bench.max_over_ranks(ms, world, dist, "cpu")
        v = bench.aggregate_value(world, 100, m)
        with open(os.path.join(outdir, f"rank{rank}.json"), "w") as f:
            json.dump({"max_ms": m, "value": v}, f)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_whole_job_value_on_two_gloo_ranks():
    with tempfile.TemporaryDirectory() as d:
        mp.start_processes(_rank_worker, args=(2, _free_port(), d), nprocs=2,
                           start_method="spawn", join=True)
        got = [json.load(open(os.path.join(d, f"rank{r}.json"))) for r in range(2)]
    for g in got:
        assert g["max_ms"] == 15.0                      # every rank gets the slowest time
        assert g["value"] == pytest.approx(2 * 100 / 0.015)  # units of both ranks / that time


def test_one_rank_needs_no_collective():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(12.5, 1) == 12.5
    assert bench.aggregate_value(1, 50, 12.5) == pytest.approx(4000.0)


def test_reference_arm_under_torchrun_prints_one_line_from_rank_0():
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
           "--steps", "1", "--warmup", "1"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
