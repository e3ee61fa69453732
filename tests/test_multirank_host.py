"""Host-side logic of the multi-rank benchmark on CPU with gloo, world size 2:
the timing collectives (barrier, max over ranks), the weak-scaling aggregate,
and the reference arm's rank-0-only rule. The GPU data path has no collective:
ranks run independent replicas of the workload."""
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


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    import datetime

    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                           timeout=datetime.timedelta(seconds=60))
    try:
        barrier, max_over_ranks = bench.make_collectives(world, torch.device("cpu"))
        barrier()
        # each rank's "device time" differs; every rank must see the slowest one
        local_ms = 3.0 + 2.5 * rank
        ms = max_over_ranks(local_ms)
        rate = bench.whole_job_rate(world, 1000.0, ms)
        barrier()
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"ms": ms, "rate": rate}, f)
    finally:
        dist.destroy_process_group()


def test_timing_collectives_two_ranks(tmp_path):
    world, port = 2, _free_port()
    mp.start_processes(_rank_main, args=(world, port, str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    slowest = 3.0 + 2.5 * (world - 1)
    for r in res:
        assert r["ms"] == pytest.approx(slowest)
        # the whole job: both replicas' units in the slowest rank's time
        assert r["rate"] == pytest.approx(world * 1000.0 / (slowest * 1e-3))


def test_single_rank_collectives_are_local():
    import bench

    barrier, max_over_ranks = bench.make_collectives(1, torch.device("cpu"))
    barrier()
    assert max_over_ranks(4.25) == 4.25
    assert bench.whole_job_rate(1, 10.0, 5.0) == pytest.approx(2000.0)


def test_reference_arm_runs_on_rank_zero_only():
    # a non-zero rank of a torchrun launch exits 0 at once and prints nothing
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "3"],
                       env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""
