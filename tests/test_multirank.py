"""The multi-rank host path of bench.py on CPU (gloo, world size 2).

The hot path does not shard (independent replicas, one per GPU), so the only
multi-rank logic is the benchmark's: every rank draws its own batch, the job's
time is the slowest rank's, ranks meet at barriers around the timed region,
and under the reference arm only rank 0 runs and prints."""
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


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    import bench
    from workloads import WORKLOADS, make_inputs
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        dist.barrier()
        t = bench.max_over_ranks(1.5 + 2.0 * rank, world, torch.device("cpu"))
        w = WORKLOADS[1]
        q = make_inputs(w, device="cpu", seed=bench.replica_seed(w, rank))["q"]
        gathered = [torch.zeros_like(q) for _ in range(world)]
        dist.all_gather(gathered, q)
        dist.barrier()
        same = bool(torch.equal(gathered[0], gathered[1]))
        out.put((rank, t, same))
    finally:
        dist.destroy_process_group()


def test_two_ranks_max_time_and_own_batches():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.SimpleQueue()
    mp.start_processes(_worker, args=(world, _free_port(), q), nprocs=world, join=True,
                       start_method="spawn")
    res = sorted(q.get() for _ in range(world))
    # both ranks report the slowest rank's time
    assert [r[1] for r in res] == [3.5, 3.5]
    # the replicas' inputs differ (weak scaling: every rank its own batch)
    assert not res[0][2]


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(2.25, 1, torch.device("cpu")) == 2.25


def test_reference_arm_runs_on_rank_zero_only():
    # under torchrun the other ranks exit 0 without work or output
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--config", "1", "--steps", "1", "--warmup", "3"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""
