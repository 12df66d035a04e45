"""The N > 1 host path of the benchmark, on CPU with gloo (world size 2).

With several GPUs every rank runs an independent replica of the step (the
path shards with no exchange), the job's time is the slowest rank's time,
and the whole-job rate counts the units all ranks processed.  These tests
run the same host functions over a real two-rank gloo process group on
127.0.0.1, and check that a nonzero rank of the reference arm leaves without
work or output."""
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, times, q):
    import datetime
    import torch.distributed as dist
    dist.init_process_group("gloo", init_method="tcp://127.0.0.1:%d" % port, rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        dist.barrier()
        got = bench.max_over_ranks(dist, times[rank], torch.device("cpu"))
        q.put((rank, got))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_two_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    times = [[12.5, 30.0], [11.0, 31.5]]          # (step ms, e2e ms) per rank
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, times, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = dict(q.get(timeout=10) for _ in range(2))
    assert res[0] == res[1] == [12.5, 31.5]


def test_max_over_ranks_without_a_group_is_the_identity():
    assert bench.max_over_ranks(None, [1.0, 2.5], torch.device("cpu")) == [1.0, 2.5]


def test_whole_job_rate_counts_every_rank():
    one = bench.whole_job_rate(1, 1.374e11, 1000, 123.3, 1e12)
    two = bench.whole_job_rate(2, 1.374e11, 1000, 123.3, 1e12)
    assert two == pytest.approx(2 * one)
    assert one == pytest.approx(1.374e11 * 1000 / 0.1233 / 1e12)


def test_reference_arm_nonzero_rank_exits_without_output():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1", MASTER_ADDR="127.0.0.1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0
    assert r.stdout.strip() == ""
