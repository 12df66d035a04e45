"""The N > 1 host path of the benchmark, on CPU with gloo (world size 2).

With several GPUs every rank either runs an independent replica of the step
(the default) or holds a row slice of one problem (--split rows: rows of W
per rank, X replicated; the MLP pair all-gathers its hidden activation before
the down product).  The job's time is the slowest rank's time, and the
whole-job rate counts the units all ranks processed.  These tests run the same
host functions over a real two-rank gloo process group on 127.0.0.1 -- the row
split with the CPU oracle doing each rank's products, checked against the
single-rank result -- and check that a nonzero rank of the reference arm
leaves without work or output."""
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


@pytest.mark.parametrize("R,world", [(4096, 2), (14336, 8), (4096, 3), (100, 4), (257, 2), (1, 2)])
def test_shard_rows_cover_every_row_once(R, world):
    seen = []
    pers = set()
    for rank in range(world):
        lo, hi, per = bench.shard_rows(R, world, rank)
        assert 0 <= lo <= hi <= R and hi - lo <= per and per % 256 == 0
        if rank < world - 1 and hi < R:
            assert hi - lo == per                   # only trailing slices are short
        seen += list(range(lo, hi))
        pers.add(per)
    assert seen == list(range(R)) and len(pers) == 1


def _split_rank_main(rank, world, port, q):
    """One rank of the row-split MLP pair, its products done by the CPU oracle:
    its rows of W_up -> its rows of H (rounded to bf16, as the GPU path stores
    H) -> all-gather of H -> its rows of W_down times the whole H."""
    import datetime
    import numpy as np
    import torch.distributed as dist
    import nm_inputs
    import oracle
    dist.init_process_group("gloo", init_method="tcp://127.0.0.1:%d" % port, rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        wl = _small_mlp()
        part = bench.split_workload(wl, world, rank, dist)
        dist_, per, R_up = part["gather"]
        T = wl["T"]
        Hb = _up_rows_bf16(part["W"], wl["X"])                    # this rank's rows of H, bf16 bits
        # the bf16 bit patterns travel as int32 (gloo has no 16-bit integer type)
        H_local = torch.zeros((per, T), dtype=torch.int32)
        H_local[:Hb.shape[0]] = torch.from_numpy(Hb.astype(np.int32))
        H_all = torch.empty((world * per, T), dtype=torch.int32)
        bench.gather_rows(dist_, H_all, H_local)
        H = H_all[:R_up].numpy().astype(np.uint16)
        Y = _down_rows(part["W2"], H)
        q.put((rank, part["rows2"], Y))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def _small_mlp():
    import nm_inputs
    Wu = nm_inputs.normal((512, 256), 11, 0.02, torch.bfloat16)
    Wd = nm_inputs.normal((256, 512), 12, 0.02, torch.bfloat16)
    X = nm_inputs.normal((256, 40), 13, 1.0, torch.bfloat16)
    return {"W": Wu, "W2": Wd, "X": X, "R": 512, "K": 256, "T": 40, "desc": "small MLP pair"}


def _up_rows_bf16(W, X):
    import oracle
    Wb = nm_inputs_bits(W)
    mask = oracle.mask_rank(Wb, 2, 4, dtype=oracle.BF16)
    v, m = oracle.compress24(Wb, mask, dtype=oracle.BF16)
    H = oracle.spmm(v, m, nm_inputs_bits(X), oracle.BF16, threads=1)
    return oracle.encode_array(H, oracle.BF16)


def _down_rows(W2, Hbits):
    import oracle
    Wb = nm_inputs_bits(W2)
    mask = oracle.mask_rank(Wb, 2, 4, dtype=oracle.BF16)
    v, m = oracle.compress24(Wb, mask, dtype=oracle.BF16)
    return oracle.spmm(v, m, Hbits, oracle.BF16, threads=1)


def nm_inputs_bits(t):
    import nm_inputs
    return nm_inputs.bits_u16(t)


def test_row_split_mlp_pair_equals_the_single_rank_result():
    """World size 2 over gloo: the row slices of Y, computed from row slices of
    W_up and W_down and an all-gathered H, reassemble to exactly the single-rank
    oracle result (the oracle computes every row on its own, in fp64)."""
    import numpy as np
    import oracle
    oracle.build()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_split_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(2)]
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    wl = _small_mlp()
    Y_ref = _down_rows(wl["W2"], _up_rows_bf16(wl["W"], wl["X"]))
    Y = np.zeros_like(Y_ref)
    covered = 0
    for _, (lo, hi), Yr in res:
        Y[lo:hi] = Yr
        covered += hi - lo
    assert covered == Y_ref.shape[0]
    assert np.array_equal(Y, Y_ref)


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
