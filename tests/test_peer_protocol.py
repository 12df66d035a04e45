"""The exchange protocol of the row-split MLP pair (`bench.py --split rows
--gather fused`), simulated on CPU with one thread per rank.

bench.Step's own launch sequence runs against a stand-in for the binding that
gives each peer call its contract, in program order per rank (the order of one
CUDA stream):

* nm_spmm_peers stores the rank's rows of H, tagged with the rank and its step
  number, into every rank's H buffer (sleeping between destinations);
* nm_peer_signal stores the epoch into the rank's slot of every flag array;
* nm_peer_wait blocks until every slot of the rank's flags holds the epoch;
* the down product (nm_spmm reading H) checks, twice with a sleep between,
  that every rank's rows hold that rank's rows of the same step.

Ranks run at different speeds, so a fast rank starts later steps while a slow
one is still reading.  With H double-buffered by step parity no read ever sees
another step's rows; the same run with one buffer does (the planted mistake).
"""
import os
import random
import sys
import threading
import time

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402

_REGISTRY = {}                 # "device address" of an exported buffer -> the tensor
_REG_LOCK = threading.Lock()


class _Rank:
    """The binding's calls for one rank (one thread)."""

    def __init__(self, rank, slow):
        self.rank, self.slow = rank, slow
        self.ups = 0                     # up products issued = this rank's step number
        self.rng = random.Random(1000 + rank)
        self.violations = []
        self.H_bufs = None

    def _nap(self, scale=1.0):
        time.sleep(self.rng.random() * 0.002 * scale * (5.0 if self.slow else 1.0))

    # buffers
    def alloc_compressed(self, R, K, dtype, dev, sm100=True):
        return (torch.zeros((R, K // 2), dtype=dtype), torch.zeros((R, K // 4), dtype=torch.uint8),
                torch.zeros((128, 128), dtype=torch.uint8))

    def nm_spmm_workspace_bytes(self, dtype, R, K, T):
        return 0

    # the bandwidth calls: nothing to model
    def nm_mask(self, *a, **k):
        pass

    nm_compress = nm_mask_compress = nm_meta_to_sm100 = nm_decompress = nm_mask

    # the peer calls
    def nm_ipc_handle(self, t):
        key = t.data_ptr()
        with _REG_LOCK:
            _REGISTRY[key] = t
        return key.to_bytes(8, "little") + bytes(56), 0

    def nm_ipc_open(self, handle, offset):
        return int.from_bytes(handle[:8], "little") + offset

    @staticmethod
    def _t(x):
        return x if isinstance(x, torch.Tensor) else _REGISTRY[int(x)]

    def nm_spmm_peers(self, values, img, X, dests, row0, ldy):
        self.ups += 1
        R = values.shape[0]
        tag = float(1000 * self.ups + self.rank)
        order = list(range(len(dests)))
        self.rng.shuffle(order)
        for j in order:
            self._nap()
            self._t(dests[j])[row0:row0 + R].fill_(tag)

    def nm_peer_signal(self, flags, rank, epoch):
        assert rank == self.rank
        for f in flags:
            self._nap(0.2)
            self._t(f)[rank] = epoch

    def nm_peer_wait(self, flags, epoch, timeout_ns):
        t0 = time.time()
        while int(flags.min()) < epoch:
            if time.time() - t0 > 20.0:
                raise TimeoutError("rank %d: flags %s never reached %d" % (self.rank, flags.tolist(), epoch))
            time.sleep(0.0002)

    def nm_spmm(self, values, img, X, Y, workspace=None):
        if self.H_bufs is None or not any(X.data_ptr() >= b.data_ptr() and
                                          X.data_ptr() < b.data_ptr() + b.numel() * b.element_size()
                                          for b in self.H_bufs):
            return                              # not the down product
        per, world = self.per, self.world
        for check in range(2):
            for j in range(world):
                rows_j = min(per, max(0, self.R_full - j * per))
                want = float(1000 * self.ups + j)
                got = X[j * per:j * per + rows_j]
                if rows_j and not bool((got == want).all()):
                    self.violations.append((self.ups, j, check, sorted(set(got.flatten().tolist()))[:4]))
            self._nap(3.0)


class _Dist:
    """torch.distributed for thread ranks: all_gather_object and barrier."""

    def __init__(self, rank, world, shared):
        self.rank, self.world, self.shared = rank, world, shared

    def get_world_size(self):
        return self.world

    def get_rank(self):
        return self.rank

    def get_backend(self):
        return "gloo"

    def all_gather_object(self, out, obj):
        self.shared["objs"][self.rank] = obj
        self.shared["barrier"].wait()
        for i in range(self.world):
            out[i] = self.shared["objs"][i]
        self.shared["barrier"].wait()

    def barrier(self):
        self.shared["barrier"].wait()


def _bf16(*shape):
    return torch.zeros(shape, dtype=torch.bfloat16)


def _run(world, steps, single_buffer=False, slow_rank=1):
    bench.IPC_MAPPINGS.clear()                # whatever earlier tests in this process mapped
    R, K, T = 256 * world, 64, 8
    wl = {"W": _bf16(R, K), "W2": _bf16(K, R), "X": _bf16(K, T), "R": R, "K": K, "T": T}
    shared = {"objs": [None] * world, "barrier": threading.Barrier(world, timeout=60)}
    ranks = [_Rank(r, r == slow_rank) for r in range(world)]
    errors = []

    def body(r):
        try:
            d = _Dist(r, world, shared)
            part = bench.split_workload(wl, world, r, d, gather="fused")
            step = bench.Step(ranks[r], part, torch.device("cpu"))
            assert step.fused
            if single_buffer:                     # the planted mistake: H reused every step
                step.H_bufs[1] = step.H_bufs[0]
                step.peer_H[1] = step.peer_H[0]
            ranks[r].H_bufs = step.H_bufs
            ranks[r].per, ranks[r].world, ranks[r].R_full = step.gather[1], world, step.gather[2]
            d.barrier()
            for _ in range(steps):
                step.run()
        except Exception as exc:  # reported to the main thread
            errors.append((r, repr(exc)))
            shared["barrier"].abort()

    threads = [threading.Thread(target=body, args=(r,)) for r in range(world)]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=120)
        assert not t.is_alive()
    assert len(bench.IPC_MAPPINGS) == 3 * world * (world - 1)   # two H buffers and the flags of every other rank
    bench.IPC_MAPPINGS.clear()
    return ranks, errors


@pytest.mark.parametrize("world", [2, 3, 4])
def test_double_buffered_exchange_never_reads_another_step(world):
    ranks, errors = _run(world, steps=12)
    assert errors == []
    for rk in ranks:
        assert rk.ups == 12
        assert rk.violations == [], rk.violations[:3]


def test_one_buffer_is_caught():
    """The check itself: with one H buffer a fast rank overwrites rows that a
    slow rank is still reading."""
    ranks, errors = _run(2, steps=12, single_buffer=True, slow_rank=1)
    assert errors == []
    assert any(rk.violations for rk in ranks)
