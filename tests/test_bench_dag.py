"""The benchmark step's dependency graph against the data flow of its launches.

bench.Step.capture() records the step as a CUDA graph in which a launch waits
only for the launches listed in Step.deps(); independent chains run on forked
streams.  A missing edge there would let two kernels race on a buffer.  This
test runs Step.calls() on CPU against a recording stand-in for the binding that
knows, for each entry point, which arguments it reads and which it writes (the
argument roles of include/nm.h), and checks for every workload kind that

  * every dependency names an earlier launch whose output the launch reads;
  * every read-after-write, write-after-read and write-after-write pair of
    launches on a shared buffer is ordered by the dependency graph.
"""
import os
import sys

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _key(t):
    return t.untyped_storage().data_ptr()


class _Recorder:
    """Allocates CPU buffers and records (reads, writes) per call, by storage."""

    def __init__(self):
        self.log = []

    def _rec(self, reads, writes):
        self.log.append(({_key(t) for t in reads if t is not None}, {_key(t) for t in writes if t is not None}))

    # allocation and sizing
    def alloc_compressed(self, R, K, dtype, dev, sm100=True):
        return (torch.empty((R, K // 2), dtype=dtype, device=dev), torch.empty((R, K // 4), dtype=torch.uint8, device=dev),
                torch.empty((128, 128), dtype=torch.uint8, device=dev))

    def alloc_compressed12(self, R, K, dtype, dev):
        return torch.empty((R, K // 2), dtype=dtype, device=dev), torch.empty((R, K // 16 + 1), dtype=torch.uint8, device=dev)

    def nm_spmm_workspace_bytes(self, dtype, R, K, T):
        return 256           # as if every product needed scratch: concurrent products must not share it

    # entry points: reads, then writes
    def nm_mask(self, W, N, M, mask):
        self._rec([W], [mask])

    def nm_mask_transposable(self, W, N, M, mask):
        self._rec([W], [mask])

    def nm_mask_scored(self, W, D, N, M, mask):
        self._rec([W, D], [mask])

    def nm_srste_step(self, W, G, N, M, decay, W_sparse, grad_out, mask):
        self._rec([W, G], [W_sparse, grad_out, mask])

    def nm_compress(self, W, mask, values, meta, img):
        self._rec([W, mask], [values, meta, img])

    def nm_compress_t(self, W, mask, values, meta, img):
        self._rec([W, mask], [values, meta, img])

    def nm_mask_compress(self, W, values, meta, img, sm100=True):
        self._rec([W], [values, meta, img])

    def nm_meta_s8_image_bytes(self, R, K):
        return 256

    def nm_meta12_image_bytes(self, R, K):
        return 256

    def nm_meta_to_sm100_s8(self, meta, R, K, out):
        self._rec([meta], [out])

    def nm_meta12_to_sm100(self, meta, R, K, out):
        self._rec([meta], [out])

    def nm_spmm12(self, values, img, X, Y):
        self._rec([values, img, X], [Y])

    def nm_meta_to_sm100(self, meta, R, K, out):
        self._rec([meta], [out])

    def nm_decompress(self, values, meta, K, out):
        self._rec([values, meta], [out])

    def nm_compress12(self, W, mask, values, meta):
        self._rec([W, mask], [values, meta])

    def nm_mask_compress12(self, W, values, meta):
        self._rec([W], [values, meta])

    def nm_decompress12(self, values, meta, K, out):
        self._rec([values, meta], [out])

    def nm_spmm(self, values, img, X, Y, workspace=None):
        self._rec([values, img, X], [Y, workspace])


def _bf16(*shape):
    return torch.randn(shape).to(torch.bfloat16)


R, K, T = 32, 64, 8
WORKLOADS = {
    "linear": {"W": _bf16(R, K), "X": _bf16(K, T), "R": R, "K": K, "T": T},
    "mlp": {"W": _bf16(R, K), "W2": _bf16(K, R), "X": _bf16(K, T), "R": R, "K": K, "T": T},
    "trans24": {"W": _bf16(R, K), "X": _bf16(K, T), "DY": _bf16(R, T), "T24": True, "R": R, "K": K, "T": T},
    "ties": {"W": torch.randn(R, K), "X": None, "R": R, "K": K, "T": 0},
    "int8": {"W": torch.randint(-128, 128, (R, K), dtype=torch.int16).to(torch.int8), "I8": True,
             "X": torch.randint(-128, 128, (K, T), dtype=torch.int16).to(torch.int8),
             "R": R, "K": K, "T": 0},
    "pairs": {"W": torch.randn(R, K), "P12": True, "X": torch.randn(K, T), "R": R, "K": K, "T": T},
    "transposable": {"W": _bf16(R, K), "TM": (4, 8), "X": None, "R": R, "K": K, "T": 0},
    "scored": {"W": _bf16(R, K), "D": torch.rand(K), "X": None, "R": R, "K": K, "T": 0},
    "srste": {"W": _bf16(R, K), "G": _bf16(R, K), "X": None, "R": R, "K": K, "T": 0},
}


def _closure(deps):
    """before[i] = every launch that the graph orders before launch i."""
    before = []
    for d in deps:
        s = set(d)
        for j in d:
            s |= before[j]
        before.append(s)
    return before


@pytest.mark.parametrize("kind", sorted(WORKLOADS))
def test_dependency_graph_covers_the_data_flow(kind):
    rec = _Recorder()
    step = bench.Step(rec, WORKLOADS[kind], torch.device("cpu"))
    assert step.kind == kind
    calls, deps = step.calls(), step.deps()
    assert len(calls) == len(deps) == step.launches() == len(step.names)
    for fn in calls:
        fn()
    assert len(rec.log) == len(calls)
    before = _closure(deps)
    for i, d in enumerate(deps):
        reads_i, writes_i = rec.log[i]
        for j in d:
            assert 0 <= j < i, (kind, i, d)
            assert rec.log[j][1] & reads_i, "%s: launch %d waits for %d but reads none of its outputs" % (kind, i, j)
        for j in range(i):
            reads_j, writes_j = rec.log[j]
            if (writes_j & reads_i) or (reads_j & writes_i) or (writes_j & writes_i):
                assert j in before[i], "%s: launches %d (%s) and %d (%s) share a buffer but are not ordered" % (
                    kind, j, step.names[j], i, step.names[i])


class _FakeDist:
    """Stands in for torch.distributed in the row-split MLP step: the all-gather
    of H is recorded like a launch (reads this rank's H rows, writes all of H)."""

    def __init__(self, rec):
        self.rec = rec

    def get_world_size(self):
        return 2

    def get_backend(self):
        return "nccl"

    def all_gather_into_tensor(self, out, local):
        self.rec._rec([local], [out])


def test_row_split_mlp_step_orders_the_all_gather():
    """--split rows: up product -> all-gather of H -> down product, and every
    buffer shared between launches ordered by the graph."""
    rec = _Recorder()
    wl = bench.split_workload(WORKLOADS["mlp"], 2, 0, _FakeDist(rec))
    step = bench.Step(rec, wl, torch.device("cpu"))
    calls, deps = step.calls(), step.deps()
    assert "all_gather_H" in step.names and len(calls) == len(deps) == len(step.names)
    for fn in calls:
        fn()
    before = _closure(deps)
    for i, d in enumerate(deps):
        reads_i, writes_i = rec.log[i]
        for j in d:
            assert rec.log[j][1] & reads_i
        for j in range(i):
            reads_j, writes_j = rec.log[j]
            if (writes_j & reads_i) or (reads_j & writes_i) or (writes_j & writes_i):
                assert j in before[i], (step.names[j], step.names[i])
    up, ag, down = (step.names.index(n) for n in ("nm_spmm_up", "all_gather_H", "nm_spmm_down"))
    assert up in before[ag] and ag in before[down]


def test_the_linear_step_forks():
    """The default step is not a chain: after the fused mask+compress, the
    image reorder, the decompression and the product are independent."""
    deps = bench.Step(_Recorder(), WORKLOADS["linear"], torch.device("cpu")).deps()
    assert deps == [[], [0], [], [2], [2], [2]]


def test_closure_catches_a_planted_race():
    """The check itself: a graph with the product's edge removed fails it."""
    rec = _Recorder()
    step = bench.Step(rec, WORKLOADS["mlp"], torch.device("cpu"))
    for fn in step.calls():
        fn()
    deps = step.deps()
    up, down = step.names.index("nm_spmm_up"), step.names.index("nm_spmm_down")
    planted = [d if i != down else [j for j in d if j != up] for i, d in enumerate(deps)]
    before = _closure(planted)                            # the down product no longer waits for the up product
    reads_down = rec.log[down][0]
    writes_up = rec.log[up][1]
    assert writes_up & reads_down and up not in before[down]


class _FusedRecorder(_Recorder):
    """The recorder plus the peer calls: nm_spmm_peers writes every destination
    that is a tensor of this process (other ranks' buffers are addresses), the
    signal writes every flag array of this process and the wait reads them."""

    def __init__(self):
        super().__init__()
        self.peers_calls, self.epochs = [], []

    def nm_ipc_handle(self, t):
        return bytes(64), 0

    def nm_ipc_open(self, handle, offset):
        return 0x7000_0000 + offset

    def nm_spmm_peers(self, values, img, X, dests, row0, ldy):
        own = [d for d in dests if isinstance(d, torch.Tensor)]
        self.peers_calls.append((own, row0, ldy, len(dests)))
        self._rec([values, img, X], own)

    def nm_peer_signal(self, flags, rank, epoch):
        self.epochs.append((rank, epoch))
        self._rec([], [f for f in flags if isinstance(f, torch.Tensor)])

    def nm_peer_wait(self, flags, epoch, timeout_ns):
        self._rec([flags], [])


class _FakeDist2(_FakeDist):
    def get_rank(self):
        return 0          # the rank that holds rows (slices are whole 256-row tiles)

    def all_gather_object(self, out, obj):
        for i in range(len(out)):
            out[i] = obj

    def barrier(self):
        pass


def test_row_split_mlp_fused_exchange():
    """--split rows --gather fused: up product (stores into every rank's H)
    -> signal -> wait -> down product, ordered by the graph; H alternates
    between two buffers by step, and the down product reads the buffer its
    step's up product wrote."""
    rec = _FusedRecorder()
    wl = bench.split_workload(WORKLOADS["mlp"], 2, 0, _FakeDist2(rec), gather="fused")
    step = bench.Step(rec, wl, torch.device("cpu"))
    assert step.fused
    names = step.names
    up, sig, wait, down = (names.index(n) for n in ("nm_spmm_up", "peer_signal", "peer_wait", "nm_spmm_down"))
    assert up < sig < wait < down and "all_gather_H" not in names
    deps = step.deps()
    assert len(step.calls()) == len(deps) == len(names) == step.own_launches()
    before = _closure(deps)
    assert up in before[sig] and sig in before[wait] and wait in before[down]
    for s in range(2):
        rec.log.clear()
        for fn in step.calls():
            fn()
        own, row0, ldy, n_dest = rec.peers_calls[-1]
        assert n_dest == 2 and row0 == wl["rows"][0] and len(own) == 1
        assert own[0].data_ptr() == step.H_bufs[(s + 1) % 2].data_ptr()
        assert _key(step.H_down) == _key(own[0])                  # the down product reads what up wrote
        assert rec.epochs[-1] == (0, s + 1)
        reads_down = rec.log[down][0]
        assert _key(own[0]) in reads_down
        for i in range(len(names)):
            reads_i, writes_i = rec.log[i]
            for j in range(i):
                reads_j, writes_j = rec.log[j]
                if (writes_j & reads_i) or (reads_j & writes_i) or (writes_j & writes_i):
                    assert j in before[i], (names[j], names[i])
    bench.IPC_MAPPINGS.clear()
