"""The row-split product's peer path on one GPU: nm_spmm_peers writing one
output into several buffers, the completion flags (nm_peer_signal /
nm_peer_wait, including a wait that gives up), and the IPC mappings between
two processes on the same GPU.

Only one GPU is available here, so "other GPUs" are stood in for by further
buffers on the same GPU, or by a second process whose buffers are reached
through CUDA IPC.  No kernel ever waits on a kernel of another process: the
child process finishes and exits before the parent's wait is launched, so
every wait here either finds its flags already set or runs out by design."""
import os
import sys
import time

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import nm_inputs  # noqa: E402
import oracle  # noqa: E402
import structured_sparsity_prune_b200 as nm  # noqa: E402

pytestmark = pytest.mark.gpu

SENTINEL = -3.0          # bf16 value that fills every destination before a call
TOL_BF16 = 8e-3          # normalised Frobenius error of a bf16 output against the fp64 oracle
THREADS = os.cpu_count() or 2


@pytest.fixture(scope="module", autouse=True)
def _built():
    from structured_sparsity_prune_b200 import build
    build.build()
    oracle.build()
    assert torch.cuda.is_available()


def _bits16(t):
    return t.detach().contiguous().view(torch.int16)


def _x_dev(X, ld):
    buf = torch.zeros((X.shape[0], ld), dtype=X.dtype, device="cuda")
    buf[:, :X.shape[1]] = X.cuda()
    return buf[:, :X.shape[1]]


def _reference(values, img, Xd, R, T, ldy):
    """nm_spmm into a buffer with the same leading dimension (same epilogue)."""
    buf = torch.empty((R, ldy), dtype=torch.bfloat16, device="cuda")
    return nm.nm_spmm(values, img, Xd, Y=buf[:, :T])


def _check_destination(buf, row0, R, T, want):
    assert torch.equal(_bits16(buf[row0:row0 + R, :T]), _bits16(want))
    outside = torch.ones(buf.shape, dtype=torch.bool, device=buf.device)
    outside[row0:row0 + R, :T] = False
    assert bool((buf[outside] == SENTINEL).all()), "a store landed outside the slice"


# (R, K, T, row0, n_peers, rows of each destination, ldy)
CASES = [
    (256, 256, 256, 0, 1, 256, 256),
    (512, 1024, 1000, 256, 2, 1024, 1000),       # ragged column tile
    (1000, 512, 328, 512, 3, 1600, 344),         # ragged row and column tiles, ldy > T
    (768, 2048, 2304, 128, 8, 1024, 2312),       # eight destinations, several column tiles
]


@pytest.mark.parametrize("R,K,T,row0,n_peers,rows,ldy", CASES)
def test_spmm_peers_writes_every_destination(R, K, T, row0, n_peers, rows, ldy):
    W = nm_inputs.normal((R, K), 301 + R, 0.02, torch.bfloat16)
    X = nm_inputs.normal((K, T), 302 + T, 1.0, torch.bfloat16)
    values, meta, img = nm.nm_mask_compress(W.cuda())
    Xd = _x_dev(X, (T + 7) // 8 * 8)
    dests = [torch.full((rows, ldy), SENTINEL, dtype=torch.bfloat16, device="cuda") for _ in range(n_peers)]
    nm.nm_spmm_peers(values, img, Xd, dests, row0, ldy)
    want = _reference(values, img, Xd, R, T, ldy)
    torch.cuda.synchronize()
    assert nm.nm_last_device_status() == 0
    for d in dests:
        _check_destination(d, row0, R, T, want)
    # and the result itself against the oracle (sampled rows, fp64)
    Wb = W.contiguous().view(torch.int16).numpy().view(np.uint16)
    Xb = X.contiguous().view(torch.int16).numpy().view(np.uint16)
    _, v_ref, m_ref = oracle.rows_parallel(1, Wb, 2, 4, oracle.BF16, threads=THREADS)
    rows_s = sorted(set([0, R - 1] + list(range(0, R, max(1, R // 24)))))
    ref = oracle.spmm(v_ref, m_ref, Xb, oracle.BF16, y_dtype=oracle.BF16, rows=rows_s, threads=THREADS)
    got = dests[-1][row0:row0 + R, :T].float().cpu().numpy().astype(np.float64)[rows_s]
    err = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    assert err < TOL_BF16, err


def test_spmm_peers_alpha_and_fp16():
    R, K, T = 512, 512, 640
    W = nm_inputs.normal((R, K), 311, 0.02, torch.float16)
    X = nm_inputs.normal((K, T), 312, 1.0, torch.float16)
    values, meta, img = nm.nm_mask_compress(W.cuda())
    Xd = _x_dev(X, T)
    dests = [torch.full((R, T), SENTINEL, dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    nm.nm_spmm_peers(values, img, Xd, dests, 0, T, alpha=0.5)
    buf = torch.empty((R, T), dtype=torch.bfloat16, device="cuda")
    want = nm.nm_spmm(values, img, Xd, Y=buf, alpha=0.5)
    torch.cuda.synchronize()
    for d in dests:
        _check_destination(d, 0, R, T, want)


@pytest.mark.parametrize("R,T,dtype,code", [
    (512, 128, torch.bfloat16, 6),    # 128 columns: the 128-column pair kernel, which has no peer stores
    (512, 64, torch.bfloat16, 6),     # the single-CTA kernels store through plain pointers
    (384, 512, torch.bfloat16, 6),    # three row tiles do not pair up
    (512, 512, torch.float32, 4),     # fp32 operands
    (512, 333, torch.bfloat16, 6),    # rows of Y not whole 16-byte units
])
def test_spmm_peers_unsupported(R, T, dtype, code):
    K = 256
    ld = (T + 7) // 8 * 8
    W = nm_inputs.normal((R, K), 321, 0.02, dtype)
    values, meta, img = nm.nm_mask_compress(W.cuda())
    Xd = _x_dev(nm_inputs.normal((K, T), 322, 1.0, dtype), ld)
    dest = torch.full((R, ld), SENTINEL, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(nm.NMError) as e:
        nm.nm_spmm_peers(values, img, Xd, [dest], 0, ld)
    assert e.value.status == code
    torch.cuda.synchronize()
    assert bool((dest == SENTINEL).all())


def test_flags_signal_then_wait():
    """Four stand-in GPUs, each with a four-slot flag array: every rank's
    signal reaches its slot on every array, and the waits that follow find
    them set."""
    n = 4
    flags = [torch.zeros(n, dtype=torch.int64, device="cuda") for _ in range(n)]
    for r in range(n):
        nm.nm_peer_signal(flags, r, 1)
    for j in range(n):
        nm.nm_peer_wait(flags[j], 1, timeout_ns=1_000_000_000)
    torch.cuda.synchronize()
    assert nm.nm_last_device_status() == 0
    assert all(f.tolist() == [1] * n for f in flags)
    # a later epoch from three ranks only: slot 3 still holds 1
    for r in range(n - 1):
        nm.nm_peer_signal(flags, r, 2)
    torch.cuda.synchronize()
    assert flags[0].tolist() == [2, 2, 2, 1]
    nm.nm_peer_wait(flags[0], 1, timeout_ns=1_000_000_000)      # an older epoch is already met
    torch.cuda.synchronize()
    assert nm.nm_last_device_status() == 0


def test_wait_gives_up_on_a_flag_nothing_sets():
    n = 3
    flags = [torch.zeros(n, dtype=torch.int64, device="cuda") for _ in range(n)]
    for r in range(n - 1):
        nm.nm_peer_signal(flags, r, 5)
    torch.cuda.synchronize()
    t0 = time.time()
    nm.nm_peer_wait(flags[1], 5, timeout_ns=2_000_000)           # 2 ms: slot 2 never reaches 5
    assert nm.nm_last_device_status() == nm.STATUS.index("NM_ERR_TIMEOUT")
    assert time.time() - t0 < 10.0
    assert nm.nm_last_device_status() == 0                        # read and cleared
    # the context is still usable: the missing rank signals, and the wait passes
    nm.nm_peer_signal(flags, n - 1, 5)
    nm.nm_peer_wait(flags[1], 5, timeout_ns=1_000_000_000)
    torch.cuda.synchronize()
    assert nm.nm_last_device_status() == 0
    assert flags[1].tolist() == [5, 5, 5]


def test_ipc_handle_offset():
    big = torch.zeros(1 << 20, dtype=torch.uint8, device="cuda")
    h0, o0 = nm.nm_ipc_handle(big)
    h1, o1 = nm.nm_ipc_handle(big[4096:])
    assert len(h0) == nm.NM_IPC_HANDLE_BYTES and h0 == h1
    assert o1 - o0 == 4096


# two "GPUs" as two processes on one GPU: the child computes rows
# [LO, R_ALL) and stores them into its own output and, through IPC, into the
# parent's; then it signals both flag arrays and exits.  The parent computes
# rows [0, LO), signals, waits (finding every flag set) and checks the whole.
R_ALL, K_IPC, T_IPC, LDY_IPC, LO = 1024, 512, 296, 304, 512


def _ipc_inputs(lo, hi):
    W = nm_inputs.normal((R_ALL, K_IPC), 331, 0.02, torch.bfloat16)[lo:hi].contiguous()
    X = nm_inputs.normal((K_IPC, T_IPC), 332, 1.0, torch.bfloat16)
    values, meta, img = nm.nm_mask_compress(W.cuda())
    return values, img, _x_dev(X, LDY_IPC)


def _child_main(h_handle, h_off, f_handle, f_off, q):
    try:
        torch.cuda.set_device(0)
        values, img, Xd = _ipc_inputs(LO, R_ALL)
        own = torch.full((R_ALL, LDY_IPC), SENTINEL, dtype=torch.bfloat16, device="cuda")
        own_flags = torch.zeros(2, dtype=torch.int64, device="cuda")
        peer_h = nm.nm_ipc_open(h_handle, h_off)
        peer_f = nm.nm_ipc_open(f_handle, f_off)
        nm.nm_spmm_peers(values, img, Xd, [own, peer_h], LO, LDY_IPC)
        nm.nm_peer_signal([own_flags, peer_f], 1, 1)
        want = _reference(values, img, Xd, R_ALL - LO, T_IPC, LDY_IPC)
        torch.cuda.synchronize()
        status = nm.nm_last_device_status()
        same = torch.equal(_bits16(own[LO:, :T_IPC]), _bits16(want))
        flags_ok = own_flags.tolist() == [0, 1]
        nm.nm_ipc_close(peer_h, h_off)
        nm.nm_ipc_close(peer_f, f_off)
        q.put(("ok", status, same, flags_ok))
    except Exception as exc:  # reported to the parent, which fails the test
        q.put(("error", repr(exc)))


def test_ipc_two_processes_one_gpu():
    H = torch.full((R_ALL, LDY_IPC), SENTINEL, dtype=torch.bfloat16, device="cuda")
    F = torch.zeros(2, dtype=torch.int64, device="cuda")
    hh, ho = nm.nm_ipc_handle(H)
    fh, fo = nm.nm_ipc_handle(F)
    torch.cuda.synchronize()                      # the fills are done before the child writes
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    child = ctx.Process(target=_child_main, args=(hh, ho, fh, fo, q))
    child.start()
    child.join(timeout=300)
    assert child.exitcode == 0
    msg = q.get(timeout=10)
    assert msg == ("ok", 0, True, True), msg
    assert F.tolist() == [0, 1]
    # the parent's own rows, its signal (the child's array is gone with the
    # child, so both slots of the list name this process's array), the wait
    values, img, Xd = _ipc_inputs(0, LO)
    nm.nm_spmm_peers(values, img, Xd, [H], 0, LDY_IPC)
    nm.nm_peer_signal([F, F], 0, 1)
    nm.nm_peer_wait(F, 1, timeout_ns=1_000_000_000)
    want_lo = _reference(values, img, Xd, LO, T_IPC, LDY_IPC)
    v_hi, i_hi, X_hi = _ipc_inputs(LO, R_ALL)
    want_hi = _reference(v_hi, i_hi, X_hi, R_ALL - LO, T_IPC, LDY_IPC)
    torch.cuda.synchronize()
    assert nm.nm_last_device_status() == 0
    assert torch.equal(_bits16(H[:LO, :T_IPC]), _bits16(want_lo))
    assert torch.equal(_bits16(H[LO:, :T_IPC]), _bits16(want_hi))
    assert bool((H[:, T_IPC:] == SENTINEL).all())
