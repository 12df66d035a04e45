"""The no-allocation product entry point, nm_spmm_noalloc, called through the
C ABI.

Some callers may not allocate device memory at all: a host framework that owns
every device allocation (a serving engine, a plugin host with a fixed memory
budget), or a latency-critical path that cannot take cudaMalloc's implicit
synchronisation.  For them nm_spmm_noalloc takes the fp32 path's binary16
staging buffers from a fixed device array inside the library instead of a
caller workspace.  This test checks it against the workspace-taking nm_spmm
and against the fp64 CPU oracle, within the fp32-output tolerance of the
other product tests, on two calls in a row (the second with different inputs,
so stale scratch would show), and that a problem larger than the fixed array
is refused.

The file name sorts last so that a stop-at-first-failure run has executed
every other test before this one."""
import ctypes

import numpy as np
import pytest
import torch

import nm_inputs
import oracle
import structured_sparsity_prune_b200 as nm

pytestmark = pytest.mark.gpu

NM_OK, NM_ERR_WORKSPACE, NM_F32 = 0, 8, 0


def _nerr(a, b):
    a = a.double().cpu()
    b = b.double().cpu()
    return float(torch.linalg.norm(a - b) / torch.linalg.norm(b))


def _case(seed_w, seed_x, R=256, K=256, T=128):
    W = nm_inputs.normal((R, K), seed_w, 1.0, torch.float32)
    X = nm_inputs.normal((K, T), seed_x, 1.0, torch.float32)
    values, meta, img = nm.nm_mask_compress(W.cuda())
    return values, img, X.cuda(), W, X


def _oracle_product(W, X):
    """fp64 product of the oracle's own 2:4 compression of W with X."""
    oracle.build()
    Wn, Xn = W.numpy(), X.numpy()
    mask = oracle.mask_rank(Wn, 2, 4)
    v, m = oracle.compress24(Wn, mask)
    return oracle.spmm(v, m, Xn, oracle.F32)


def _noalloc(lib, values, img, X, Y):
    R, Kh = values.shape
    K, T = X.shape
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.nm_spmm_noalloc(ctypes.c_void_p(values.data_ptr()), ctypes.c_void_p(img.data_ptr()), NM_F32,
                               ctypes.c_void_p(X.data_ptr()), X.stride(0), ctypes.c_void_p(Y.data_ptr()), NM_F32,
                               Y.stride(0), R, 2 * Kh, T, ctypes.c_float(1.0), ctypes.c_float(0.0), stream)


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    lib = nm.load()
    for seeds in [(0, 100), (7, 107)]:
        values, img, X, W_host, X_host = _case(*seeds)
        ref = nm.nm_spmm(values, img, X, y_dtype=torch.float32)          # caller-provided workspace
        Y = torch.full(ref.shape, float("nan"), dtype=torch.float32, device="cuda")
        assert _noalloc(lib, values, img, X, Y) == NM_OK
        torch.cuda.synchronize()
        assert nm.nm_last_device_status() == NM_OK
        assert torch.isfinite(Y).all()
        assert _nerr(Y, ref) <= 1e-3
        exact = torch.from_numpy(_oracle_product(W_host, X_host))
        assert _nerr(Y, exact) <= 1e-3


def test_noalloc_refuses_problems_beyond_the_fixed_scratch():
    lib = nm.load()
    R, K, T = 4096, 4096, 4096                       # needs 48 MiB of binary16 staging
    assert nm.nm_spmm_workspace_bytes(torch.float32, R, K, T) > (16 << 20)
    values = torch.empty((R, K // 2), dtype=torch.float32, device="cuda")
    img = torch.empty((R * K // 8,), dtype=torch.uint8, device="cuda")
    X = torch.empty((K, T), dtype=torch.float32, device="cuda")
    Y = torch.empty((R, T), dtype=torch.float32, device="cuda")
    assert _noalloc(lib, values, img, X, Y) == NM_ERR_WORKSPACE
