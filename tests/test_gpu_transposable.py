"""GPU parity of the greedy transposable N:M mask (nm_mask_transposable)
against the CPU oracle: masks must be identical byte for byte (the greedy's
decisions are integer comparisons of magnitude keys and positions)."""
import numpy as np
import pytest
import torch

import oracle
import nm_inputs
import structured_sparsity_prune_b200 as nm

pytestmark = pytest.mark.gpu

CODE = {torch.float32: oracle.F32, torch.bfloat16: oracle.BF16, torch.float16: oracle.F16}


def _bits(t):
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.float32:
        return t.view(torch.int32).numpy().view(np.uint32)
    return t.view(torch.int16).numpy().view(np.uint16)


@pytest.fixture(scope="module", autouse=True)
def _built():
    from structured_sparsity_prune_b200 import build
    build.build()
    oracle.build()
    assert torch.cuda.is_available()


def _check(W, N, M):
    got = nm.nm_mask_transposable(W.cuda(), N, M).cpu().numpy()
    ref = oracle.mask_transposable(_bits(W), N, M, dtype=CODE[W.dtype])
    assert np.array_equal(got, ref)
    return got


NM = [(1, 2), (1, 4), (2, 4), (3, 4), (4, 8), (2, 8), (1, 8), (7, 8), (1, 3), (2, 5), (3, 6), (3, 7)]


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16, torch.float16])
@pytest.mark.parametrize("N,M", NM)
def test_random_weights(dtype, N, M):
    # columns: a multiple of M that keeps rows 16-byte aligned for every dtype
    C = M * 16
    W = nm_inputs.normal((M * 20, C), 100 + 10 * N + M, 1.0, dtype)
    m = _check(W, N, M)
    b = m.reshape(20, M, 16, M)
    assert (b.sum(axis=3) <= N).all() and (b.sum(axis=1) <= N).all()


@pytest.mark.parametrize("N,M", [(4, 8), (2, 4), (2, 8)])
def test_many_exact_ties(N, M):
    W = nm_inputs.small_int((M * 32, M * 32), 120 + M, lo=-3, hi=3, dtype=torch.bfloat16)
    _check(W, N, M)


def test_all_zero_and_all_equal_blocks():
    W = torch.zeros((64, 64), dtype=torch.float32)
    W[32:, :] = 1.0
    W[:8, 8:16] = -0.0
    _check(W, 4, 8)


def test_strided_rows():
    Wfull = nm_inputs.normal((64, 96), 130, 1.0, torch.bfloat16).cuda()
    W = Wfull[:, :64]
    mfull = torch.full((64, 80), 5, dtype=torch.uint8, device="cuda")
    nm.nm_mask_transposable(W, 4, 8, mask=mfull[:, :64])
    ref = oracle.mask_transposable(_bits(W.contiguous()), 4, 8, dtype=oracle.BF16)
    assert np.array_equal(mfull[:, :64].cpu().numpy(), ref)
    assert torch.all(mfull[:, 64:] == 5)


def test_linear_4096_full_size():
    W, _ = nm_inputs.linear_4096()
    _check(W, 4, 8)


def test_transposed_weight_gives_the_transposed_mask():
    W = nm_inputs.normal((256, 512), 131, 1.0, torch.float32)
    a = nm.nm_mask_transposable(W.cuda(), 4, 8).cpu()
    b = nm.nm_mask_transposable(W.t().contiguous().cuda(), 4, 8).cpu()
    assert torch.equal(a.t(), b)


def test_argument_errors():
    W = torch.zeros((16, 16), dtype=torch.bfloat16, device="cuda")
    m = torch.empty((16, 16), dtype=torch.uint8, device="cuda")
    lib = nm.load()
    s = torch.cuda.current_stream().cuda_stream
    assert lib.nm_mask_transposable(W.data_ptr(), 1, 16, 16, 16, 8, 8, m.data_ptr(), 16, s) == 5   # N >= M
    assert lib.nm_mask_transposable(W.data_ptr(), 1, 12, 16, 16, 4, 8, m.data_ptr(), 16, s) == 2   # R % M
    assert lib.nm_mask_transposable(W.data_ptr(), 1, 16, 12, 16, 4, 8, m.data_ptr(), 16, s) == 2   # C % M
    assert lib.nm_mask_transposable(None, 1, 16, 16, 16, 4, 8, m.data_ptr(), 16, s) == 1           # NULL
