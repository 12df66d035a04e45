"""GPU parity of the saliency-scored N:M mask (nm_mask_scored) against the
CPU oracle: masks must be identical byte for byte.  Both sides evaluate the
score fl(fl(w*w) / fl(d*d)) in binary32 with the same rounding, so the
decisions, ties included, are the same."""
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


def _check(W, d, N, M):
    got = nm.nm_mask_scored(W.cuda(), d.cuda(), N, M).cpu().numpy()
    ref = oracle.mask_scored(_bits(W), d.numpy(), N, M, dtype=CODE[W.dtype])
    assert np.array_equal(got, ref)


NM = [(1, 2), (1, 4), (2, 4), (3, 4), (2, 8), (4, 8), (1, 3), (2, 6)]


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16, torch.float16])
@pytest.mark.parametrize("N,M", NM)
def test_random_weights(dtype, N, M):
    C = 96 if 96 % M == 0 else 120
    W = nm_inputs.normal((200, C), 31 + M, 1.0, dtype)
    d = nm_inputs.normal((C,), 41 + M).abs() + 0.05
    _check(W, d, N, M)


@pytest.mark.parametrize("N,M", NM)
def test_many_exact_ties(N, M):
    C = 96 if 96 % M == 0 else 120
    W = nm_inputs.small_int((160, C), 51, lo=-4, hi=4, dtype=torch.bfloat16)
    g = torch.Generator().manual_seed(52)
    d = torch.tensor([0.5, 1.0, 2.0, 4.0])[torch.randint(0, 4, (C,), generator=g)].float()
    _check(W, d, N, M)


def test_zero_d_and_zero_weights():
    W = nm_inputs.normal((64, 64), 61, 1.0, torch.float32)
    W[::3, ::5] = 0.0
    d = nm_inputs.normal((64,), 62).abs()
    d[::7] = 0.0                       # x/0 = inf, 0/0 = NaN
    for N, M in [(2, 4), (1, 4), (4, 8)]:
        _check(W, d, N, M)


def test_scalar_path_when_c_is_not_a_multiple_of_16():
    """C = 40 (not a multiple of 16) takes the per-group path; rows of W and
    of the mask sit in buffers padded to 16-byte row strides."""
    C = 40
    Wfull = nm_inputs.normal((130, 48), 71, 1.0, torch.bfloat16).cuda()
    W = Wfull[:, :C]
    d = (nm_inputs.normal((C,), 72).abs() + 0.1).cuda()
    for N, M in [(2, 4), (1, 5), (3, 8)]:
        mfull = torch.full((130, 48), 9, dtype=torch.uint8, device="cuda")
        nm.nm_mask_scored(W, d, N, M, mask=mfull[:, :C])
        ref = oracle.mask_scored(_bits(W.contiguous()), d.cpu().numpy(), N, M, dtype=oracle.BF16)
        assert np.array_equal(mfull[:, :C].cpu().numpy(), ref)
        assert torch.all(mfull[:, C:] == 9)


def test_strided_rows():
    Wfull = nm_inputs.normal((100, 80), 73, 1.0, torch.float16).cuda()
    W = Wfull[:, :64]
    d = (nm_inputs.normal((64,), 74).abs() + 0.1).cuda()
    mfull = torch.full((100, 96), 7, dtype=torch.uint8, device="cuda")
    nm.nm_mask_scored(W, d, 2, 4, mask=mfull[:, :64])
    ref = oracle.mask_scored(_bits(W.contiguous()), d.cpu().numpy(), 2, 4, dtype=oracle.F16)
    assert np.array_equal(mfull[:, :64].cpu().numpy(), ref)
    assert torch.all(mfull[:, 64:] == 7)


def test_saliency_workload_full_size():
    """The linear_4096 weight with d from the synthetic inverse Hessian, every row."""
    W, _ = nm_inputs.linear_4096()
    d = nm_inputs.saliency_d(4096)
    _check(W, d, 2, 4)


def test_unit_d_equals_the_magnitude_mask():
    W = nm_inputs.normal((256, 256), 75, 1.0, torch.bfloat16).cuda()
    d = torch.ones(256, dtype=torch.float32, device="cuda")
    assert torch.equal(nm.nm_mask_scored(W, d, 2, 4), nm.nm_mask(W, 2, 4))


def test_argument_errors():
    W = torch.zeros((8, 16), dtype=torch.bfloat16, device="cuda")
    d = torch.ones(16, dtype=torch.float32, device="cuda")
    lib = nm.load()
    m = torch.empty((8, 16), dtype=torch.uint8, device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    assert lib.nm_mask_scored(W.data_ptr(), 1, None, 8, 16, 16, 2, 4, m.data_ptr(), 16, s) == 1       # NM_ERR_NULL
    assert lib.nm_mask_scored(W.data_ptr(), 1, d.data_ptr() + 4, 8, 16, 16, 2, 4, m.data_ptr(), 16, s) == 3  # ALIGN
    assert lib.nm_mask_scored(W.data_ptr(), 1, d.data_ptr(), 8, 16, 16, 4, 4, m.data_ptr(), 16, s) == 5  # NM_ERR_NM
    assert lib.nm_mask_scored(W.data_ptr(), 1, d.data_ptr(), 8, 15, 16, 2, 4, m.data_ptr(), 16, s) == 2  # SHAPE


@pytest.mark.parametrize("N,M", [(2, 4), (1, 4), (4, 8)])
def test_scores_one_ulp_apart(N, M):
    """w = c * d in binary32: every score of a group is c^2 up to the rounding
    of the two squares and the quotient, so scores tie or differ by an ulp or
    two and the mask depends on every quotient's last bit."""
    g = torch.Generator().manual_seed(76)
    R, C = 1024, 512
    d = (torch.rand(C, generator=g) * 3.5 + 0.5).float()
    c = (torch.rand(R, 1, generator=g) * 2.0 + 0.01).float()
    W = (c * d[None, :]).float()
    _check(W, d, N, M)
