"""GPU parity of the 1:2 compression kernels against the CPU oracle (values,
metadata and decompressed matrices compared bit for bit)."""
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


DT = [torch.float32, torch.bfloat16, torch.float16]


@pytest.mark.parametrize("dtype", DT)
@pytest.mark.parametrize("R,C", [(1, 16), (37, 48), (128, 256), (300, 1040)])
def test_fused_matches_mask_then_compress(dtype, R, C):
    W = nm_inputs.normal((R, C), R + C, 1.0, dtype)
    v, m = nm.nm_mask_compress12(W.cuda())
    Wb = _bits(W)
    mask = oracle.mask_rank(Wb, 1, 2, dtype=CODE[dtype])
    rv, rm = oracle.compress12(Wb, mask, dtype=CODE[dtype])
    assert np.array_equal(_bits(v), rv.view(Wb.dtype))
    assert np.array_equal(m.cpu().numpy(), rm)
    back = nm.nm_decompress12(v, m, C).cpu()
    assert np.array_equal(_bits(back), oracle.decompress12(rv, rm, C, dtype=CODE[dtype]).view(Wb.dtype))


@pytest.mark.parametrize("dtype", DT)
def test_ties_keep_the_first(dtype):
    W = nm_inputs.small_int((64, 128), 7, lo=-2, hi=2, dtype=dtype)
    v, m = nm.nm_mask_compress12(W.cuda())
    rv, rm = oracle.compress12(_bits(W), oracle.mask_rank(_bits(W), 1, 2, dtype=CODE[dtype]), dtype=CODE[dtype])
    assert np.array_equal(m.cpu().numpy(), rm)


@pytest.mark.parametrize("dtype", DT)
def test_given_mask_and_invalid_pairs(dtype):
    R, C = 96, 64
    W = nm_inputs.normal((R, C), 8, 1.0, dtype)
    g = torch.Generator().manual_seed(9)
    second = torch.randint(0, 2, (R, C // 2), generator=g, dtype=torch.uint8)
    mask = torch.stack([1 - second, second], dim=2).reshape(R, C).contiguous()
    v, m = nm.nm_compress12(W.cuda(), mask.cuda())
    rv, rm = oracle.compress12(_bits(W), mask.numpy(), dtype=CODE[dtype])
    assert np.array_equal(_bits(v), rv.view(_bits(W).dtype)) and np.array_equal(m.cpu().numpy(), rm)
    bad = mask.clone()
    bad[3, 10:12] = 1          # both kept
    bad[5, 20:22] = 0          # none kept
    bad[7, 30] = 2             # not a 0/1 byte
    cnt = torch.zeros(1, dtype=torch.int32, device="cuda")
    v2, m2 = nm.nm_compress12(W.cuda(), bad.cuda(), invalid_pairs=cnt)
    assert int(cnt.item()) == 3
    # an invalid pair stores its first element with index 0
    assert _bits(v2)[3, 5] == _bits(W)[3, 10] and ((m2.cpu().numpy()[3, 0] >> 5) & 1) == 0


def test_strided_rows_and_decompress_leading_dim():
    R, C = 40, 64
    Wfull = nm_inputs.normal((R, C + 32), 10, 1.0, torch.float32).cuda()
    W = Wfull[:, :C]
    v, m = nm.nm_mask_compress12(W)
    out = torch.full((R, C + 16), 7.0, device="cuda")
    nm.nm_decompress12(v, m, C, out=out[:, :C])
    Wb = _bits(W.contiguous())
    rv, rm = oracle.compress12(Wb, oracle.mask_rank(Wb, 1, 2), dtype=oracle.F32)
    assert np.array_equal(_bits(out[:, :C].contiguous()), oracle.decompress12(rv, rm, C, dtype=oracle.F32))
    assert torch.all(out[:, C:] == 7.0)


def test_fp32_workload_full_size():
    """fp32 8192 x 8192 (the ties workload, many exact ties), every row."""
    W = nm_inputs.ties_fp32()
    v, m = nm.nm_mask_compress12(W.cuda())
    Wb = _bits(W)
    rv, rm = oracle.compress12(Wb, oracle.mask_rank(Wb, 1, 2), dtype=oracle.F32)
    assert np.array_equal(_bits(v), rv) and np.array_equal(m.cpu().numpy(), rm)


def test_argument_errors():
    lib = nm.load()
    W = torch.zeros((8, 24), dtype=torch.float32, device="cuda")
    v = torch.empty((8, 12), dtype=torch.float32, device="cuda")
    m = torch.empty((8, 2), dtype=torch.uint8, device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    assert lib.nm_mask_compress12(W.data_ptr(), 0, 8, 24, 24, v.data_ptr(), m.data_ptr(), s) == 2   # C % 16
    assert lib.nm_mask_compress12(None, 0, 8, 16, 24, v.data_ptr(), m.data_ptr(), s) == 1           # NULL
