"""GPU parity of nm_compress_t (2:4 compression of W^T under mask^T) against
the CPU oracle, and of the backward product dX = (W (.) mask)^T dY that it
feeds.  The oracle side is the oracle's own compression of the transposed
matrices: values, canonical metadata and the tensor-core image must match
byte for byte; the product must be within the bf16-output tolerance of the
oracle's fp64 product."""
import os

import numpy as np
import pytest
import torch

import oracle
import nm_inputs
import structured_sparsity_prune_b200 as nm

pytestmark = pytest.mark.gpu

CODE = {torch.float32: oracle.F32, torch.bfloat16: oracle.BF16, torch.float16: oracle.F16, torch.int8: oracle.S8}
THREADS = os.cpu_count() or 2


def _bits(t):
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.float32:
        return t.view(torch.int32).numpy().view(np.uint32)
    if t.dtype in (torch.bfloat16, torch.float16):
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


@pytest.fixture(scope="module", autouse=True)
def _built():
    from structured_sparsity_prune_b200 import build
    build.build()
    oracle.build()
    assert torch.cuda.is_available()


def _weights(shape, dtype, seed):
    if dtype == torch.int8:
        g = torch.Generator().manual_seed(seed)
        return torch.randint(-128, 128, shape, generator=g, dtype=torch.int16).to(torch.int8)
    return nm_inputs.normal(shape, seed, 1.0, dtype)


def _column_mask(R, C, seed):
    """A mask that is 2:4 down every column (groups of four consecutive rows)."""
    g = torch.Generator().manual_seed(seed)
    pairs = torch.tensor([(0, 1), (0, 2), (0, 3), (1, 2), (1, 3), (2, 3)])
    choice = pairs[torch.randint(0, 6, (R // 4, C), generator=g)]          # (R/4, C, 2)
    m = torch.zeros((R // 4, C, 4), dtype=torch.uint8)
    m.scatter_(2, choice, 1)
    return m.permute(0, 2, 1).reshape(R, C).contiguous()


def _dev(t, pad=16):
    """Device copy in a buffer whose rows are 16-byte aligned."""
    R, C = t.shape
    per = pad // t.element_size()
    buf = torch.zeros((R, (C + per - 1) // per * per), dtype=t.dtype, device="cuda")
    buf[:, :C] = t.cuda()
    return buf[:, :C]


def _check(W, mask):
    R, C = W.shape
    ctr = torch.zeros((1,), dtype=torch.int32, device="cuda")
    v, m, img = nm.nm_compress_t(_dev(W), _dev(mask), invalid_groups=ctr)
    torch.cuda.synchronize()
    Wt = np.ascontiguousarray(_bits(W).T)
    Mt = np.ascontiguousarray(mask.numpy().T)
    v_ref, m_ref = oracle.compress24(Wt, Mt, dtype=CODE[W.dtype])
    assert np.array_equal(_bits(v), np.ascontiguousarray(v_ref).view(_bits(v).dtype))
    assert np.array_equal(m.cpu().numpy(), m_ref)
    assert np.array_equal(img.cpu().numpy(), oracle.meta_sm100(m_ref, C, R))
    return int(ctr.item())


# R % 8 == 0 always; R % 32 != 0 and R % 16 != 0 take the byte-wise metadata
# and per-octet value stores; C not a multiple of the 16-byte chunk takes the
# element-wise staging loads; sizes past 128 pad the image in both directions.
SHAPES = [(256, 32), (256, 256), (512, 96), (136, 200), (8, 40), (1000, 48), (264, 130), (40, 1)]


@pytest.mark.parametrize("R,C", SHAPES)
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16, torch.float16, torch.int8])
def test_column_masks(R, C, dtype):
    W = _weights((R, C), dtype, R * 3 + C)
    assert _check(W, _column_mask(R, C, R + C)) == 0


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16, torch.int8])
def test_transposable_mask_from_the_oracle(dtype):
    """The greedy keeps at most two per row and column of a 4x4 block; the
    groups it leaves short are stored with +0.0 fillers on both sides."""
    R, C = 128, 96
    W = _weights((R, C), dtype, 11)
    mask = torch.from_numpy(oracle.mask_transposable(_bits(W), 2, 4, dtype=CODE[dtype]))
    assert _check(W, mask) == 0
    back = nm.nm_decompress(*nm.nm_compress_t(_dev(W), _dev(mask))[:2], R)
    assert np.array_equal(_bits(back), np.where(mask.numpy().T == 1, _bits(W).T, 0))


def test_invalid_and_sparser_groups():
    R, C = 64, 40
    W = _weights((R, C), torch.bfloat16, 5)
    mask = _column_mask(R, C, 6)
    bad = [(0, 0, [1, 1, 1, 0]), (60, 39, [2, 0, 1, 0])]                 # invalid
    sparse = [(4, 7, [0, 0, 0, 0]), (12, 33, [1, 0, 0, 0]), (20, 3, [0, 0, 0, 1])]   # valid, +0.0 fillers
    fixed = mask.clone()
    for r, c, pat in bad:
        mask[r:r + 4, c] = torch.tensor(pat, dtype=torch.uint8)
        fixed[r:r + 4, c] = torch.tensor([1, 1, 0, 0], dtype=torch.uint8)   # documented fallback (0,1)
    for r, c, pat in sparse:
        mask[r:r + 4, c] = torch.tensor(pat, dtype=torch.uint8)
        fixed[r:r + 4, c] = torch.tensor(pat, dtype=torch.uint8)
    ctr = torch.zeros((1,), dtype=torch.int32, device="cuda")
    v, m, img = nm.nm_compress_t(_dev(W), _dev(mask), invalid_groups=ctr)
    assert int(ctr.item()) == len(bad)
    v_ref, m_ref = oracle.compress24(np.ascontiguousarray(_bits(W).T), np.ascontiguousarray(fixed.numpy().T),
                                     dtype=oracle.BF16)
    assert np.array_equal(_bits(v), v_ref)
    assert np.array_equal(m.cpu().numpy(), m_ref)
    assert np.array_equal(img.cpu().numpy(), oracle.meta_sm100(m_ref, C, R))


def test_shape_and_alignment_errors():
    W = torch.zeros((12, 16), dtype=torch.bfloat16, device="cuda")
    mask = torch.zeros((12, 16), dtype=torch.uint8, device="cuda")
    with pytest.raises(RuntimeError):
        nm.nm_compress_t(W, mask)            # R % 8 != 0


def test_backward_product_on_the_transposed_operand():
    """dX = (W (.) mask)^T dY through nm_spmm on the transposed compression."""
    R, C, T = 512, 384, 200
    W = nm_inputs.normal((R, C), 21, 0.02, torch.bfloat16)
    dY = nm_inputs.normal((R, T), 22, 1.0, torch.bfloat16)
    mask = nm.nm_mask_transposable(W.cuda(), 2, 4)
    v, m, img = nm.nm_compress_t(W.cuda(), mask)
    dX = nm.nm_spmm(v, img, _dev(dY))
    torch.cuda.synchronize()
    assert nm.nm_last_device_status() == 0
    Wt = np.ascontiguousarray(_bits(W).T)
    v_ref, m_ref = oracle.compress24(Wt, np.ascontiguousarray(mask.cpu().numpy().T), dtype=oracle.BF16)
    ref = oracle.spmm(v_ref, m_ref, _bits(dY), oracle.BF16, threads=THREADS)
    dXf = dX.float().cpu().numpy().astype(np.float64)
    assert np.linalg.norm(dXf - ref) / np.linalg.norm(ref) <= 8e-3
    # and against the dense product on the masked transpose, independently of the compression
    Wm = (W.float() * mask.cpu().float()).double()
    dense = (Wm.T @ dY.double()).numpy()
    assert np.linalg.norm(dXf - dense) / np.linalg.norm(dense) <= 8e-3


def test_linear_4096_full_size():
    """The 4096 x 4096 bf16 weight under its transposable 2:4 mask, whole matrix, bit-exact."""
    W, _ = nm_inputs.linear_4096()
    mask = nm.nm_mask_transposable(W.cuda(), 2, 4)
    assert _check(W, mask.cpu()) == 0
