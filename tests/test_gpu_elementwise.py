"""GPU parity: mask, fused mask+compress, compress, decompress and the
metadata image, bit for bit against the CPU oracle on the same seeded inputs."""
import os

import numpy as np
import pytest
import torch

import oracle
import nm_inputs
import structured_sparsity_prune_b200 as nm

pytestmark = pytest.mark.gpu

CODE = {torch.float32: oracle.F32, torch.bfloat16: oracle.BF16, torch.float16: oracle.F16, torch.int8: oracle.S8}


def _bits(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.float32:
        return t.view(torch.int32).numpy().view(np.uint32)
    if t.dtype in (torch.bfloat16, torch.float16):
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def _rand(shape, dtype, seed, kind="normal"):
    if kind == "ties":
        return nm_inputs.ties(shape, seed).to(dtype)
    if kind == "special":
        g = torch.Generator().manual_seed(seed)
        x = torch.randn(*shape, generator=g)
        pick = torch.randint(0, 10, shape, generator=g)
        x[pick == 0] = 0.0
        x[pick == 1] = -0.0
        x[pick == 2] = float("inf")
        x[pick == 3] = float("-inf")
        x[pick == 4] = float("nan")
        x[pick == 5] = 1e-40 if dtype == torch.float32 else 1e-6   # subnormal-ish
        return x.to(dtype)
    return nm_inputs.normal(shape, seed, 1.0, dtype)


@pytest.fixture(scope="module", autouse=True)
def _built():
    from structured_sparsity_prune_b200 import build
    build.build()
    oracle.build()
    assert torch.cuda.is_available()


NM = [(1, 2), (1, 4), (2, 4), (3, 4), (1, 8), (2, 8), (4, 8), (7, 8), (2, 3), (2, 5), (3, 6), (4, 7)]


@pytest.mark.parametrize("N,M", NM)
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16, torch.float16])
@pytest.mark.parametrize("kind", ["normal", "ties", "special"])
def test_mask_small(N, M, dtype, kind):
    R, C = 67, M * 48            # ragged rows; C a multiple of 16 when M | 16
    W = _rand((R, C), dtype, 10 * N + M, kind)
    got = nm.nm_mask(W.cuda(), N, M).cpu().numpy()
    ref = oracle.mask_rank(_bits(W), N, M, dtype=CODE[dtype])
    assert np.array_equal(got, ref)


@pytest.mark.parametrize("N,M", [(2, 4), (4, 8)])
def test_mask_strided_and_unaligned_c(N, M):
    """ldw > C and C not a multiple of 16 (scalar path)."""
    R, C = 33, 24 if M == 4 else 40
    full = _rand((R, C + 8), torch.bfloat16, 3, "ties")
    W = full.cuda()[:, :C]
    mask = torch.full((R, 64), 7, dtype=torch.uint8, device="cuda")
    nm.nm_mask(W, N, M, mask=mask[:, :C])
    ref = oracle.mask_rank(_bits(full[:, :C]), N, M, dtype=oracle.BF16)
    assert np.array_equal(mask[:, :C].cpu().numpy(), ref)
    assert torch.all(mask[:, C:] == 7)   # nothing written past C


@pytest.mark.parametrize("N,M", [(1, 4), (2, 4), (4, 8), (2, 8)])
def test_mask_heavy_ties_full_size(N, M):
    """The 8192 x 8192 fp32 k/100 workload, whole matrix, bit-exact."""
    W = nm_inputs.ties_fp32()
    got = nm.nm_mask(W.cuda(), N, M).cpu().numpy()
    ref, _, _ = oracle.rows_parallel(0, _bits(W), N, M, oracle.F32, threads=max(1, (os.cpu_count() or 2)))
    assert np.array_equal(got, ref)



def _check_compressed(W, values, meta, img, code):
    Wb = _bits(W)
    R, C = Wb.shape
    mask = oracle.mask_rank(Wb, 2, 4, dtype=code)
    v_ref, m_ref = oracle.compress24(Wb, mask, dtype=code)
    assert np.array_equal(_bits(values), np.ascontiguousarray(v_ref).view(_bits(values).dtype))
    assert np.array_equal(meta.cpu().numpy(), m_ref)
    if img is not None:
        assert np.array_equal(img.cpu().numpy(), oracle.meta_sm100(m_ref, R, C))


# C % 32 == 0 takes the row-streaming compressor (image padded in rows and in
# 32-column units: 77 x 160, 300 x 96, 5 x 32); other C the tile compressor.
SHAPES = [(128, 128), (256, 256), (67, 200), (300, 392), (1, 8), (129, 136), (5, 32), (250, 1000),
          (77, 160), (300, 96), (1000, 384), (16, 4096)]


@pytest.mark.parametrize("R,C", SHAPES)
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16, torch.float16])
def test_mask_compress(R, C, dtype):
    W = _rand((R, C), dtype, R + C, "special" if dtype != torch.float32 else "normal")
    values, meta, img = nm.nm_mask_compress(W.cuda())
    _check_compressed(W, values, meta, img, CODE[dtype])


def test_mask_compress_without_image_and_strided():
    R, C = 96, 256
    full = _rand((R, C + 64), torch.bfloat16, 42, "ties")
    values, meta, img = nm.nm_mask_compress(full.cuda()[:, :C], sm100=False)
    assert img is None
    _check_compressed(full[:, :C], values, meta, None, oracle.BF16)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16, torch.int8])
def test_mask_compress_strided_with_image(dtype):
    R, C = 200, 160
    if dtype == torch.int8:
        full = torch.randint(-128, 128, (R, C + 32), generator=torch.Generator().manual_seed(5), dtype=torch.int8)
    else:
        full = _rand((R, C + 32), dtype, 43, "normal")
    values, meta, img = nm.nm_mask_compress(full.cuda()[:, :C])
    _check_compressed(full[:, :C], values, meta, img, CODE[dtype])


# 16-bit weights with C % 256 == 0 and at least 2^27 entries take the staged
# fused compressor (64-row x 256-column tiles through a shared-memory ring):
# ragged R (not a multiple of 64 or 128), strided rows, and no image; the
# whole matrix is compared.
RING_CASES = [(16449, 8192, 0), (16384, 8448, 256), (134217, 1024, 0)]


@pytest.mark.parametrize("R,C,pad", RING_CASES)
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_mask_compress_staged(R, C, pad, dtype):
    full = _rand((R, C + pad), dtype, R + C + pad, "special")
    Wd = full.cuda()[:, :C]
    values, meta, img = nm.nm_mask_compress(Wd)
    _check_compressed(full[:, :C], values, meta, img, CODE[dtype])
    v2, m2, none = nm.nm_mask_compress(Wd, sm100=False)
    assert none is None
    assert torch.equal(v2.view(torch.int16), values.view(torch.int16)) and torch.equal(m2, meta)
    assert nm.nm_last_device_status() == 0


@pytest.mark.parametrize("R,C", [(256, 256), (67, 200), (130, 64), (77, 160), (1000, 384)])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_compress_with_given_mask(R, C, dtype):
    W = _rand((R, C), dtype, 7, "normal")
    # a valid but not magnitude-based mask: random (i0 < i1) per group
    g = torch.Generator().manual_seed(9)
    pairs = torch.tensor([(0, 1), (0, 2), (0, 3), (1, 2), (1, 3), (2, 3)])
    choice = pairs[torch.randint(0, 6, (R, C // 4), generator=g)]
    mask = torch.zeros((R, C // 4, 4), dtype=torch.uint8)
    mask.scatter_(2, choice, 1)
    mask = mask.reshape(R, C)
    ctr = torch.zeros((1,), dtype=torch.int32, device="cuda")
    mbuf = torch.zeros((R, (C + 15) // 16 * 16), dtype=torch.uint8, device="cuda")   # 16-byte rows
    mbuf[:, :C] = mask.cuda()
    values, meta, img = nm.nm_compress(W.cuda(), mbuf[:, :C], invalid_groups=ctr)
    v_ref, m_ref = oracle.compress24(_bits(W), mask.numpy(), dtype=CODE[dtype])
    assert np.array_equal(_bits(values), np.ascontiguousarray(v_ref).view(_bits(values).dtype))
    assert np.array_equal(meta.cpu().numpy(), m_ref)
    assert np.array_equal(img.cpu().numpy(), oracle.meta_sm100(m_ref, R, C))
    assert int(ctr.item()) == 0


def test_compress_counts_invalid_groups():
    R, C = 64, 128
    W = _rand((R, C), torch.bfloat16, 1)
    mask = torch.zeros((R, C), dtype=torch.uint8)
    mask[:, 0::4] = 1
    mask[:, 1::4] = 1
    # invalid: more than two ones, a byte other than 0/1.  Valid but sparser:
    # none or one kept (stored with +0.0 fillers at the lowest unkept positions).
    bad = [(0, 0, [1, 1, 1, 0]), (63, 31, [2, 0, 1, 0])]
    sparse = [(3, 5, [0, 0, 0, 0]), (10, 7, [1, 0, 0, 0]), (20, 2, [0, 0, 1, 0])]
    fixed = mask.clone()
    for r, g, pat in bad:
        mask[r, 4 * g:4 * g + 4] = torch.tensor(pat, dtype=torch.uint8)
        fixed[r, 4 * g:4 * g + 4] = torch.tensor([1, 1, 0, 0], dtype=torch.uint8)   # fallback (0,1), W's values
    for r, g, pat in sparse:
        mask[r, 4 * g:4 * g + 4] = torch.tensor(pat, dtype=torch.uint8)
        fixed[r, 4 * g:4 * g + 4] = torch.tensor(pat, dtype=torch.uint8)
    ctr = torch.zeros((1,), dtype=torch.int32, device="cuda")
    values, meta, img = nm.nm_compress(W.cuda(), mask.cuda(), invalid_groups=ctr)
    assert int(ctr.item()) == len(bad)
    v_ref, m_ref = oracle.compress24(_bits(W), fixed.numpy(), dtype=oracle.BF16)
    assert np.array_equal(_bits(values), v_ref)
    assert np.array_equal(meta.cpu().numpy(), m_ref)
    assert np.array_equal(img.cpu().numpy(), oracle.meta_sm100(m_ref, R, C))
    m = meta.cpu().numpy()
    for r, g, _ in bad + sparse[:2]:      # pattern (0,1)
        assert (m[r, g // 2] >> (4 * (g % 2))) & 0xF == 0x4


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("R,C", [(64, 128), (77, 208)])   # row and tile compressors
def test_compress_sparser_masks_roundtrip(dtype, R, C):
    """1:4 magnitude masks through nm_compress: the oracle's form, and
    decompression gives select(mask, W, +0.0)."""
    W = _rand((R, C), dtype, 31, "special")
    mask = nm.nm_mask(W.cuda(), 1, 4)
    values, meta, img = nm.nm_compress(W.cuda(), mask)
    v_ref, m_ref = oracle.compress24(_bits(W), mask.cpu().numpy(), dtype=CODE[dtype])
    assert np.array_equal(_bits(values), np.ascontiguousarray(v_ref).view(_bits(values).dtype))
    assert np.array_equal(meta.cpu().numpy(), m_ref)
    assert np.array_equal(img.cpu().numpy(), oracle.meta_sm100(m_ref, R, C))
    back = _bits(nm.nm_decompress(values, meta, C))
    assert np.array_equal(back, np.where(mask.cpu().numpy() == 1, _bits(W), 0))


# staged-read decompression (C % 32 == 0, R*C % 128 == 0): a partial last
# 8192-element unit, rows that straddle units, one row, a single unit
RING_SHAPES = [(67, 256), (7, 2176), (1, 128), (3, 8192), (129, 4096), (516, 96)]


@pytest.mark.parametrize("R,C", SHAPES + RING_SHAPES)
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16, torch.float16])
def test_decompress(R, C, dtype):
    W = _rand((R, C), dtype, 3 * R + C, "special")
    Wb = _bits(W)
    code = CODE[dtype]
    mask = oracle.mask_rank(Wb, 2, 4, dtype=code)
    v_ref, m_ref = oracle.compress24(Wb, mask, dtype=code)
    vals = torch.from_numpy(np.ascontiguousarray(v_ref).view(np.int32 if code == oracle.F32 else np.int16))
    vals = vals.view(dtype).cuda()
    out = torch.full((R, C + 8), 3.0, dtype=dtype, device="cuda")
    nm.nm_decompress(vals, torch.from_numpy(m_ref).cuda(), C, out=out[:, :C])
    ref = oracle.decompress24(v_ref, m_ref, C, dtype=code)
    assert np.array_equal(_bits(out[:, :C]), np.ascontiguousarray(ref).view(_bits(out).dtype))
    assert torch.all(out[:, C:] == 3.0)


@pytest.mark.parametrize("R,C", SHAPES)
def test_meta_to_sm100(R, C):
    rng = np.random.default_rng(R * 7 + C)
    nib = rng.choice([0x4, 0x8, 0xC, 0x9, 0xD, 0xE], size=(R, C // 4)).astype(np.uint8)
    meta = (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)
    got = nm.nm_meta_to_sm100(torch.from_numpy(meta).cuda(), R, C).cpu().numpy()
    assert np.array_equal(got, oracle.meta_sm100(meta, R, C))


@pytest.mark.parametrize("N", [1, 2, 3])
def test_mask_24_large_bf16(N):
    """2^25 bf16 entries: the two-rows form of the M = 4 mask (smaller 16-bit
    weights take the four-rows form), whole matrix, byte for byte."""
    W = nm_inputs.normal((8192, 4096), 45, 0.02, torch.bfloat16)
    got = nm.nm_mask(W.cuda(), N, 4).cpu().numpy()
    assert np.array_equal(got, oracle.mask_rank(_bits(W), N, 4, dtype=oracle.BF16))


@pytest.mark.parametrize("R,C,dtype", [(8192, 4096, torch.bfloat16), (4096, 8192, torch.float32)])
def test_mask_compress_large_weights(R, C, dtype):
    """2^25 entries: the magnitude compressor's two-block form (smaller
    weights take the three-block form), whole matrix, bit-exact."""
    W = nm_inputs.normal((R, C), 44, 0.02, dtype)
    values, meta, img = nm.nm_mask_compress(W.cuda())
    _, v_ref, m_ref = oracle.rows_parallel(1, _bits(W), 2, 4, CODE[dtype], threads=os.cpu_count() or 2)
    assert np.array_equal(_bits(values), np.ascontiguousarray(v_ref).view(_bits(values).dtype))
    assert np.array_equal(meta.cpu().numpy(), m_ref)
    assert np.array_equal(img.cpu().numpy(), oracle.meta_sm100(m_ref, R, C))


@pytest.mark.parametrize("which", ["mlp_up", "mlp_down", "decode"])
def test_mask_compress_decompress_full_size(which):
    """The MLP pair's weights (14336 x 4096, 4096 x 14336) and the 28672 x 8192
    decode weight, whole matrices, bf16: the fused mask + compress matches the
    oracle byte for byte (values, metadata, image), and decompression returns
    W (.) mask with +0.0 at the pruned positions."""
    if which == "decode":
        W = nm_inputs.decode_skinny_W()
    else:
        W_up, W_down, _ = nm_inputs.mlp_pair()
        W = W_up if which == "mlp_up" else W_down
    R, C = W.shape
    values, meta, img = nm.nm_mask_compress(W.cuda())
    dense = nm.nm_decompress(values, meta, C)
    Wb = _bits(W)
    mask_ref, v_ref, m_ref = oracle.rows_parallel(1, Wb, 2, 4, oracle.BF16, threads=os.cpu_count() or 2)
    assert np.array_equal(_bits(values), v_ref)
    assert np.array_equal(meta.cpu().numpy(), m_ref)
    assert np.array_equal(img.cpu().numpy(), oracle.meta_sm100(m_ref, R, C))
    assert np.array_equal(_bits(dense), np.where(mask_ref == 1, Wb, np.uint16(0)))


def test_linear_4096_mask_compress_full_size():
    """The 4096 x 4096 bf16 transformer-linear weight, whole matrix, bit-exact."""
    W, _ = nm_inputs.linear_4096()
    values, meta, img = nm.nm_mask_compress(W.cuda())
    Wb = _bits(W)
    _, v_ref, m_ref = oracle.rows_parallel(1, Wb, 2, 4, oracle.BF16, threads=os.cpu_count() or 2)
    assert np.array_equal(_bits(values), v_ref)
    assert np.array_equal(meta.cpu().numpy(), m_ref)
    assert np.array_equal(img.cpu().numpy(), oracle.meta_sm100(m_ref, 4096, 4096))
