"""Pins for the oracle's int8 2:4 product, its 1:2 (sparse TF32) product and
the two metadata images those tensor-core products read (CPU only).

Sources: review of "Accelerating Sparse Deep Neural Networks", "Structured
sparse GEMM on tensor cores" (sparse x dense = dense; the sparse tensor cores
take FP16/BF16/INT8 at 2:4 and TF32 only at 1:2); NVIDIA PTX ISA, tcgen05
sparse-matrix metadata (.kind::i8 and .kind::tf32)."""
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _int8(shape, seed, lo=-128, hi=128):
    return np.random.default_rng(seed).integers(lo, hi, shape).astype(np.int8)


def _compress_s8(W):
    mask = oracle.mask_rank(W, 2, 4)
    values, meta = oracle.compress24(W, mask)
    return mask, values, meta


# ---------------------------------------------------------------- int8 2:4 product
@pytest.mark.parametrize("R,K,T", [(8, 32, 5), (33, 96, 17), (64, 256, 40)])
def test_int8_product_equals_int64_matmul_of_the_masked_matrix(R, K, T):
    """Y equals an int64 numpy matmul of the decompressed (masked) weight with X,
    exactly, and also W * mask formed directly from the mask."""
    W = _int8((R, K), R + K)
    X = _int8((K, T), T + 7)
    mask, values, meta = _compress_s8(W)
    Y = oracle.spmm(values, meta, X, oracle.S8)
    dense = oracle.decompress24(values, meta, K).astype(np.int64)
    expect = dense @ X.astype(np.int64)
    assert np.array_equal(Y, expect.astype(np.float64))
    assert np.array_equal(np.where(mask == 1, W.astype(np.int64), 0) @ X.astype(np.int64), expect)


def test_int8_product_extremes_are_exact():
    """-128 everywhere: each group keeps two -128 entries, every product is
    2^14, and a row sums K/2 of them: 16384 * 4096 = 2^26 at K = 8192."""
    R, K, T = 4, 8192, 3
    W = np.full((R, K), -128, dtype=np.int8)
    X = np.full((K, T), -128, dtype=np.int8)
    _, values, meta = _compress_s8(W)
    Y = oracle.spmm(values, meta, X, oracle.S8)
    assert np.all(Y == 16384.0 * (K // 2))


def test_int8_one_hot_rows_select_rows_of_x():
    """Row r of W holds a single 1 at column c_r: Y's row r is X's row c_r."""
    R, K, T = 16, 64, 9
    cols = np.random.default_rng(3).integers(0, K, R)
    W = np.zeros((R, K), dtype=np.int8)
    W[np.arange(R), cols] = 1
    X = _int8((K, T), 4)
    _, values, meta = _compress_s8(W)
    Y = oracle.spmm(values, meta, X, oracle.S8)
    assert np.array_equal(Y, X[cols].astype(np.float64))


def test_int8_alpha_beta():
    R, K, T = 12, 64, 6
    W = _int8((R, K), 5)
    X = _int8((K, T), 6)
    Y0 = np.random.default_rng(7).standard_normal((R, T)).astype(np.float32)
    _, values, meta = _compress_s8(W)
    exact = oracle.spmm(values, meta, X, oracle.S8)
    Y = oracle.spmm(values, meta, X, oracle.S8, alpha=0.25, beta=-2.0, Y_in=Y0, y_dtype=oracle.F32)
    assert np.array_equal(Y, 0.25 * exact - 2.0 * Y0.astype(np.float64))


# ---------------------------------------------------------------- 1:2 product
def _compress12(W):
    mask = oracle.mask_rank(W, 1, 2)
    values, meta = oracle.compress12(W, mask)
    return mask, values, meta


@pytest.mark.parametrize("R,K,T", [(8, 16, 3), (33, 96, 17), (64, 256, 40)])
def test_12_product_on_integer_values_is_exact(R, K, T):
    """Small integers in fp32: every product and partial sum is exact in double,
    so Y equals the float64 matmul of the decompressed weight exactly."""
    rng = np.random.default_rng(R * K)
    W = rng.integers(-8, 9, (R, K)).astype(np.float32)
    X = rng.integers(-8, 9, (K, T)).astype(np.float32)
    mask, values, meta = _compress12(W)
    Y = oracle.spmm12(values, meta, X)
    dense = oracle.decompress12(values, meta, K).astype(np.float64)
    assert np.array_equal(Y, dense @ X.astype(np.float64))
    assert np.array_equal(Y, np.where(mask == 1, W, 0).astype(np.float64) @ X.astype(np.float64))


def test_12_product_random_matches_float64_matmul():
    rng = np.random.default_rng(11)
    R, K, T = 40, 128, 24
    W = rng.standard_normal((R, K)).astype(np.float32)
    X = rng.standard_normal((K, T)).astype(np.float32)
    _, values, meta = _compress12(W)
    Y = oracle.spmm12(values, meta, X)
    ref = oracle.decompress12(values, meta, K).astype(np.float64) @ X.astype(np.float64)
    assert np.max(np.abs(Y - ref)) <= 1e-12 * np.max(np.abs(ref))


def test_12_one_hot_rows_select_rows_of_x():
    R, K, T = 16, 64, 5
    cols = np.random.default_rng(12).integers(0, K, R)
    W = np.zeros((R, K), dtype=np.float32)
    W[np.arange(R), cols] = 1.0
    X = np.random.default_rng(13).standard_normal((K, T)).astype(np.float32)
    _, values, meta = _compress12(W)
    assert np.array_equal(oracle.spmm12(values, meta, X), X[cols].astype(np.float64))


# ---------------------------------------------------------------- .kind::i8 image
def _positions(name, fields):
    out = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                parts = line.split("|")
                out.append(tuple(int(x) for x in parts[0].split()) + tuple(int(x) for x in parts[1:]))
    assert all(len(o) == fields for o in out)
    return out


@pytest.mark.parametrize("pos", _positions("meta_image_i8_positions.txt", 3), ids=lambda p: "r%d_b%d" % p[:2])
def test_i8_image_hand_positions(pos):
    r, b, byte = pos
    R, C = 256, 512
    meta = np.full((R, C // 8), 0x44, dtype=np.uint8)
    meta[r, b] = 0xD9                                   # groups (1,2) and (1,3)
    img = oracle.meta_sm100_s8(meta, R, C)
    base = oracle.meta_sm100_s8(np.full((R, C // 8), 0x44, dtype=np.uint8), R, C)
    assert np.nonzero(img != base)[0].tolist() == [byte]
    assert img[byte] == 0xD9


@pytest.mark.parametrize("R,C", [(256, 512), (100, 384), (129, 24), (1, 8)])
def test_i8_image_is_the_canonical_metadata_retiled(R, C):
    """Read back by a numpy reshape: 128-row tiles, 16-byte (128-column) blocks,
    2 * ceil(C/256) blocks per row tile; every byte outside the matrix is 0x44."""
    meta = np.random.default_rng(R + C).integers(0, 256, (R, C // 8)).astype(np.uint8)
    img = oracle.meta_sm100_s8(meta, R, C)
    rt, nk = (R + 127) // 128, 2 * ((C + 255) // 256)
    assert img.size == rt * nk * 2048
    full = img.reshape(rt, nk, 128, 16).transpose(0, 2, 1, 3).reshape(rt * 128, nk * 16)
    assert np.array_equal(full[:R, :C // 8], meta)
    pad = np.ones(full.shape, dtype=bool)
    pad[:R, :C // 8] = False
    assert np.all(full[pad] == 0x44)


# ---------------------------------------------------------------- .kind::tf32 image
@pytest.mark.parametrize("pos", _positions("meta_image_tf32_positions.txt", 4), ids=lambda p: "r%d_p%d" % p[:2])
def test_tf32_image_hand_positions(pos):
    """Every pair keeps element 0 (field 0x4) except pair (r, p), which keeps
    element 1 (field 0xE)."""
    r, p, byte, shift = pos
    R, C = 256, 128
    meta = np.zeros((R, C // 16), dtype=np.uint8)
    meta[r, p // 8] |= np.uint8(1 << (p % 8))
    img = oracle.meta12_sm100(meta, R, C)
    base = oracle.meta12_sm100(np.zeros((R, C // 16), dtype=np.uint8), R, C)
    assert np.nonzero(img != base)[0].tolist() == [byte]
    assert (img[byte] >> shift) & 0xF == 0xE
    assert (base[byte] >> shift) & 0xF == 0x4


@pytest.mark.parametrize("R,C", [(256, 128), (100, 80), (129, 16)])
def test_tf32_image_is_the_f16_image_of_the_halves(R, C):
    """The 1:2 matrix seen as 16-bit halves is 2:4 with groups (0,1) or (2,3):
    expanding each index bit to that 2:4 pattern and building the .kind::f16
    image of the R x 2C matrix of halves gives the .kind::tf32 image."""
    meta = np.random.default_rng(R * C).integers(0, 256, (R, C // 16)).astype(np.uint8)
    bits = np.unpackbits(meta, axis=1, bitorder="little")[:, :C // 2]      # index of each pair
    nib = np.where(bits == 1, 0xE, 0x4).astype(np.uint8)                      # 2:4 field per half-group
    canon = (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)            # two groups per byte
    f16_img = oracle.meta_sm100(canon, R, 2 * C)
    img = oracle.meta12_sm100(meta, R, C)
    assert img.size == ((R + 127) // 128) * ((C + 63) // 64) * 2048
    assert f16_img.size == img.size
    assert np.array_equal(img, f16_img)
