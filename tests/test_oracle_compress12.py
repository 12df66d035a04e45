"""Pins of the oracle's 1:2 compression (sparse TF32's pattern: one value of
every pair kept; review of "Accelerating Sparse Deep Neural Networks",
"Structured sparse GEMM on tensor cores").  Independent checks:

* hand-derived rows (tests/golden/compress12_cases.txt), one of which runs
  the 1:2 magnitude mask first;
* decompress(compress(W, mask)) == select(mask, W, +0) bit for bit;
* an independent numpy restatement of the layout (kept element and index
  bit per pair);
* sizes: C/2 values and C/16 metadata bytes per row, so fp32 storage is
  33 bits per pair instead of 64;
* masks without exactly one 1 per pair are rejected."""
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "compress12_cases.txt")


def _cases():
    out = []
    with open(GOLDEN) as f:
        lines = f.read().splitlines()
    for line in lines:
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        w, m, v, meta = [p.split() for p in line.split("|")]
        out.append((np.array([[float(x) for x in w]], np.float32), np.array([[int(x) for x in m]], np.uint8),
                    np.array([[float(x) for x in v]], np.float32), int(meta[0], 16)))
    return out


@pytest.mark.parametrize("case", _cases())
def test_golden(case):
    W, mask, values, meta = case
    v, m = oracle.compress12(W, mask)
    assert np.array_equal(v.view(np.uint32), values.view(np.uint32))
    assert m.tolist() == [[meta]]


def test_golden_mask_case_is_the_magnitude_mask():
    W, mask, _, _ = _cases()[-1]
    assert np.array_equal(oracle.mask_rank(W, 1, 2), mask)


def _rand_mask(rng, R, C):
    first = rng.integers(0, 2, size=(R, C // 2)).astype(np.uint8)
    m = np.zeros((R, C), np.uint8)
    m[:, 0::2] = 1 - first
    m[:, 1::2] = first
    return m


@pytest.mark.parametrize("dtype", ["f32", "bf16", "f16"])
def test_round_trip_is_the_masked_weight(dtype):
    rng = np.random.default_rng(5)
    R, C = 24, 64
    if dtype == "f32":
        W, code = rng.standard_normal((R, C)).astype(np.float32), oracle.F32
        bits = W.view(np.uint32)
    else:
        W = rng.standard_normal((R, C)).astype(np.float16)
        code = oracle.F16 if dtype == "f16" else oracle.BF16
        bits = W.view(np.uint16)
    mask = _rand_mask(rng, R, C)
    v, m = oracle.compress12(bits, mask, dtype=code)
    back = oracle.decompress12(v, m, C, dtype=code)
    assert np.array_equal(back, np.where(mask == 1, bits, 0).astype(bits.dtype))
    assert v.shape == (R, C // 2) and m.shape == (R, C // 16)


def test_matches_an_independent_restatement():
    rng = np.random.default_rng(6)
    R, C = 10, 48
    W = rng.standard_normal((R, C)).astype(np.float32)
    mask = _rand_mask(rng, R, C)
    v, m = oracle.compress12(W, mask)
    idx = mask[:, 1::2]                                   # 1 where the second of the pair is kept
    exp_v = np.where(idx == 1, W[:, 1::2], W[:, 0::2])
    exp_m = np.packbits(idx, axis=1, bitorder="little")
    assert np.array_equal(v.view(np.uint32), exp_v.view(np.uint32))
    assert np.array_equal(m, exp_m)


def test_storage_is_33_bits_per_fp32_pair():
    R, C = 4, 32
    v, m = oracle.compress12(np.ones((R, C), np.float32), np.tile(np.array([1, 0], np.uint8), (R, C // 2)))
    assert (v.nbytes * 8 + m.nbytes * 8) / (R * C / 2) == 33.0


@pytest.mark.parametrize("bad", [[1, 1], [0, 0], [2, 0]])
def test_rejects_masks_without_one_per_pair(bad):
    mask = np.tile(np.array([1, 0], np.uint8), (1, 8))
    mask[0, 4:6] = bad
    with pytest.raises(Exception):
        oracle.compress12(np.ones((1, 16), np.float32), mask)
