"""Pins of the oracle on int8 weights (two's complement; magnitude |x|, so
-128 outranks 127).  The pages' INT8 2:4 path (TensorRT with sparse INT8) is
the reason for this element type; the selection and compression rules are
the ones of the floating-point types.  Independent checks:

* hand-derived groups, including -128 against a 127 / -127 tie;
* the exhaustive pattern search with exact sums (a different algorithm)
  selects the same entries as the rank rule;
* numpy's stable sort by (-|x|, index), taking the first N of each group;
* compress / decompress round trip and byte counts (1 byte per kept value)."""
import numpy as np
import pytest

import oracle

CASES = [
    # (N, M, group, expected mask)
    (2, 4, [-128, 127, -127, 1], [1, 1, 0, 0]),   # |-128| = 128 wins; 127 / -127 tie -> the first
    (1, 4, [-3, 3, 2, -3], [1, 0, 0, 0]),
    (3, 4, [0, 0, 0, 0], [1, 1, 1, 0]),
    (2, 4, [0, -1, 0, 1], [0, 1, 0, 1]),
    (2, 8, [1, 2, 3, 4, -4, -3, -2, -1], [0, 0, 0, 1, 1, 0, 0, 0]),
    (1, 2, [-128, 127], [1, 0]),
]


@pytest.mark.parametrize("case", CASES)
def test_hand_derived(case):
    N, M, g, expect = case
    W = np.array([g], dtype=np.int8)
    assert oracle.mask_rank(W, N, M).tolist() == [expect]


def _numpy_mask(W, N, M):
    R, C = W.shape
    mag = np.abs(W.astype(np.int16)).reshape(R, C // M, M)
    order = np.argsort(-mag, axis=2, kind="stable")      # larger |x| first, equal |x| in index order
    mask = np.zeros_like(mag, dtype=np.uint8)
    np.put_along_axis(mask, order[:, :, :N], 1, axis=2)
    return mask.reshape(R, C)


@pytest.mark.parametrize("N,M", [(1, 2), (1, 4), (2, 4), (3, 4), (2, 8), (4, 8), (3, 6)])
def test_rank_rule_matches_a_stable_sort_and_the_exhaustive_search(N, M):
    rng = np.random.default_rng(40 + N * M)
    C = 48
    W = rng.integers(-128, 128, size=(64, C)).astype(np.int8)
    W[::5, ::3] = -128
    W[::7, 1::4] = 127
    W[::3, 2::5] = 0
    m = oracle.mask_rank(W, N, M)
    assert np.array_equal(m, _numpy_mask(W, N, M))
    assert np.array_equal(m, oracle.mask_exhaustive(W, N, M))


def test_compress_round_trip_and_sizes():
    rng = np.random.default_rng(41)
    W = rng.integers(-128, 128, size=(32, 64)).astype(np.int8)
    mask = oracle.mask_rank(W, 2, 4)
    v, meta = oracle.compress24(W, mask)
    assert v.dtype == np.int8 and v.shape == (32, 32) and meta.shape == (32, 8)
    back = oracle.decompress24(v, meta, 64)
    assert np.array_equal(back.view(np.int8), np.where(mask == 1, W, 0).astype(np.int8))
    # 2:4 int8 storage: 8 bits per kept value + 2 bits of metadata -> 20 bits per 4 weights, not 32
    assert (v.nbytes + meta.nbytes) * 8 / (W.size / 4) == 20.0
