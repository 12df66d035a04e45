"""Pins of the oracle's saliency-scored N:M mask ("sparsegpt.py", fasterprune,
semi-structured branch: the score w^2 / d^2 in binary32, the M-N smallest of
each group pruned).  Each check is independent of the oracle's C code:

* hand-derived groups (tests/golden/scored_cases.txt);
* d == 1 on bf16 weights: w*w is exact in binary32 and the quotient by 1 is
  exact, so the scores order exactly as |w| and the mask equals the
  magnitude mask;
* d a power of two per column: the score is (w / d)^2 exactly, so the mask
  equals the magnitude mask of the exactly rescaled weights;
* an independent numpy binary32 evaluation (elementwise IEEE products and
  quotient, stable per-group sort) on inputs with many exact ties."""
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "scored_cases.txt")


def _cases():
    out = []
    with open(GOLDEN) as f:
        lines = f.read().splitlines()
    for line in lines:
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        head, w, d, m = [p.split() for p in line.split("|")]
        out.append((int(head[0]), int(head[1]), [float(x) for x in w], [float(x) for x in d], [int(x) for x in m]))
    return out


@pytest.mark.parametrize("case", _cases())
def test_golden(case):
    N, M, w, d, expect = case
    W = np.array([w], dtype=np.float32)
    got = oracle.mask_scored(W, np.array(d, dtype=np.float32), N, M)
    assert got.tolist() == [expect]


NM = [(1, 2), (1, 4), (2, 4), (3, 4), (2, 8), (4, 8)]


def _bf16(x):
    """float32 array -> uint16 bf16 bit patterns (round to nearest even)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def _bf16_to_f32(b):
    return (b.astype(np.uint32) << 16).view(np.float32)


@pytest.mark.parametrize("N,M", NM)
def test_unit_d_is_the_magnitude_mask(N, M):
    rng = np.random.default_rng(7)
    W = _bf16(rng.integers(-6, 7, size=(64, 96)).astype(np.float32) * np.float32(0.375))
    got = oracle.mask_scored(W, np.ones(96, np.float32), N, M, dtype=oracle.BF16)
    assert np.array_equal(got, oracle.mask_rank(W, N, M, dtype=oracle.BF16))


@pytest.mark.parametrize("N,M", NM)
def test_power_of_two_d_rescales_exactly(N, M):
    rng = np.random.default_rng(8)
    W = _bf16(rng.standard_normal((48, 64)).astype(np.float32))
    k = rng.integers(-3, 4, size=64)
    d = np.ldexp(np.ones(64), k).astype(np.float32)
    got = oracle.mask_scored(W, d, N, M, dtype=oracle.BF16)
    scaled = (_bf16_to_f32(W) / d[None, :]).astype(np.float32)     # exact: division by a power of two
    assert np.array_equal(got, oracle.mask_rank(scaled, N, M))


def _numpy_scored(Wf32, d, N, M):
    """Independent evaluation: numpy binary32 elementwise IEEE arithmetic,
    keys = bit pattern with the sign cleared, a stable descending sort."""
    with np.errstate(divide="ignore", invalid="ignore"):
        s = (Wf32 * Wf32) / (d * d)[None, :]
    key = s.astype(np.float32).view(np.uint32) & np.uint32(0x7FFFFFFF)
    R, C = Wf32.shape
    g = key.reshape(R, C // M, M).astype(np.int64)
    order = np.argsort(-g, axis=2, kind="stable")        # equal keys keep index order
    mask = np.zeros_like(g, dtype=np.uint8)
    np.put_along_axis(mask, order[:, :, :N], 1, axis=2)
    return mask.reshape(R, C)


@pytest.mark.parametrize("N,M", NM)
def test_matches_an_independent_binary32_evaluation(N, M):
    rng = np.random.default_rng(9)
    R, C = 80, 64
    Wf = (rng.integers(-5, 6, size=(R, C)) * 0.3).astype(np.float32)     # repeated values: many ties
    d = rng.choice(np.array([0.5, 1.0, 1.5, 3.0, 0.1], np.float32), size=C)
    got = oracle.mask_scored(Wf, d, N, M)
    assert np.array_equal(got, _numpy_scored(Wf, d, N, M))
    # inexact quotients from generic values
    Wg = rng.standard_normal((R, C)).astype(np.float32)
    dg = rng.uniform(0.05, 2.0, size=C).astype(np.float32)
    assert np.array_equal(oracle.mask_scored(Wg, dg, N, M), _numpy_scored(Wg, dg, N, M))


def test_half_and_bfloat_inputs_are_scored_from_their_exact_values():
    rng = np.random.default_rng(10)
    R, C = 32, 32
    d = rng.uniform(0.1, 3.0, size=C).astype(np.float32)
    h = rng.standard_normal((R, C)).astype(np.float16)
    got_h = oracle.mask_scored(h.view(np.uint16), d, 2, 4, dtype=oracle.F16)
    assert np.array_equal(got_h, _numpy_scored(h.astype(np.float32), d, 2, 4))
    b = _bf16(rng.standard_normal((R, C)).astype(np.float32))
    got_b = oracle.mask_scored(b, d, 2, 4, dtype=oracle.BF16)
    assert np.array_equal(got_b, _numpy_scored(_bf16_to_f32(b), d, 2, 4))


def test_exactly_n_kept_per_group():
    rng = np.random.default_rng(11)
    W = rng.standard_normal((16, 48)).astype(np.float32)
    d = rng.uniform(0.0, 2.0, size=48).astype(np.float32)
    d[::5] = 0.0
    W[::3, ::7] = 0.0                                     # some 0/0 scores
    for N, M in NM:
        m = oracle.mask_scored(W, d, N, M)
        assert np.all(m.reshape(16, 48 // M, M).sum(axis=2) == N)
