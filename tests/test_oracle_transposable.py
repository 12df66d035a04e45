"""Pins of the oracle's greedy transposable N:M mask (nubint.ai review of the
N:M transposable-masks paper: in every M x M block keep the largest L1 norm
with at most N kept entries per row and per column; a greedy
2-approximation).  Independent checks:

* hand-derived blocks (tests/golden/transposable_cases.txt);
* the 2-approximation bound against the exact optimum, found by exhaustive
  search over every admissible mask of small blocks, and for N = 1 also by
  scipy's assignment solver;
* the set the greedy returns has no blocking entry: no left-out entry is
  preferred (larger |w|, then lower row-major position) by both its row and
  its column over what they kept.  This characterises the greedy result
  without running the greedy;
* transposing W transposes the mask (distinct magnitudes);
* at most N kept per row and per column of every block."""
import itertools
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "transposable_cases.txt")


def _cases():
    out = []
    with open(GOLDEN) as f:
        lines = f.read().splitlines()
    for line in lines:
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        head, w, m = [p.split() for p in line.split("|")]
        N, M = int(head[0]), int(head[1])
        out.append((N, M, np.array([float(x) for x in w], np.float32).reshape(M, M),
                    np.array([int(x) for x in m], np.uint8).reshape(M, M)))
    return out


@pytest.mark.parametrize("case", _cases())
def test_golden(case):
    N, M, W, expect = case
    assert np.array_equal(oracle.mask_transposable(W, N, M), expect)


def _blocks(mask, M):
    R, C = mask.shape
    return mask.reshape(R // M, M, C // M, M).transpose(0, 2, 1, 3)


def _admissible(M, N):
    """Every M x M 0/1 mask with at most N ones per row and per column (M <= 4)."""
    bits = np.array(list(itertools.product([0, 1], repeat=M * M)), dtype=np.uint8).reshape(-1, M, M)
    ok = (bits.sum(axis=2) <= N).all(axis=1) & (bits.sum(axis=1) <= N).all(axis=1)
    return bits[ok]


@pytest.mark.parametrize("N,M", [(1, 2), (1, 3), (2, 3), (1, 4), (2, 4), (3, 4)])
def test_within_half_of_the_exhaustive_optimum(N, M):
    rng = np.random.default_rng(20 + 10 * N + M)
    masks = _admissible(M, N)
    for _ in range(150):
        W = rng.standard_normal((M, M)).astype(np.float32)
        A = np.abs(W).astype(np.float64)
        opt = (masks * A).sum(axis=(1, 2)).max()
        got = (oracle.mask_transposable(W, N, M) * A).sum()
        assert got <= opt * (1 + 1e-12)
        assert got >= 0.5 * opt * (1 - 1e-12)


def test_n1_against_the_assignment_solver():
    from scipy.optimize import linear_sum_assignment
    rng = np.random.default_rng(31)
    for M in (2, 3, 5, 8):
        for _ in range(50):
            W = rng.standard_normal((M, M)).astype(np.float32)
            A = np.abs(W).astype(np.float64)
            r, c = linear_sum_assignment(-A)
            opt = A[r, c].sum()
            got = (oracle.mask_transposable(W, 1, M) * A).sum()
            assert 0.5 * opt * (1 - 1e-12) <= got <= opt * (1 + 1e-12)


def _no_blocking_entry(W, mask, N, M):
    """Check: no entry outside the mask is ranked above N kept entries in both
    its row and its column (rank: larger magnitude key, then lower row-major
    position within the block)."""
    key = W.astype(np.float32).view(np.uint32) & np.uint32(0x7FFFFFFF)
    for bi in range(W.shape[0] // M):
        for bj in range(W.shape[1] // M):
            k = key[bi * M:(bi + 1) * M, bj * M:(bj + 1) * M].astype(np.int64)
            m = mask[bi * M:(bi + 1) * M, bj * M:(bj + 1) * M]
            rank = {}
            order = sorted(((-int(k[i, j]), i * M + j) for i in range(M) for j in range(M)))
            for pos_in_order, (_, p) in enumerate(order):
                rank[p] = pos_in_order
            for i in range(M):
                for j in range(M):
                    if m[i, j]:
                        continue
                    above_row = sum(1 for jj in range(M) if m[i, jj] and rank[i * M + jj] < rank[i * M + j])
                    above_col = sum(1 for ii in range(M) if m[ii, j] and rank[ii * M + j] < rank[i * M + j])
                    assert above_row >= N or above_col >= N, (bi, bj, i, j)
            assert (m.sum(axis=1) <= N).all() and (m.sum(axis=0) <= N).all()


@pytest.mark.parametrize("N,M", [(1, 2), (2, 4), (1, 4), (3, 4), (4, 8), (2, 8), (3, 6)])
def test_no_blocking_entry(N, M):
    rng = np.random.default_rng(40 + N + M)
    W = (rng.integers(-6, 7, size=(4 * M, 3 * M)) * 0.25).astype(np.float32)   # many ties
    _no_blocking_entry(W, oracle.mask_transposable(W, N, M), N, M)
    W2 = rng.standard_normal((2 * M, 2 * M)).astype(np.float32)
    _no_blocking_entry(W2, oracle.mask_transposable(W2, N, M), N, M)


@pytest.mark.parametrize("N,M", [(2, 4), (4, 8), (1, 8), (5, 8)])
def test_transpose_gives_the_transposed_mask(N, M):
    rng = np.random.default_rng(50 + N)
    W = rng.standard_normal((3 * M, 5 * M)).astype(np.float32)          # distinct magnitudes
    a = oracle.mask_transposable(W, N, M)
    b = oracle.mask_transposable(np.ascontiguousarray(W.T), N, M)
    assert np.array_equal(a.T, b)


def test_bf16_and_f16_rank_by_their_own_bits():
    rng = np.random.default_rng(60)
    h = rng.standard_normal((16, 16)).astype(np.float16)
    got = oracle.mask_transposable(h.view(np.uint16), 4, 8, dtype=oracle.F16)
    ref = oracle.mask_transposable(h.astype(np.float32), 4, 8)          # exact widening keeps the order
    assert np.array_equal(got, ref)


def test_rejects_bad_shapes():
    with pytest.raises(Exception):
        oracle.mask_transposable(np.zeros((6, 8), np.float32), 4, 8)     # R not a multiple of M
