"""Pins for the oracle's N:M mask selection (CPU only).

The oracle has two mask variants written independently: the rank rule (S)
and the exhaustive best-pattern search with exact sums (E).  Here both are
pinned to things outside the oracle:
  * hand-derived fixtures (tests/golden/mask_cases.txt, each with its source),
  * brute force over every 4-element group from a small alphabet, judged by a
    Python restatement of the pages' *definition* (max kept |w| sum, exact
    rational arithmetic, smallest index tuple on ties),
  * numpy's stable lexsort on (-|w|, index) (a library routine),
  * the invariant "exactly N ones per group".
"""
import itertools
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
import nm_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _parse_val(tok):
    tok = tok.strip()
    if tok.lstrip("-").startswith("0x"):
        return float.fromhex(tok)
    return float(tok)


def _golden_masks():
    out = []
    with open(os.path.join(GOLDEN, "mask_cases.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if not line:
                continue
            nm, vals, exp = line.split("|")
            N, M = map(int, nm.split())
            w = np.array([_parse_val(t) for t in vals.split()], dtype=np.float32)
            out.append((N, M, w, np.array([int(t) for t in exp.split()], dtype=np.uint8)))
    return out


@pytest.mark.parametrize("case", _golden_masks(), ids=lambda c: "%d:%d %s" % (c[0], c[1], c[2].tolist()))
def test_golden_masks(case):
    N, M, w, expected = case
    got = oracle.mask_rank(w.reshape(1, -1), N, M)[0]
    assert got.tolist() == expected.tolist()
    if np.all(np.isfinite(w)):
        assert oracle.mask_exhaustive(w.reshape(1, -1), N, M)[0].tolist() == expected.tolist()


def _mag_key(x: float) -> int:
    """IEEE binary32 bit pattern with the sign cleared, via numpy (not the oracle)."""
    return int(np.array([x], dtype=np.float32).view(np.uint32)[0] & 0x7FFFFFFF)


def _definition_mask(w, N):
    """The pages' exhaustive definition restated with exact rationals:
    among all N-subsets, maximise the kept sum of |w|; ties between subsets go
    to the lexicographically smallest ascending index tuple."""
    best, best_sum = None, None
    for combo in itertools.combinations(range(len(w)), N):
        s = sum(Fraction(abs(float(w[i]))) for i in combo)
        if best_sum is None or s > best_sum:
            best, best_sum = combo, s
    m = [0] * len(w)
    for i in best:
        m[i] = 1
    return m


def _lexsort_mask(W, N):
    """numpy stable lexsort: primary key -|w| (as bit magnitude), secondary index."""
    W32 = np.ascontiguousarray(W, dtype=np.float32)
    mags = (W32.view(np.uint32) & np.uint32(0x7FFFFFFF)).astype(np.int64)
    out = np.zeros(W.shape, dtype=np.uint8)
    idx = np.arange(W.shape[-1])
    for r in range(W.shape[0]):
        order = np.lexsort((idx, -mags[r]))
        out[r, order[:N]] = 1
    return out


ALPHABET = [-2.0, -1.0, -0.0, 0.0, 1.0, 2.0]


@pytest.mark.parametrize("N", [1, 2, 3])
def test_bruteforce_all_4_groups(N):
    groups = np.array(list(itertools.product(ALPHABET, repeat=4)), dtype=np.float32)  # 1296 x 4
    W = groups.reshape(-1, 4)
    S = oracle.mask_rank(W, N, 4)
    E = oracle.mask_exhaustive(W, N, 4)
    L = _lexsort_mask(W, N)
    for r in range(W.shape[0]):
        d = _definition_mask(W[r], N)
        assert S[r].tolist() == d, (W[r], S[r], d)
    assert np.array_equal(S, E)
    assert np.array_equal(S, L)
    assert np.all(S.sum(axis=1) == N)


NM_LIST = [(1, 2), (1, 4), (2, 4), (3, 4), (2, 8), (4, 8), (1, 8), (7, 8), (2, 3), (2, 5), (3, 6), (4, 7)]


@pytest.mark.parametrize("N,M", NM_LIST)
@pytest.mark.parametrize("code", [oracle.F32, oracle.BF16, oracle.F16])
def test_rank_equals_exhaustive_random(N, M, code):
    rng = np.random.default_rng(1000 * N + M + 7 * code)
    R, C = 37, M * 11
    if code == oracle.F32:
        W = rng.standard_normal((R, C)).astype(np.float32)
        W[rng.random((R, C)) < 0.2] = 0.0                     # plenty of exact ties
        W[rng.random((R, C)) < 0.1] *= np.float32(2.0 ** -140)  # subnormals
    elif code == oracle.F16:
        W = rng.integers(-4, 5, (R, C)).astype(np.float16)      # heavy ties
        W[rng.random((R, C)) < 0.1] = np.float16(2.0 ** -20)    # subnormal
    else:
        W = rng.integers(0, 0x7F80, (R, C)).astype(np.uint16)   # finite bf16 patterns
        W |= (rng.random((R, C)) < 0.5).astype(np.uint16) << 15
    S = oracle.mask_rank(W, N, M, dtype=code)
    E = oracle.mask_exhaustive(W, N, M, dtype=code)
    assert np.array_equal(S, E)
    assert np.all(S.reshape(R, C // M, M).sum(axis=2) == N)


@pytest.mark.parametrize("N,M", [(1, 4), (2, 4), (4, 8), (2, 8)])
def test_heavy_ties_workload_sample(N, M):
    """A 256-row sample of the fp32 k/100 heavy-ties workload: S == E == lexsort."""
    W = nm_inputs.ties((256, 1024), nm_inputs.SEEDS["ties_fp32.W"]).numpy()
    S = oracle.mask_rank(W, N, M)
    E = oracle.mask_exhaustive(W, N, M)
    assert np.array_equal(S, E)
    L = _lexsort_mask(W.reshape(-1, M), N).reshape(W.shape)
    assert np.array_equal(S, L)


def test_fp_sum_trap():
    """With fp64 sums, {0,1}, {0,2} and {0,3} all score 1.0 and a first-best
    search keeps index 1; exact sums keep the larger 2^-80 at index 2."""
    w = np.array([[1.0, 0.0, 2.0 ** -80, 2.0 ** -90]], dtype=np.float32)
    fp64_sums = [sum(float(abs(w[0, i])) for i in c) for c in itertools.combinations(range(4), 2)]
    assert fp64_sums[0] == fp64_sums[1] == fp64_sums[2] == 1.0     # the trap is real
    assert oracle.mask_exhaustive(w, 2, 4)[0].tolist() == [1, 0, 1, 0]
    assert oracle.mask_rank(w, 2, 4)[0].tolist() == [1, 0, 1, 0]


def test_magnitude_key_matches_numpy():
    rng = np.random.default_rng(3)
    bits = rng.integers(0, 2 ** 32, 2000, dtype=np.uint64).astype(np.uint32)
    for b in bits[:500]:
        assert oracle._load().oracle_mag(int(b), oracle.F32) == _mag_key(np.uint32(b).view(np.float32))


def test_nonfinite_rejected_by_exhaustive_only():
    w = np.array([[np.inf, 1, 2, 3]], dtype=np.float32)
    with pytest.raises(ValueError):
        oracle.mask_exhaustive(w, 2, 4)
    assert oracle.mask_rank(w, 2, 4)[0].tolist() == [1, 0, 0, 1]


@pytest.mark.parametrize("N,M,C", [(2, 4, 6), (0, 4, 8), (4, 4, 8), (2, 9, 18)])
def test_bad_arguments(N, M, C):
    with pytest.raises(ValueError):
        oracle.mask_rank(np.zeros((2, C), dtype=np.float32), N, M)
