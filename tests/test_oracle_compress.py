"""Pins for the oracle's 2:4 compression, decompression and the tensor-core
metadata permutation (CPU only)."""
import os

import numpy as np
import pytest

import oracle
import nm_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
VALID_NIBBLES = {0x4, 0x8, 0xC, 0x9, 0xD, 0xE}   # (i0,i1) with i0 < i1, i0 | i1 << 2


def _val(tok):
    tok = tok.strip()
    return float.fromhex(tok) if tok.lstrip("-").startswith("0x") else float(tok)


def _golden_compress():
    rows = []
    with open(os.path.join(GOLDEN, "compress_cases.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if not line:
                continue
            w, m, v, meta = line.split("|")
            rows.append((np.array([_val(t) for t in w.split()], dtype=np.float32),
                         np.array([int(t) for t in m.split()], dtype=np.uint8),
                         np.array([_val(t) for t in v.split()], dtype=np.float32),
                         int(meta.strip(), 16)))
    return rows


@pytest.mark.parametrize("case", _golden_compress(), ids=lambda c: str(c[0].tolist()))
def test_golden_compress(case):
    w, m, v, meta = case
    values, metab = oracle.compress24(w.reshape(1, 8), m.reshape(1, 8))
    assert values.view(np.uint32).tolist() == [v.view(np.uint32).tolist()]   # bit-exact, -0 kept
    assert metab.tolist() == [[meta]]
    back = oracle.decompress24(values, metab, 8)
    expect = np.where(m.astype(bool), w, np.float32(0.0)).astype(np.float32)
    assert back.view(np.uint32).tolist() == [expect.view(np.uint32).tolist()]


def _random_case(code, R, C, seed):
    rng = np.random.default_rng(seed)
    if code == oracle.F32:
        W = rng.standard_normal((R, C)).astype(np.float32)
        W[rng.random((R, C)) < 0.15] = -0.0
    elif code == oracle.F16:
        W = rng.standard_normal((R, C)).astype(np.float16)
        W[rng.random((R, C)) < 0.15] = np.float16(-0.0)
    else:
        W = rng.integers(0, 0x10000, (R, C)).astype(np.uint16)
        W[(W & 0x7F80) == 0x7F80] = 0x8000                     # keep it finite; -0 patterns
    return W


@pytest.mark.parametrize("code", [oracle.F32, oracle.BF16, oracle.F16])
def test_roundtrip_and_invariants(code):
    R, C = 19, 64
    W = _random_case(code, R, C, 11 + code)
    mask = oracle.mask_rank(W, 2, 4, dtype=code)
    values, meta = oracle.compress24(W, mask, dtype=code)
    # sizes: R*C/2 values, R*C/2 2-bit fields = R*C/8 bytes
    assert values.shape == (R, C // 2) and meta.shape == (R, C // 8)
    # decompress(compress(W)) == select(mask, W, +0) bit for bit
    back = oracle.decompress24(values, meta, C, dtype=code)
    width = np.uint32 if code == oracle.F32 else np.uint16
    Wb = np.ascontiguousarray(W).view(width)
    expect = np.where(mask.astype(bool), Wb, width(0))
    assert np.array_equal(np.ascontiguousarray(back).view(width), expect)
    # every group's nibble is a valid ascending pair and matches the mask
    nib = np.stack([(meta >> 0) & 0xF, (meta >> 4) & 0xF], axis=-1).reshape(R, C // 4)
    assert set(np.unique(nib).tolist()) <= VALID_NIBBLES
    for r in range(R):
        for g in range(C // 4):
            i0, i1 = nib[r, g] & 3, nib[r, g] >> 2
            assert mask[r, 4 * g:4 * g + 4].tolist() == [int(i in (i0, i1)) for i in range(4)]


def test_all_zero_group_stores_two_values():
    """A group with more than two zeros still stores two values (pattern (0,1))."""
    W = np.zeros((1, 8), dtype=np.float32)
    W[0, 6] = 5.0
    mask = oracle.mask_rank(W, 2, 4)
    values, meta = oracle.compress24(W, mask)
    assert values.tolist() == [[0.0, 0.0, 0.0, 5.0]]   # group 1 keeps (0, 2): a zero and the 5
    assert meta[0, 0] & 0xF == 0x4                  # group 0 -> indices (0, 1)
    assert (meta[0, 0] >> 4) == (0 | (2 << 2))      # group 1 -> (0, 2)


def test_storage_saving_36_of_64_bits():
    """36 bits instead of 64 per four 16-bit weights: the pages' 44% saving."""
    R, C = 8, 64
    W = _random_case(oracle.BF16, R, C, 5)
    values, meta = oracle.compress24(W, oracle.mask_rank(W, 2, 4, dtype=oracle.BF16), dtype=oracle.BF16)
    bits_compressed = values.nbytes * 8 + meta.nbytes * 8
    bits_dense = R * C * 16
    assert bits_compressed * 64 == bits_dense * 36
    assert abs(1 - bits_compressed / bits_dense - 0.4375) < 1e-12


@pytest.mark.parametrize("bad", [[1, 1, 1, 0], [1, 1, 1, 1], [2, 1, 0, 0], [0, 0, 3, 0]])
def test_invalid_mask_rejected(bad):
    """More than two kept, or a mask byte other than 0/1, is not a 2:4 mask."""
    W = np.ones((1, 8), dtype=np.float32)
    m = np.array([bad + [1, 1, 0, 0]], dtype=np.uint8)
    with pytest.raises(ValueError):
        oracle.compress24(W, m)


# A group that keeps fewer than two ("Benefits of 2:4 sparsity": a group with
# more zeros still stores two values) is stored as the kept positions plus the
# lowest unkept ones, ascending, the unkept ones with value +0.0.  Worked by
# hand: (mask of the group) -> (pair, stored values, nibble idx0 | idx1 << 2).
SPARSE_GROUPS = [
    ([0, 0, 1, 0], (0, 2), (0.0, 3.0), 0x8),
    ([1, 0, 0, 0], (0, 1), (1.5, 0.0), 0x4),
    ([0, 1, 0, 0], (0, 1), (0.0, -2.0), 0x4),
    ([0, 0, 0, 1], (0, 3), (0.0, 4.0), 0xC),
    ([0, 0, 0, 0], (0, 1), (0.0, 0.0), 0x4),
    ([0, 0, 1, 1], (2, 3), (3.0, 4.0), 0xE),
]


@pytest.mark.parametrize("group,pair,vals,nib", SPARSE_GROUPS)
def test_groups_with_fewer_than_two_kept(group, pair, vals, nib):
    W = np.array([[1.5, -2.0, 3.0, 4.0, -1.0, -1.0, 5.0, 6.0]], dtype=np.float32)
    m = np.array([group + [0, 1, 0, 0]], dtype=np.uint8)      # second group: keeps index 1 only
    values, meta = oracle.compress24(W, m)
    assert values[0, :2].tolist() == list(vals)
    assert (meta[0, 0] & 0xF) == nib
    # the second group [-1, -1, 5, 6] keeping index 1: pair (0, 1), values (+0.0, -1.0)
    assert values[0, 2:].tolist() == [0.0, -1.0] and (meta[0, 0] >> 4) == 0x4
    # stored fillers are +0.0, not -0.0, even where W is negative
    assert values.view(np.uint32)[0, 2] == 0


@pytest.mark.parametrize("code", [oracle.F32, oracle.BF16, oracle.F16])
def test_sparser_masks_roundtrip_to_select(code):
    """decompress(compress(W, mask)) == select(mask, W, +0.0) for any mask with
    at most two ones per group: 1:4 magnitude masks and random ones."""
    R, C = 16, 64
    W = _random_case(code, R, C, 17)
    rng = np.random.default_rng(3)
    masks = [oracle.mask_rank(W, 1, 4, dtype=code)]
    rand = np.zeros((R, C), dtype=np.uint8)
    for r in range(R):
        for g in range(C // 4):
            k = rng.integers(0, 3)
            rand[r, 4 * g + rng.choice(4, size=k, replace=False)] = 1
    masks.append(rand)
    for mask in masks:
        values, meta = oracle.compress24(W, mask, dtype=code)
        back = oracle.decompress24(values, meta, C, dtype=code)
        assert np.array_equal(back, np.where(mask == 1, W, np.zeros_like(W)))


# ---------------------------------------------------------------- metadata image
def _positions():
    out = []
    with open(os.path.join(GOLDEN, "meta_sm100_positions.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                a, b, c = line.split("|")
                r, g = map(int, a.split())
                out.append((r, g, int(b), int(c)))
    return out


@pytest.mark.parametrize("pos", _positions(), ids=lambda p: "r%d_g%d" % (p[0], p[1]))
def test_meta_sm100_hand_positions(pos):
    r, g, byte, shift = pos
    R = C = 256
    # every group (0,1) = nibble 0x4, except group (r, g) which gets (1,3) = 0xD
    meta = np.full((R, C // 8), 0x44, dtype=np.uint8)
    k0 = 2 * g                                  # kept entries 2g, 2g+1 -> same byte, nibble g%2
    meta[r, k0 // 4] &= ~np.uint8(0xF << (4 * (g % 2))) & 0xFF
    meta[r, k0 // 4] |= np.uint8(0xD << (4 * (g % 2)))
    img = oracle.meta_sm100(meta, R, C)
    base = oracle.meta_sm100(np.full((R, C // 8), 0x44, dtype=np.uint8), R, C)
    diff = np.nonzero(img != base)[0]
    assert diff.tolist() == [byte]
    assert (img[byte] >> shift) & 0xF == 0xD
    assert (base[byte] >> shift) & 0xF == 0x4


@pytest.mark.parametrize("R,C", [(128, 128), (256, 384), (200, 72), (1, 8), (129, 136)])
def test_meta_sm100_is_a_permutation(R, C):
    """Every group nibble lands in its own 4-bit slot; padding slots carry 0x4."""
    rng = np.random.default_rng(R * 1000 + C)
    nib = rng.choice(sorted(VALID_NIBBLES), size=(R, C // 4)).astype(np.uint8)
    meta = (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)
    img = oracle.meta_sm100(meta, R, C)
    Rp, Cp = -(-R // 128) * 128, -(-C // 128) * 128
    assert img.size == Rp * Cp // 8 == oracle.meta_sm100_bytes(R, C)
    # tag each group with a distinct count: the multiset of slot values equals the input's
    slots = np.stack([img & 0xF, img >> 4], axis=-1).ravel()
    n_pad = Rp * Cp // 4 - R * C // 4
    vals, counts = np.unique(slots, return_counts=True)
    expect = dict(zip(*np.unique(nib, return_counts=True)))
    expect[0x4] = expect.get(0x4, 0) + n_pad
    assert dict(zip(vals.tolist(), counts.tolist())) == {int(k): int(v) for k, v in expect.items()}
    # one-hot probe: moving a single group's nibble changes exactly one slot
    for (r, g) in [(0, 0), (R - 1, C // 4 - 1), (R // 2, C // 8)]:
        m2 = np.full_like(meta, 0x44)
        m2[r, g // 2] = np.uint8((0xE << (4 * (g % 2))) | (0x4 << (4 * (1 - g % 2))))
        a = oracle.meta_sm100(m2, R, C)
        b = oracle.meta_sm100(np.full_like(meta, 0x44), R, C)
        assert np.count_nonzero(a != b) == 1
