"""Pins for the oracle's SR-STE step (CPU only).

The step follows "SR-STE sparse training", SR-STE forward / backward: the
forward returns output * w_b and the backward grad_output + decay * (1 - mask)
* weight.  The listing's mask comes from torch.ones with no dtype, so each
product and the sum are binary32 operations rounded on their own, and the
gradient is returned in the weight's dtype.  The golden cases are derived by
hand; a second test shows they separate this reading from a fused
multiply-add and from rounding every step to the 16-bit element type."""
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
CODES = {"f32": oracle.F32, "bf16": oracle.BF16, "f16": oracle.F16}
# (fraction bits, smallest normal exponent) of each element type
FMT = {"f32": (23, -126), "bf16": (7, -126), "f16": (10, -14)}


def _val(tok):
    return float.fromhex(tok) if "0x" in tok else float(tok)


def _cases():
    out = []
    with open(os.path.join(GOLDEN, "srste_cases.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if not line:
                continue
            head, w, g, ws, go = line.split("|")
            dt, N, M, decay = head.split()
            arr = lambda s: np.array([_val(t) for t in s.split()], dtype=np.float64)
            out.append((dt, int(N), int(M), float.fromhex(decay) if "0x" in decay else float(decay),
                        arr(w), arr(g), arr(ws), arr(go)))
    return out


def _width(code):
    return np.uint32 if code == oracle.F32 else np.uint16


@pytest.mark.parametrize("case", _cases(), ids=lambda c: "%s-%s" % (c[0], c[4].tolist()))
def test_golden(case):
    dt, N, M, decay, w, g, ws_exp, go_exp = case
    code = CODES[dt]
    wb = oracle.encode_array(w.reshape(1, -1), code)
    gb = oracle.encode_array(g.reshape(1, -1), code)
    assert np.array_equal(oracle.decode_array(wb, code)[0], w), "inputs must be exact in the dtype"
    ws, go, mask = oracle.srste(wb, gb, N, M, decay, dtype=code)
    width = _width(code)
    assert np.ascontiguousarray(ws).view(width)[0].tolist() == oracle.encode_array(ws_exp, code).tolist()
    assert np.ascontiguousarray(go).view(width)[0].tolist() == oracle.encode_array(go_exp, code).tolist()


def _round(x: Fraction, dt: str) -> Fraction:
    """x rounded to nearest even in the element type (no overflow in these cases)."""
    fbits, emin = FMT[dt]
    if x == 0:
        return x
    a = abs(x)
    e = math.floor(math.log2(a))
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    q = max(e, emin) - fbits
    sc = a / Fraction(2) ** q
    n = sc.numerator // sc.denominator
    rem = sc - n
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and n % 2):
        n += 1
    return (1 if x > 0 else -1) * n * Fraction(2) ** q


def test_golden_cases_separate_the_readings():
    """For every element type some golden line differs under a single fused
    multiply-add (the exact g + decay * w rounded once to binary32), and for the
    16-bit types some line differs when every step rounds to the element type;
    so a regression to either form fails test_golden."""
    fused_differs, elementwise_differs = set(), set()
    for dt, N, M, decay, w, g, _, go_exp in _cases():
        d = Fraction(decay)
        mags = np.abs(w)
        for i in range(M):
            beaten = sum(1 for j in range(M) if mags[j] > mags[i] or (mags[j] == mags[i] and j < i))
            c = Fraction(0) if beaten < N else d
            expect = Fraction(go_exp[i])
            fused = _round(_round(Fraction(g[i]) + c * Fraction(w[i]), "f32"), dt)
            if fused != expect:
                fused_differs.add(dt)
            if dt != "f32":
                per_op = _round(Fraction(g[i]) + _round(_round(c, dt) * Fraction(w[i]), dt), dt)
                if per_op != expect:
                    elementwise_differs.add(dt)
    assert fused_differs == {"f32", "bf16", "f16"}
    assert elementwise_differs == {"bf16", "f16"}


def _listing_in_torch(w_bits, g_bits, mask, decay, code):
    """The page's forward and backward arithmetic evaluated by PyTorch on the CPU,
    given the mask: a float32 mask (as torch.ones makes it), output * mask, and
    grad + decay * (1 - mask) * weight, returned in the weight's dtype."""
    tdt = {oracle.F32: torch.float32, oracle.BF16: torch.bfloat16, oracle.F16: torch.float16}[code]
    iv = torch.int32 if code == oracle.F32 else torch.int16
    w = torch.from_numpy(np.ascontiguousarray(w_bits).view(np.int32 if code == oracle.F32 else np.int16)).view(tdt)
    g = torch.from_numpy(np.ascontiguousarray(g_bits).view(np.int32 if code == oracle.F32 else np.int16)).view(tdt)
    m = torch.from_numpy(mask.astype(np.float32))
    fwd = (w.clone() * m).to(tdt)
    bwd = (g + decay * (1 - m) * w).to(tdt)
    width = _width(code)
    return fwd.view(iv).numpy().view(width), bwd.view(iv).numpy().view(width)


@pytest.mark.parametrize("code", [oracle.F32, oracle.BF16, oracle.F16])
@pytest.mark.parametrize("N,M", [(2, 4), (1, 4), (4, 8), (2, 8)])
def test_page_listing_arithmetic_random(code, N, M):
    """Random weights and 1e-3-scale gradients at the page's default decay:
    equal bit for bit to PyTorch evaluating the listing's expressions (given the
    oracle's mask), and the mask keeps exactly N of every M."""
    rng = np.random.default_rng(N * 10 + M + 100 * code)
    R, C = 16, 8 * M
    wb = oracle.encode_array(rng.standard_normal((R, C)), code)
    gb = oracle.encode_array(rng.standard_normal((R, C)) * 1e-3, code)
    ws, go, mask = oracle.srste(wb, gb, N, M, 0.0002, dtype=code)
    fwd, bwd = _listing_in_torch(wb, gb, mask, 0.0002, code)
    width = _width(code)
    assert np.array_equal(np.ascontiguousarray(ws).view(width), fwd)
    assert np.array_equal(np.ascontiguousarray(go).view(width), bwd)
    assert np.array_equal(mask, oracle.mask_rank(wb, N, M, dtype=code))
    assert np.all(mask.reshape(R, C // M, M).sum(axis=2) == N)


@pytest.mark.parametrize("code", [oracle.F32, oracle.BF16, oracle.F16])
def test_exact_cases_reduce_to_plain_arithmetic(code):
    """Inputs with few significant bits and a power-of-two decay: decay * w and
    g + decay * w are exact in binary32, so the result is the exact value
    rounded once to the element type, and the masked weight is w * mask."""
    rng = np.random.default_rng(3 + code)
    R, C = 24, 64
    w = rng.integers(-64, 65, (R, C)).astype(np.float64) / 8.0
    g = rng.integers(-64, 65, (R, C)).astype(np.float64) / 16.0
    decay = 2.0 ** -6
    wb = oracle.encode_array(w, code)
    gb = oracle.encode_array(g, code)
    ws, go, mask = oracle.srste(wb, gb, 2, 4, decay, dtype=code)
    width = _width(code)
    wd, gd = oracle.decode_array(wb, code), oracle.decode_array(gb, code)
    exact = gd + np.where(mask.astype(bool), 0.0, decay * wd)
    assert np.array_equal(np.ascontiguousarray(go).view(width), oracle.encode_array(exact, code))
    assert np.array_equal(mask, oracle.mask_rank(wb, 2, 4, dtype=code))
    assert np.array_equal(np.ascontiguousarray(ws).view(width), oracle.encode_array(wd * mask, code))


def test_zero_decay_leaves_gradient_values():
    rng = np.random.default_rng(9)
    w = rng.standard_normal((8, 32)).astype(np.float32)
    g = rng.standard_normal((8, 32)).astype(np.float32)
    _, go, _ = oracle.srste(w, g, 2, 4, 0.0)
    assert np.array_equal(go, g)
