"""Pins for the oracle's SR-STE step (CPU only)."""
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _cases():
    out = []
    with open(os.path.join(GOLDEN, "srste_cases.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if not line:
                continue
            head, w, g, ws, go = line.split("|")
            N, M, decay = head.split()
            arr = lambda s: np.array([float(t) for t in s.split()], dtype=np.float32)
            out.append((int(N), int(M), float(decay), arr(w), arr(g), arr(ws), arr(go)))
    return out


@pytest.mark.parametrize("case", _cases(), ids=lambda c: str(c[3].tolist()))
def test_golden(case):
    N, M, decay, w, g, ws_exp, go_exp = case
    ws, go, mask = oracle.srste(w.reshape(1, -1), g.reshape(1, -1), N, M, decay)
    assert ws[0].view(np.uint32).tolist() == ws_exp.view(np.uint32).tolist()
    assert go[0].tolist() == go_exp.tolist()


@pytest.mark.parametrize("code", [oracle.F32, oracle.BF16, oracle.F16])
def test_exact_cases_reduce_to_plain_arithmetic(code):
    """Inputs with few significant bits and a power-of-two decay: g + decay * w is
    exact in float64, so one rounding of that exact value to the element type
    must equal the oracle's fused multiply-add path bit for bit."""
    rng = np.random.default_rng(3 + code)
    R, C = 24, 64
    w = rng.integers(-64, 65, (R, C)).astype(np.float64) / 8.0
    g = rng.integers(-64, 65, (R, C)).astype(np.float64) / 16.0
    decay = 2.0 ** -6
    wb = oracle.encode_array(w, code)
    gb = oracle.encode_array(g, code)
    ws, go, mask = oracle.srste(wb, gb, 2, 4, decay, dtype=code)
    width = np.uint32 if code == oracle.F32 else np.uint16
    exact = oracle.decode_array(gb, code) + np.where(mask.astype(bool), 0.0, decay * oracle.decode_array(wb, code))
    expect = oracle.encode_array(exact, code)
    assert np.array_equal(np.ascontiguousarray(go).view(width), expect)
    assert np.array_equal(mask, oracle.mask_rank(wb, 2, 4, dtype=code))
    assert np.array_equal(np.ascontiguousarray(ws).view(width), np.where(mask.astype(bool), wb, width(0)))


@pytest.mark.parametrize("N,M", [(2, 4), (1, 4), (4, 8), (2, 8)])
def test_page_default_decay_random(N, M):
    """decay = 0.0002 (the page's default) on random fp32 data: within half an
    ulp of binary32 of the float64 formula grad + decay * (1 - mask) * w."""
    rng = np.random.default_rng(N * 10 + M)
    R, C = 16, 8 * M
    w = rng.standard_normal((R, C)).astype(np.float32)
    g = (rng.standard_normal((R, C)) * 1e-3).astype(np.float32)
    ws, go, mask = oracle.srste(w, g, N, M, 0.0002)
    ref = g.astype(np.float64) + np.float64(np.float32(0.0002)) * (1 - mask) * w.astype(np.float64)
    ulp = np.spacing(np.abs(ref).astype(np.float32)).astype(np.float64)
    assert np.all(np.abs(go.astype(np.float64) - ref) <= 0.5 * ulp)
    assert np.all(mask.reshape(R, C // M, M).sum(axis=2) == N)
    kept = mask.astype(bool)
    assert np.array_equal(go[kept].view(np.uint32), g[kept].view(np.uint32))
    assert np.array_equal(ws[kept].view(np.uint32), w[kept].view(np.uint32))
    assert np.all(ws[~kept].view(np.uint32) == 0)


def test_zero_decay_leaves_gradient_values():
    rng = np.random.default_rng(9)
    w = rng.standard_normal((8, 32)).astype(np.float32)
    g = rng.standard_normal((8, 32)).astype(np.float32)
    _, go, _ = oracle.srste(w, g, 2, 4, 0.0)
    assert np.array_equal(go, g)
