"""Pins for the oracle's fp64 sparse x dense product and its number formats
(CPU only).  The references here are library routines (numpy / torch
conversions and matmul) and closed forms, never the oracle itself."""
import numpy as np
import pytest
import torch

import oracle
import nm_inputs


# ------------------------------------------------------------------ formats
def test_f16_decode_all_patterns_vs_numpy():
    bits = np.arange(65536, dtype=np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = oracle.decode_array(bits, oracle.F16)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(ref[~nan]))


def test_bf16_decode_all_patterns_vs_torch():
    bits = np.arange(65536, dtype=np.uint16)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    got = oracle.decode_array(bits, oracle.BF16)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


def test_f32_decode_sample_vs_numpy():
    rng = np.random.default_rng(0)
    bits = rng.integers(0, 2 ** 32, 3000, dtype=np.uint64).astype(np.uint32)
    bits[:6] = [0, 0x80000000, 1, 0x007FFFFF, 0x7F7FFFFF, 0x7F800000]
    with np.errstate(invalid="ignore"):   # the sample holds NaN patterns on purpose
        ref = bits.view(np.float32).astype(np.float64)
    got = np.array([oracle.decode(int(b), oracle.F32) for b in bits])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan) and np.array_equal(got[~nan], ref[~nan])


def _rne_samples():
    rng = np.random.default_rng(1)
    x = np.concatenate([
        rng.standard_normal(3000) * np.exp2(rng.integers(-30, 30, 3000)),
        np.exp2(rng.uniform(-160, 140, 2000)) * rng.choice([-1, 1], 2000),
        [0.0, -0.0, 65504.0, 65519.99, 65520.0, 1e9, 2.0 ** -24, 2.0 ** -25, 3 * 2.0 ** -26,
         1 + 2.0 ** -11, 1 + 3 * 2.0 ** -11, 1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8],
    ])
    return x


def test_f16_encode_rne_vs_numpy():
    x = _rne_samples()
    with np.errstate(over="ignore"):     # values past the binary16 range round to infinity
        ref = x.astype(np.float16).view(np.uint16)
    got = oracle.encode_array(x, oracle.F16)
    assert np.array_equal(got, ref)


def test_bf16_encode_rne_vs_torch():
    # torch rounds fp32 -> bf16 to nearest-even; feed values exact in fp32
    with np.errstate(over="ignore"):     # values past the binary32 range become infinities, dropped next
        x = _rne_samples().astype(np.float32).astype(np.float64)
    x = x[np.isfinite(x)]
    ref = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = oracle.encode_array(x, oracle.BF16)
    assert np.array_equal(got, ref)


def test_f32_encode_rne_vs_numpy():
    x = _rne_samples()
    with np.errstate(over="ignore"):
        ref = x.astype(np.float32).view(np.uint32)
    got = oracle.encode_array(x, oracle.F32)
    assert np.array_equal(got, ref)


# ------------------------------------------------------------------ spmm
def _compressed(W, code):
    mask = oracle.mask_rank(W, 2, 4, dtype=code)
    values, meta = oracle.compress24(W, mask, dtype=code)
    return mask, values, meta


def _dense_masked_f64(W, mask, code):
    width = np.uint32 if code == oracle.F32 else np.uint16
    Wf = oracle.decode_array(np.ascontiguousarray(W).view(width), code)
    return np.where(mask.astype(bool), Wf, 0.0)


def test_integer_valued_is_exact():
    """Small integers: every partial sum is an exact integer, so the fp64
    product equals an int64 matmul of the masked dense matrix exactly."""
    R, K, T = 40, 96, 24
    W = nm_inputs.small_int((R, K), 7, dtype=torch.bfloat16)
    X = nm_inputs.small_int((K, T), 8, dtype=torch.bfloat16)
    Wb, Xb = nm_inputs.bits_u16(W), nm_inputs.bits_u16(X)
    mask, values, meta = _compressed(Wb, oracle.BF16)
    Y = oracle.spmm(values, meta, Xb, oracle.BF16, threads=2)
    Wi = (W.to(torch.int64).numpy()) * mask
    Yi = Wi @ X.to(torch.int64).numpy()
    assert np.array_equal(Y, Yi.astype(np.float64))


@pytest.mark.parametrize("code", [oracle.F32, oracle.BF16, oracle.F16])
def test_matches_numpy_matmul(code):
    R, K, T = 33, 128, 17
    rng = np.random.default_rng(5 + code)
    if code == oracle.F32:
        W = rng.standard_normal((R, K)).astype(np.float32)
        X = rng.standard_normal((K, T)).astype(np.float32)
        Xb = X
    elif code == oracle.F16:
        W = rng.standard_normal((R, K)).astype(np.float16)
        X = rng.standard_normal((K, T)).astype(np.float16)
        Xb = X
    else:
        W = nm_inputs.bits_u16(torch.from_numpy(rng.standard_normal((R, K)).astype(np.float32)).to(torch.bfloat16))
        Xb = nm_inputs.bits_u16(torch.from_numpy(rng.standard_normal((K, T)).astype(np.float32)).to(torch.bfloat16))
    mask, values, meta = _compressed(W, code)
    width = np.uint32 if code == oracle.F32 else np.uint16
    Xf = oracle.decode_array(np.ascontiguousarray(Xb).view(width), code)
    ref = _dense_masked_f64(W, mask, code) @ Xf
    Y = oracle.spmm(values, meta, Xb, code, threads=3)
    assert np.allclose(Y, ref, rtol=1e-13, atol=1e-13)


def test_one_hot_rows_select_x_rows():
    """W with one +1 per row at column c_r: row r of Y is exactly row c_r of X."""
    R, K, T = 16, 64, 9
    rng = np.random.default_rng(9)
    W = np.zeros((R, K), dtype=np.float16)
    cols = rng.integers(0, K, R)
    W[np.arange(R), cols] = 1.0
    X = rng.standard_normal((K, T)).astype(np.float16)
    mask, values, meta = _compressed(W, oracle.F16)
    Y = oracle.spmm(values, meta, X, oracle.F16)
    assert np.array_equal(Y, X[cols].astype(np.float64))


def test_alpha_beta_and_beta_zero_never_reads_y():
    R, K, T = 12, 32, 8
    rng = np.random.default_rng(2)
    W = rng.standard_normal((R, K)).astype(np.float32)
    X = rng.standard_normal((K, T)).astype(np.float32)
    Yin = rng.standard_normal((R, T)).astype(np.float32)
    mask, values, meta = _compressed(W, oracle.F32)
    base = oracle.spmm(values, meta, X, oracle.F32)
    ab = oracle.spmm(values, meta, X, oracle.F32, alpha=2.0, beta=0.5, Y_in=Yin, y_dtype=oracle.F32)
    assert np.allclose(ab, 2.0 * base + 0.5 * Yin.astype(np.float64), rtol=1e-14, atol=1e-14)
    nan_y = np.full((R, T), np.nan, dtype=np.float32)
    z = oracle.spmm(values, meta, X, oracle.F32, alpha=1.0, beta=0.0, Y_in=nan_y, y_dtype=oracle.F32)
    assert np.array_equal(z, base)


def test_row_subset_equals_full():
    R, K, T = 50, 64, 5
    rng = np.random.default_rng(4)
    W = rng.standard_normal((R, K)).astype(np.float32)
    X = rng.standard_normal((K, T)).astype(np.float32)
    mask, values, meta = _compressed(W, oracle.F32)
    full = oracle.spmm(values, meta, X, oracle.F32)
    rows = np.array([49, 0, 17, 17, 3])
    sub = oracle.spmm(values, meta, X, oracle.F32, rows=rows)
    assert np.array_equal(sub, full[rows])
