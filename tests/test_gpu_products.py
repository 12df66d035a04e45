"""GPU parity of the int8 2:4 product and the TF32 1:2 product against the CPU
oracle, and of their metadata images.

Sources: review of "Accelerating Sparse Deep Neural Networks", "Structured
sparse GEMM on tensor cores" (the sparse tensor cores take INT8 at 2:4 and
TF32 only at 1:2; INT8 dimensions in multiples of 32).

Bars: the int8 product accumulates in s32, so its int32 output is compared
bit for bit with the oracle's exact int64 sum (and fp32 / bf16 outputs with
the exactly rounded value where the sums stay below 2^24).  The TF32 product
reads values and X with 10 fraction bits: every product a*b then carries a
relative error below 2^-10 from each operand, 2^-9 together, and with
independent signs across the K terms the normalised Frobenius error of Y is
the root mean square of those per-term errors, so at most 2^-9 plus fp32
accumulation (well below 2^-12 here): the bar is 2e-3.  Integer inputs of
magnitude <= 8 are exact in TF32 and give an exact fp32 Y."""
import os

import numpy as np
import pytest
import torch

import nm_inputs
import oracle
import structured_sparsity_prune_b200 as nm

pytestmark = pytest.mark.gpu

THREADS = os.cpu_count() or 2
TF32_TOL = 2e-3
KERNELS = ["default", "pair256", "pair192", "pair128", "single256", "single128", "single64", "single64x2",
           "single32x2", "single16x2"]


@pytest.fixture(scope="module", autouse=True)
def _built():
    from structured_sparsity_prune_b200 import build
    build.build()
    oracle.build()
    assert torch.cuda.is_available()


def _dev_x(X, mult):
    """X on the device with a leading dimension that is a multiple of `mult` elements."""
    K, T = X.shape
    buf = torch.zeros((K, (T + mult - 1) // mult * mult), dtype=X.dtype, device="cuda")
    buf[:, :T] = X.cuda()
    return buf[:, :T]


def _nerr(Y, ref):
    y = Y.detach().double().cpu().numpy()
    den = np.linalg.norm(ref)
    return np.linalg.norm(y - ref) / (den if den > 0 else 1.0)


# ---------------------------------------------------------------- int8 2:4
def _s8_case(R, K, T, seed):
    W = nm_inputs.small_int8((R, K), seed)
    X = nm_inputs.small_int8((K, T), seed + 1)
    return W, X


def _s8_gpu(W, X, y_dtype=torch.int32, kernel="default", alpha=1.0, beta=0.0, Y0=None):
    R, K = W.shape
    values, meta, _ = nm.nm_mask_compress(W.cuda(), sm100=False)
    img = nm.nm_meta_to_sm100_s8(meta, R, K)
    Y = None if Y0 is None else Y0.clone().cuda()
    Y = nm.nm_spmm_test(values, img, _dev_x(X, 16), Y=Y, y_dtype=y_dtype, alpha=alpha, beta=beta, kernel=kernel)
    torch.cuda.synchronize()
    assert nm.nm_last_device_status() == 0
    return Y.cpu(), values, meta


def _s8_ref(W, X, rows=None, alpha=1.0, beta=0.0, Y0=None):
    Wn = W.numpy()
    mask = oracle.mask_rank(Wn, 2, 4)
    v, m = oracle.compress24(Wn, mask)
    return oracle.spmm(v, m, X.numpy(), oracle.S8, alpha=alpha, beta=beta,
                       Y_in=None if Y0 is None else Y0.numpy(), y_dtype=oracle.F32, rows=rows, threads=THREADS)


S8_CASES = [(128, 64, 8), (256, 256, 256), (300, 160, 100), (700, 512, 500), (129, 96, 33), (512, 1024, 1000),
            (1, 32, 1), (257, 32, 130), (384, 288, 1), (2, 4096, 7)]


@pytest.mark.parametrize("R,K,T", S8_CASES)
def test_int8_product_is_exact(R, K, T):
    """Ragged R, K (multiples of 32) and T: the int32 output equals the exact sum."""
    W, X = _s8_case(R, K, T, R + K + T)
    Y, values, meta = _s8_gpu(W, X)
    ref = _s8_ref(W, X)
    assert np.array_equal(Y.numpy().astype(np.float64), ref)


@pytest.mark.parametrize("kern", KERNELS)
def test_int8_every_tile_configuration_is_exact(kern):
    R, K, T = 700, 768, 500
    W, X = _s8_case(R, K, T, 31)
    Y, _, _ = _s8_gpu(W, X, kernel=kern)
    assert np.array_equal(Y.numpy().astype(np.float64), _s8_ref(W, X))


def test_int8_float_outputs_and_alpha_beta():
    """fp32 output alpha * sum: exact (sums far below 2^24, alpha a power of two);
    bf16 output its round-to-nearest-even; fp32 with beta: within 1e-6."""
    R, K, T = 384, 256, 200
    W, X = _s8_case(R, K, T, 41)
    exact = _s8_ref(W, X)
    Yf, _, _ = _s8_gpu(W, X, torch.float32, alpha=0.25)
    assert np.array_equal(Yf.numpy().astype(np.float64), 0.25 * exact)
    Yb, _, _ = _s8_gpu(W, X, torch.bfloat16, alpha=0.25)
    bits = Yb.view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(bits, oracle.encode_array(0.25 * exact, oracle.BF16))
    Y0 = nm_inputs.normal((R, T), 42, 100.0, torch.float32)
    Yab, _, _ = _s8_gpu(W, X, torch.float32, alpha=0.5, beta=-1.5, Y0=Y0)
    ref = _s8_ref(W, X, alpha=0.5, beta=-1.5, Y0=Y0)
    assert _nerr(Yab, ref) <= 1e-6


def test_int8_image_kernel_matches_oracle_and_drives_the_product():
    for R, C in [(256, 512), (100, 384), (129, 96), (1, 32)]:
        meta = torch.randint(0, 256, (R, C // 8), dtype=torch.uint8)
        img = nm.nm_meta_to_sm100_s8(meta.cuda(), R, C)
        assert np.array_equal(img.cpu().numpy(), oracle.meta_sm100_s8(meta.numpy(), R, C))
    # an oracle-built image in the product
    R, K, T = 256, 512, 64
    W, X = _s8_case(R, K, T, 51)
    Wn = W.numpy()
    v, m = oracle.compress24(Wn, oracle.mask_rank(Wn, 2, 4))
    img = torch.from_numpy(oracle.meta_sm100_s8(m, R, K)).cuda()
    Y = nm.nm_spmm(torch.from_numpy(v.view(np.int8)).cuda(), img, _dev_x(X, 16), y_dtype=torch.int32)
    torch.cuda.synchronize()
    assert np.array_equal(Y.cpu().numpy().astype(np.float64), oracle.spmm(v, m, X.numpy(), oracle.S8))


def _sample_rows(R, per_tile=2):
    rng = np.random.default_rng(R)
    rows = []
    for t in range(0, R, 128):
        rows += sorted(rng.choice(np.arange(t, min(R, t + 128)), size=min(per_tile, min(R, t + 128) - t),
                                  replace=False).tolist())
    return np.array(rows, dtype=np.int64)


@pytest.mark.parametrize("T", [16, 64, 256, 1024])
def test_int8_full_size_decode_weight(T):
    """The 28672 x 8192 decode weight quantised to int8, X the decode activations
    quantised to int8: sampled rows of every row tile, exact."""
    W = nm_inputs.int8_decode()
    X = nm_inputs.decode_X_int8(T)
    Y, _, _ = _s8_gpu(W, X)
    rows = _sample_rows(W.shape[0], 1)
    ref = _s8_ref(W, X, rows=rows)
    assert np.array_equal(Y.numpy()[rows].astype(np.float64), ref)


# ---------------------------------------------------------------- TF32 1:2
def _tf32_gpu(W, X, y_dtype=torch.float32, kernel=None, alpha=1.0, beta=0.0, Y0=None):
    R, K = W.shape
    values, meta = nm.nm_mask_compress12(W.cuda())
    img = nm.nm_meta12_to_sm100(meta, R, K)
    Y = None if Y0 is None else Y0.clone().cuda()
    if kernel is None:
        Y = nm.nm_spmm12(values, img, _dev_x(X, 4), Y=Y, y_dtype=y_dtype, alpha=alpha, beta=beta)
    else:
        Y = nm.nm_spmm12_test(values, img, _dev_x(X, 4), Y=Y, y_dtype=y_dtype, alpha=alpha, beta=beta,
                              kernel=kernel)
    torch.cuda.synchronize()
    assert nm.nm_last_device_status() == 0
    return Y.cpu()


def _tf32_ref(W, X, rows=None, alpha=1.0, beta=0.0, Y0=None):
    Wn = W.numpy()
    v, m = oracle.compress12(Wn, oracle.mask_rank(Wn, 1, 2))
    return oracle.spmm12(v, m, X.numpy(), alpha=alpha, beta=beta, Y_in=None if Y0 is None else Y0.numpy(),
                         rows=rows, threads=THREADS)


TF32_CASES = [(128, 64, 8), (256, 256, 256), (300, 160, 100), (700, 512, 500), (129, 96, 33), (40, 16, 3),
              (1, 16, 1), (257, 48, 129), (384, 80, 2)]


@pytest.mark.parametrize("R,K,T", TF32_CASES)
def test_tf32_integer_inputs_are_exact(R, K, T):
    W = nm_inputs.small_int((R, K), R + K, dtype=torch.float32)
    X = nm_inputs.small_int((K, T), T + 5, dtype=torch.float32)
    Y = _tf32_gpu(W, X)
    assert np.array_equal(Y.numpy().astype(np.float64), _tf32_ref(W, X))


@pytest.mark.parametrize("R,K,T", TF32_CASES)
def test_tf32_random_within_tolerance(R, K, T):
    W = nm_inputs.normal((R, K), R * 3 + K, 0.02, torch.float32)
    X = nm_inputs.normal((K, T), T * 3 + 1, 1.0, torch.float32)
    Y = _tf32_gpu(W, X)
    assert _nerr(Y, _tf32_ref(W, X)) <= TF32_TOL


@pytest.mark.parametrize("kern", KERNELS)
def test_tf32_every_tile_configuration_is_exact_on_integers(kern):
    R, K, T = 700, 384, 500
    W = nm_inputs.small_int((R, K), 61, dtype=torch.float32)
    X = nm_inputs.small_int((K, T), 62, dtype=torch.float32)
    Y = _tf32_gpu(W, X, kernel=kern)
    assert np.array_equal(Y.numpy().astype(np.float64), _tf32_ref(W, X))


def test_tf32_bf16_output_alpha_beta():
    R, K, T = 384, 256, 200
    W = nm_inputs.normal((R, K), 71, 0.02, torch.float32)
    X = nm_inputs.normal((K, T), 72, 1.0, torch.float32)
    Y0 = nm_inputs.normal((R, T), 73, 1.0, torch.float32)
    Y = _tf32_gpu(W, X, torch.float32, alpha=1.5, beta=0.5, Y0=Y0)
    assert _nerr(Y, _tf32_ref(W, X, alpha=1.5, beta=0.5, Y0=Y0)) <= TF32_TOL
    Yb = _tf32_gpu(W, X, torch.bfloat16)
    assert _nerr(Yb, _tf32_ref(W, X)) <= 8e-3


def test_tf32_image_kernel_matches_oracle_and_drives_the_product():
    for R, C in [(256, 128), (100, 80), (129, 16), (1, 64)]:
        meta = torch.randint(0, 256, (R, C // 16), dtype=torch.uint8)
        img = nm.nm_meta12_to_sm100(meta.cuda(), R, C)
        assert np.array_equal(img.cpu().numpy(), oracle.meta12_sm100(meta.numpy(), R, C))
    R, K, T = 256, 256, 64
    W = nm_inputs.small_int((R, K), 81, dtype=torch.float32)
    X = nm_inputs.small_int((K, T), 82, dtype=torch.float32)
    Wn = W.numpy()
    v, m = oracle.compress12(Wn, oracle.mask_rank(Wn, 1, 2))
    img = torch.from_numpy(oracle.meta12_sm100(m, R, K)).cuda()
    Y = nm.nm_spmm12(torch.from_numpy(v).cuda(), img, _dev_x(X, 4))
    torch.cuda.synchronize()
    assert np.array_equal(Y.cpu().numpy().astype(np.float64), oracle.spmm12(v, m, X.numpy()))


def test_tf32_full_size_fp32_weight():
    """The fp32 8192 x 8192 weight (1:2 pattern) times X fp32 8192 x 4096:
    sampled rows of every row tile within the TF32 bar."""
    W = nm_inputs.fp32_linear()
    X = nm_inputs.fp32_linear_X(4096)
    Y = _tf32_gpu(W, X)
    rows = _sample_rows(W.shape[0], 2)
    ref = _tf32_ref(W, X, rows=rows)
    assert _nerr(Y[torch.as_tensor(rows)], ref) <= TF32_TOL
