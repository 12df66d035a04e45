"""GPU parity of the 2:4 sparse x dense product against the fp64 CPU oracle.

Tolerances (normalised Frobenius error ||Y - Y_ref|| / ||Y_ref||): 1e-3 for
fp32 output, 8e-3 for bf16 output; exact where the arithmetic is exact
(integer-valued inputs, one-hot rows)."""
import os

import numpy as np
import pytest
import torch

import oracle
import nm_inputs
import structured_sparsity_prune_b200 as nm

pytestmark = pytest.mark.gpu

CODE = {torch.float32: oracle.F32, torch.bfloat16: oracle.BF16, torch.float16: oracle.F16}
TOL = {torch.float32: 1e-3, torch.bfloat16: 8e-3}
THREADS = os.cpu_count() or 2


def _bits(t):
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.float32:
        return t.view(torch.int32).numpy().view(np.uint32)
    return t.view(torch.int16).numpy().view(np.uint16)


def _nerr(Y, ref):
    Yf = Y.detach().float().cpu().numpy().astype(np.float64)
    den = np.linalg.norm(ref)
    return np.linalg.norm(Yf - ref) / (den if den > 0 else 1.0)


def _dev(X):
    """Device copy of X in a buffer whose rows are 16-byte aligned (ldx % 8 == 0)."""
    K, T = X.shape
    buf = torch.zeros((K, (T + 7) // 8 * 8), dtype=X.dtype, device="cuda")
    buf[:, :T] = X.cuda()
    return buf[:, :T]


def _ok_status():
    assert nm.nm_last_device_status() == 0


@pytest.fixture(scope="module", autouse=True)
def _built():
    from structured_sparsity_prune_b200 import build
    build.build()
    oracle.build()
    assert torch.cuda.is_available()


def _run(W, X, y_dtype=torch.bfloat16, alpha=1.0, beta=0.0, Y0=None, rows=None, kernel=None):
    """GPU: fused compress then spmm (a forced tile configuration through the
    test entry point when `kernel` is given).  Oracle: its own compress then
    fp64 spmm."""
    ab = W.dtype
    values, meta, img = nm.nm_mask_compress(W.cuda())
    Y = None if Y0 is None else Y0.clone().cuda()
    if kernel is None:
        Y = nm.nm_spmm(values, img, _dev(X), Y=Y, y_dtype=y_dtype, alpha=alpha, beta=beta)
    else:
        Y = nm.nm_spmm_test(values, img, _dev(X), Y=Y, y_dtype=y_dtype, alpha=alpha, beta=beta, kernel=kernel)
    torch.cuda.synchronize()
    _ok_status()
    Wb = _bits(W)
    code = CODE[ab]
    _, v_ref, m_ref = oracle.rows_parallel(1, Wb, 2, 4, code, threads=THREADS)
    ref = oracle.spmm(v_ref, m_ref, _bits(X), code, alpha=alpha, beta=beta,
                      Y_in=None if Y0 is None else _bits(Y0), y_dtype=CODE[y_dtype], rows=rows, threads=THREADS)
    return Y.cpu() if rows is None else Y.cpu()[torch.as_tensor(rows)], ref


@pytest.mark.parametrize("y_dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("ab", [torch.bfloat16, torch.float16])
def test_small_square(ab, y_dtype):
    W = nm_inputs.normal((256, 256), 11, 0.02, ab)
    X = nm_inputs.normal((256, 128), 12, 1.0, ab)
    Y, ref = _run(W, X, y_dtype)
    assert _nerr(Y, ref) <= TOL[y_dtype]


CASES = [(1, 16, 1), (100, 48, 8), (128, 128, 16), (200, 64, 17), (333, 320, 64), (129, 192, 100),
         (256, 256, 128), (64, 512, 200), (300, 128, 256), (130, 256, 300), (40, 640, 520), (257, 384, 33)]


@pytest.mark.parametrize("R,K,T", CASES)
def test_ragged_shapes(R, K, T):
    W = nm_inputs.normal((R, K), R + K, 0.02, torch.bfloat16)
    X = nm_inputs.normal((K, T), T + 3, 1.0, torch.bfloat16)
    Y, ref = _run(W, X, torch.float32)
    assert _nerr(Y, ref) <= 1e-3


@pytest.mark.parametrize("T", [8, 64, 130, 256, 512])
def test_integer_inputs_are_exact(T):
    """Integers in [-8, 8], K = 256: every partial sum is exact in fp32, so the
    fp32 output equals the exact product bit for bit, and the bf16 output is
    its round-to-nearest-even."""
    R, K = 192, 256
    W = nm_inputs.small_int((R, K), 21, dtype=torch.bfloat16)
    X = nm_inputs.small_int((K, T), 22, dtype=torch.bfloat16)
    Y, ref = _run(W, X, torch.float32)
    assert np.array_equal(Y.numpy().astype(np.float64), ref)
    Yb, ref_b = _run(W, X, torch.bfloat16)
    expect = oracle.encode_array(ref_b, oracle.BF16)
    assert np.array_equal(_bits(Yb), expect)


def test_one_hot_rows_select_x_rows():
    R, K, T = 256, 512, 192
    g = torch.Generator().manual_seed(5)
    cols = torch.randint(0, K, (R,), generator=g)
    W = torch.zeros((R, K), dtype=torch.bfloat16)
    W[torch.arange(R), cols] = 1.0
    X = nm_inputs.normal((K, T), 6, 1.0, torch.bfloat16)
    values, meta, img = nm.nm_mask_compress(W.cuda())
    Y = nm.nm_spmm(values, img, X.cuda(), y_dtype=torch.float32)
    assert torch.equal(Y.cpu(), X[cols].float())


def test_oracle_image_drives_the_kernel():
    """The kernel reading an image built by the oracle (not by the GPU)."""
    R, K, T = 256, 384, 96
    W = nm_inputs.normal((R, K), 31, 1.0, torch.bfloat16)
    X = nm_inputs.normal((K, T), 32, 1.0, torch.bfloat16)
    Wb = _bits(W)
    v_ref, m_ref = oracle.compress24(Wb, oracle.mask_rank(Wb, 2, 4, dtype=oracle.BF16), dtype=oracle.BF16)
    img = torch.from_numpy(oracle.meta_sm100(m_ref, R, K)).cuda()
    vals = torch.from_numpy(np.ascontiguousarray(v_ref).view(np.int16)).view(torch.bfloat16).cuda()
    Y = nm.nm_spmm(vals, img, X.cuda(), y_dtype=torch.float32)
    ref = oracle.spmm(v_ref, m_ref, _bits(X), oracle.BF16, threads=THREADS)
    assert _nerr(Y, ref) <= 1e-3


@pytest.mark.parametrize("y_dtype", [torch.float32, torch.bfloat16])
def test_alpha_beta(y_dtype):
    R, K, T = 200, 256, 160
    W = nm_inputs.normal((R, K), 41, 0.02, torch.bfloat16)
    X = nm_inputs.normal((K, T), 42, 1.0, torch.bfloat16)
    Y0 = nm_inputs.normal((R, T), 43, 1.0, y_dtype)
    Y, ref = _run(W, X, y_dtype, alpha=2.0, beta=0.5, Y0=Y0)
    assert _nerr(Y, ref) <= TOL[y_dtype]


def test_beta_zero_never_reads_y():
    R, K, T = 130, 128, 72
    W = nm_inputs.normal((R, K), 51, 1.0, torch.bfloat16)
    X = nm_inputs.normal((K, T), 52, 1.0, torch.bfloat16)
    Y0 = torch.full((R, T), float("nan"), dtype=torch.float32)
    Y, ref = _run(W, X, torch.float32, alpha=1.0, beta=0.0, Y0=Y0)
    assert torch.isfinite(Y).all()
    assert _nerr(Y, ref) <= 1e-3


def test_strided_x_and_y():
    R, K, T = 160, 256, 100
    W = nm_inputs.normal((R, K), 61, 1.0, torch.float16)
    Xfull = nm_inputs.normal((K, T + 28), 62, 1.0, torch.float16)
    values, meta, img = nm.nm_mask_compress(W.cuda())
    Yfull = torch.full((R, T + 60), 9.0, dtype=torch.float32, device="cuda")
    nm.nm_spmm(values, img, Xfull.cuda()[:, :T], Y=Yfull[:, :T])
    Wb = _bits(W)
    v_ref, m_ref = oracle.compress24(Wb, oracle.mask_rank(Wb, 2, 4, dtype=oracle.F16), dtype=oracle.F16)
    ref = oracle.spmm(v_ref, m_ref, _bits(Xfull[:, :T].contiguous()), oracle.F16, threads=THREADS)
    assert _nerr(Yfull[:, :T], ref) <= 1e-3
    assert torch.all(Yfull[:, T:] == 9.0)


def test_fp32_inputs_small_workload():
    """The 256 x 256 fp32 weight, X 256 x 128 fp32: rounded to binary16 inside
    the call, fp32 accumulation and output; within 1e-3 of the fp64 product."""
    W, X = nm_inputs.small_fp32()
    Y, ref = _run(W, X, torch.float32)
    err = _nerr(Y, ref)
    assert err <= 1e-3, err


def test_repeat_calls_are_deterministic():
    W = nm_inputs.normal((384, 512), 71, 0.02, torch.bfloat16).cuda()
    X = nm_inputs.normal((512, 384), 72, 1.0, torch.bfloat16).cuda()
    values, meta, img = nm.nm_mask_compress(W)
    a = nm.nm_spmm(values, img, X)
    b = nm.nm_spmm(values, img, X)
    assert torch.equal(a, b)


def _sample_rows(R, per_tile=2):
    rows = []
    for t in range((R + 127) // 128):
        for j in range(per_tile):
            r = t * 128 + (37 * j + 11 * t) % 128
            if r < R:
                rows.append(r)
    rows.append(R - 1)
    return np.array(sorted(set(rows)), dtype=np.int64)


def test_linear_4096_full_size_sampled_rows():
    """4096 x 4096 x 4096 bf16 (bf16 out), rows sampled across every row tile."""
    W, X = nm_inputs.linear_4096()
    rows = _sample_rows(4096, 2)
    Y, ref = _run(W, X, torch.bfloat16, rows=rows)
    assert _nerr(Y, ref) <= 8e-3


def test_mlp_pair_full_size_sampled_rows():
    """The MLP pair at full size: up 14336 x 4096 x 8192, then down 4096 x
    14336 x 8192, bf16 out, rows sampled across every row tile.  The down
    product takes a seeded stand-in for H of the same shape and distribution,
    so no oracle input comes from the device."""
    W_up, W_down, X = nm_inputs.mlp_pair()
    H, ref = _run(W_up, X, torch.bfloat16, rows=_sample_rows(W_up.shape[0], 2))
    assert _nerr(H, ref) <= 8e-3
    Y, ref = _run(W_down, nm_inputs.mlp_hidden(), torch.bfloat16, rows=_sample_rows(W_down.shape[0], 2))
    assert _nerr(Y, ref) <= 8e-3


@pytest.mark.parametrize("T", [16, 64, 256, 1024])
def test_decode_skinny_full_size_sampled_rows(T):
    W = nm_inputs.decode_skinny_W()
    X = nm_inputs.decode_skinny_X(T)
    rows = _sample_rows(W.shape[0], 1)
    Y, ref = _run(W, X, torch.bfloat16, rows=rows)
    assert _nerr(Y, ref) <= 8e-3



KERNELS = ["pair256", "pair192", "pair128", "single256", "single128", "single64", "single64x2",
           "single32x2", "single16x2"]


@pytest.mark.parametrize("kern", KERNELS)
def test_every_tile_shape_is_exact_on_integers(kern):
    """Each tile configuration, forced through the test entry point, on a shape
    ragged in R (700 = 5.5 row tiles) and T (500 columns, a partial last tile
    for every width): integer inputs make the fp32 output exact and the bf16
    output its round-to-nearest-even, on both epilogue paths."""
    R, K, T = 700, 384, 500
    W = nm_inputs.small_int((R, K), 81, dtype=torch.bfloat16)
    X = nm_inputs.small_int((K, T), 82, dtype=torch.bfloat16)
    Y, ref = _run(W, X, torch.float32, kernel=kern)
    assert np.array_equal(Y.numpy().astype(np.float64), ref)
    Yb, ref_b = _run(W, X, torch.bfloat16, kernel=kern)
    assert np.array_equal(_bits(Yb), oracle.encode_array(ref_b, oracle.BF16))


@pytest.mark.parametrize("kern", KERNELS)
def test_every_tile_shape_alpha_beta(kern):
    R, K, T = 700, 256, 500
    W = nm_inputs.normal((R, K), 83, 0.02, torch.bfloat16)
    X = nm_inputs.normal((K, T), 84, 1.0, torch.bfloat16)
    Y0 = nm_inputs.normal((R, T), 85, 1.0, torch.bfloat16)
    Y, ref = _run(W, X, torch.bfloat16, alpha=1.5, beta=0.5, Y0=Y0, kernel=kern)
    assert _nerr(Y, ref) <= 8e-3


@pytest.mark.parametrize("R,T", [(2560, 2048), (2500, 2000)])
def test_half_width_last_wave_is_exact(R, T):
    """80 pair tiles on 74 pairs: the last 6 tiles run as 12 half-width items
    (ragged in R and T in the second case); integer inputs make the fp32
    output exact and the bf16 output its round-to-nearest-even."""
    K = 128
    W = nm_inputs.small_int((R, K), 91, dtype=torch.bfloat16)
    X = nm_inputs.small_int((K, T), 92, dtype=torch.bfloat16)
    Y, ref = _run(W, X, torch.float32, kernel="pair256")
    assert np.array_equal(Y.numpy().astype(np.float64), ref)
    Yb, ref_b = _run(W, X, torch.bfloat16, kernel="pair256")
    assert np.array_equal(_bits(Yb), oracle.encode_array(ref_b, oracle.BF16))


def test_half_width_last_wave_matches_whole_tiles():
    """Splitting the last wave does not change the summation order, so the
    result equals the unsplit run bit for bit."""
    W = nm_inputs.normal((4096, 1024), 93, 0.02, torch.bfloat16).cuda()
    X = nm_inputs.normal((1024, 4096), 94, 1.0, torch.bfloat16).cuda()
    values, meta, img = nm.nm_mask_compress(W)
    a = nm.nm_spmm(values, img, X)
    b = nm.nm_spmm_test(values, img, X, tail_split=False)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


@pytest.mark.parametrize("kern,R,T", [("pair256", 1024, 1024), ("single256", 640, 512), ("single16x2", 384, 16)])
def test_bounded_wait_runs_out_and_the_next_call_is_clean(kern, R, T):
    """The failure path of the product kernel's bounded waits, driven without a
    fault: through the test entry point the producer never fills its first
    pipeline stage and every wait is limited to 5 ms, so the MMA issuer's wait
    on that stage runs out.  The kernel must record NM_ERR_TIMEOUT, stop its
    other roles, let its copies land, free its tensor memory and return; the
    next ordinary call on the same stream must then run and match the oracle,
    and leave the status word clear."""
    K = 512
    W = nm_inputs.normal((R, K), 97, 0.02, torch.bfloat16)
    X = nm_inputs.normal((K, T), 98, 1.0, torch.bfloat16)
    values, meta, img = nm.nm_mask_compress(W.cuda())
    Xd = _dev(X)
    assert nm.nm_last_device_status() == 0
    nm.nm_spmm_test(values, img, Xd, y_dtype=torch.float32, kernel=kern, wait_limit_ns=5_000_000, skip_step=0)
    assert nm.nm_last_device_status() == 9          # NM_ERR_TIMEOUT, read and cleared
    assert nm.nm_last_device_status() == 0
    Y, ref = _run(W, X, torch.float32)              # an ordinary call afterwards
    assert _nerr(Y, ref) <= 1e-3
    Y2 = nm.nm_spmm_test(values, img, Xd, y_dtype=torch.float32, kernel=kern)
    torch.cuda.synchronize()
    assert nm.nm_last_device_status() == 0
    assert _nerr(Y2.cpu(), ref) <= 1e-3


@pytest.mark.skipif(torch.cuda.device_count() < 2, reason="needs two visible GPUs")
def test_second_device_after_the_first():
    """The kernels' shared-memory attributes, the SM count and the scratch address
    are cached per device: products on device 1 after products on device 0 (the
    CTA-pair kernel and the skinny one, both above 48 KB of shared memory) run
    and stay exact on integer inputs."""
    prev = torch.cuda.current_device()
    try:
        for dev in (0, 1, 0):
            torch.cuda.set_device(dev)
            for R, K, T in [(512, 256, 512), (384, 256, 16)]:
                W = nm_inputs.small_int((R, K), 91 + T, dtype=torch.bfloat16)
                X = nm_inputs.small_int((K, T), 92 + T, dtype=torch.bfloat16)
                Y, ref = _run(W, X, torch.float32)
                assert np.array_equal(Y.numpy().astype(np.float64), ref)
    finally:
        torch.cuda.set_device(prev)


# (R, K, T, ldy, y_dtype, beta, kernel): outputs that are views with ldy > T
VIEW_CASES = [
    (1000, 512, 333, 344, torch.bfloat16, 0.0, "default"),   # ragged T: plain stores
    (1024, 512, 330, 344, torch.float32, 0.0, "default"),
    (1000, 512, 328, 344, torch.bfloat16, 0.0, "default"),   # whole 16-byte rows: staged bulk stores
    (1024, 512, 332, 344, torch.float32, 0.0, "default"),
    (1000, 512, 333, 344, torch.bfloat16, 0.5, "default"),   # beta != 0 reads and writes Y in place
    (256, 256, 77, 80, torch.bfloat16, 0.0, "pair128"),
    (384, 256, 333, 344, torch.bfloat16, 0.0, "single256"),
    (384, 256, 45, 48, torch.float32, 0.0, "single64x2"),
]


@pytest.mark.parametrize("R,K,T,ldy,y_dtype,beta,kernel", VIEW_CASES)
def test_output_view_writes_nothing_outside(R, K, T, ldy, y_dtype, beta, kernel):
    """Y a view (R x T, leading dim ldy > T) of a larger buffer whose other
    elements hold a sentinel: every element outside the view keeps it, for
    each epilogue (staged bulk stores, plain vector stores, element stores)."""
    S = -3.0
    W = nm_inputs.normal((R, K), 401 + T, 0.02, torch.bfloat16)
    X = nm_inputs.normal((K, T), 402 + T, 1.0, torch.bfloat16)
    Y0 = nm_inputs.normal((R, T), 403, 1.0, y_dtype) if beta else None
    values, meta, img = nm.nm_mask_compress(W.cuda())
    big = torch.full((R + 40, ldy), S, dtype=y_dtype, device="cuda")
    Yv = big[:R, :T]
    if Y0 is not None:
        Yv.copy_(Y0.cuda())
    nm.nm_spmm_test(values, img, _dev(X), Y=Yv, y_dtype=y_dtype, beta=beta, kernel=kernel)
    torch.cuda.synchronize()
    _ok_status()
    outside = torch.ones(big.shape, dtype=torch.bool, device="cuda")
    outside[:R, :T] = False
    assert bool((big[outside] == S).all()), "stores outside the R x T view"
    Wb = _bits(W)
    _, v_ref, m_ref = oracle.rows_parallel(1, Wb, 2, 4, oracle.BF16, threads=THREADS)
    ref = oracle.spmm(v_ref, m_ref, _bits(X), oracle.BF16, beta=beta, Y_in=None if Y0 is None else _bits(Y0),
                      y_dtype=CODE[y_dtype], threads=THREADS)
    assert _nerr(Yv, ref) <= TOL[y_dtype]


def test_mlp_chain_against_an_fp64_chain():
    """The MLP pair's chain at a reduced size: the up product, H kept in bf16
    on the GPU, the down product; against the oracle's chain with H in fp64
    (the down weight decompressed by the oracle, one fp64 matmul).  The only
    error beyond each product's own is H's bf16 rounding (at most 2^-9
    relative per element, about 2^-9 / sqrt(3) RMS), so the chain stays within
    the bf16-output bound."""
    R, K, T = 2048, 512, 1024
    Wu = nm_inputs.normal((R, K), 511, 0.02, torch.bfloat16)
    Wd = nm_inputs.normal((K, R), 512, 0.02, torch.bfloat16)
    X = nm_inputs.normal((K, T), 513, 1.0, torch.bfloat16)
    vu, mu, iu = nm.nm_mask_compress(Wu.cuda())
    vd, md, idn = nm.nm_mask_compress(Wd.cuda())
    H = nm.nm_spmm(vu, iu, X.cuda())
    Y = nm.nm_spmm(vd, idn, H)
    torch.cuda.synchronize()
    _ok_status()
    _, vu_r, mu_r = oracle.rows_parallel(1, _bits(Wu), 2, 4, oracle.BF16, threads=THREADS)
    H_ref = oracle.spmm(vu_r, mu_r, _bits(X), oracle.BF16, threads=THREADS)
    _, vd_r, md_r = oracle.rows_parallel(1, _bits(Wd), 2, 4, oracle.BF16, threads=THREADS)
    Wd_m = oracle.decode_array(oracle.decompress24(vd_r, md_r, R, dtype=oracle.BF16), oracle.BF16)
    err = _nerr(Y, Wd_m @ H_ref)
    print("MLP chain (bf16 H) against the fp64 chain: normalised error %.3e" % err)
    assert err <= 8e-3
