"""GPU parity on int8 weights (NM_S8) against the CPU oracle: masks, 2:4
compression (values, canonical metadata, tensor-core image), compression
under a mask, decompression and the transposable mask, byte for byte.  The
int8 sparse product is not built, so nm_spmm must refuse int8 operands."""
import numpy as np
import pytest
import torch

import oracle
import nm_inputs
import structured_sparsity_prune_b200 as nm

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from structured_sparsity_prune_b200 import build
    build.build()
    oracle.build()
    assert torch.cuda.is_available()


def _int8(shape, seed):
    g = torch.Generator().manual_seed(seed)
    W = torch.randint(-128, 128, shape, generator=g, dtype=torch.int16).to(torch.int8)
    W[::5, ::3] = -128
    W[::7, 1::4] = 127
    W[::3, 2::5] = 0
    return W


@pytest.mark.parametrize("N,M", [(1, 2), (1, 4), (2, 4), (3, 4), (2, 8), (4, 8), (3, 6)])
@pytest.mark.parametrize("C", [96, 48])
def test_mask(N, M, C):
    W = _int8((130, C), N * 10 + M)
    got = nm.nm_mask(W.cuda(), N, M).cpu().numpy()
    assert np.array_equal(got, oracle.mask_rank(W.numpy(), N, M))


def _all_groups_of_sixteen_values():
    """Every group of four drawn from 16 values with ties, both extremes and
    both signs of equal magnitudes: 16**4 groups, 1024 per row."""
    vals = np.array([-128, -127, -64, -5, -3, -2, -1, 0, 1, 2, 3, 5, 63, 64, 126, 127], dtype=np.int8)
    idx = np.indices((16, 16, 16, 16)).reshape(4, -1).T          # (65536, 4)
    return torch.from_numpy(vals[idx].reshape(64, 4096).copy())


@pytest.mark.parametrize("N", [1, 2, 3])
def test_mask_every_group_of_sixteen_values(N):
    W = _all_groups_of_sixteen_values()
    got = nm.nm_mask(W.cuda(), N, 4).cpu().numpy()
    assert np.array_equal(got, oracle.mask_rank(W.numpy(), N, 4))


def test_mask_compress_every_group_of_sixteen_values():
    W = _all_groups_of_sixteen_values()
    v, meta, img = nm.nm_mask_compress(W.cuda())
    rv, rm = oracle.compress24(W.numpy(), oracle.mask_rank(W.numpy(), 2, 4))
    assert np.array_equal(v.cpu().numpy(), rv)
    assert np.array_equal(meta.cpu().numpy(), rm)
    assert np.array_equal(img.cpu().numpy(), oracle.meta_sm100(rm, 64, 4096))


@pytest.mark.parametrize("R,C", [(256, 256), (200, 96), (130, 48)])
def test_mask_compress_and_image(R, C):
    W = _int8((R, C), R + C)
    v, meta, img = nm.nm_mask_compress(W.cuda())
    Wn = W.numpy()
    rv, rm = oracle.compress24(Wn, oracle.mask_rank(Wn, 2, 4))
    assert np.array_equal(v.cpu().numpy(), rv)
    assert np.array_equal(meta.cpu().numpy(), rm)
    assert np.array_equal(img.cpu().numpy(), oracle.meta_sm100(rm, R, C))
    back = nm.nm_decompress(v, meta, C).cpu().numpy()
    assert np.array_equal(back, oracle.decompress24(rv, rm, C).view(np.int8))


def test_compress_under_a_mask_counts_invalid_groups():
    R, C = 64, 128
    W = _int8((R, C), 3)
    mask = oracle.mask_rank(W.numpy(), 2, 4)
    bad = mask.copy()
    bad[2, 0:4] = [1, 1, 1, 0]        # invalid: three kept
    bad[9, 8:12] = [0, 0, 0, 0]       # valid: stored as (0,1) with zero values
    cnt = torch.zeros(1, dtype=torch.int32, device="cuda")
    v, meta, _ = nm.nm_compress(W.cuda(), torch.from_numpy(mask).cuda())
    rv, rm = oracle.compress24(W.numpy(), mask)
    assert np.array_equal(v.cpu().numpy(), rv) and np.array_equal(meta.cpu().numpy(), rm)
    nm.nm_compress(W.cuda(), torch.from_numpy(bad).cuda(), invalid_groups=cnt)
    assert int(cnt.item()) == 1


@pytest.mark.parametrize("N,M", [(4, 8), (2, 4), (1, 8)])
def test_transposable(N, M):
    W = _int8((M * 24, M * 16), 50 + M)
    got = nm.nm_mask_transposable(W.cuda(), N, M).cpu().numpy()
    assert np.array_equal(got, oracle.mask_transposable(W.numpy(), N, M))


def test_full_size_decode_weight_quantised():
    """The decode-sized weight quantised to int8 (round(w / 0.02 * 32), clamped), every row."""
    Wf = nm_inputs.decode_skinny_W().float()
    W = torch.clamp(torch.round(Wf / 0.02 * 32), -128, 127).to(torch.int8)
    v, meta, _ = nm.nm_mask_compress(W.cuda(), sm100=False)
    rv, rm = oracle.compress24(W.numpy(), oracle.mask_rank(W.numpy(), 2, 4))
    assert np.array_equal(v.cpu().numpy(), rv) and np.array_equal(meta.cpu().numpy(), rm)


def test_float_only_calls_refuse_int8():
    """int8 weights go to the selection, compression and product calls, not to
    the floating-point ones; the int8 product takes no 16-bit output type
    (host checks, nothing is launched)."""
    lib = nm.load()
    s = torch.cuda.current_stream().cuda_stream
    W = torch.zeros((128, 128), dtype=torch.int8, device="cuda")
    v, meta, img = nm.nm_mask_compress(W)
    X = torch.zeros((128, 64), dtype=torch.int8, device="cuda")
    Y = torch.empty((128, 64), dtype=torch.float16, device="cuda")
    st = lib.nm_spmm(v.data_ptr(), img.data_ptr(), 3, X.data_ptr(), 64, Y.data_ptr(), 2, 64, 128, 128, 64,
                     1.0, 0.0, None, 0, s)
    assert st == 4                                                     # NM_ERR_DTYPE: no fp16 output
    d = torch.ones(128, dtype=torch.float32, device="cuda")
    m = torch.empty((128, 128), dtype=torch.uint8, device="cuda")
    assert lib.nm_mask_scored(W.data_ptr(), 3, d.data_ptr(), 128, 128, 128, 2, 4, m.data_ptr(), 128, s) == 4
    import ctypes
    vb, mb, sb = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    assert lib.nm_sizes(128, 128, 2, 4, 3, ctypes.addressof(vb), ctypes.addressof(mb), ctypes.addressof(sb)) == 0
    assert (vb.value, mb.value) == (128 * 64, 128 * 16)
