"""Out-of-bounds write checks for every entry point that writes device memory.

compute-sanitizer is not available here, so guard bands stand in for its
memory checker: each output is a view inside a larger buffer whose other bytes
(4 KiB before and after it, and the gaps between rows when the row stride is
wider than a row) hold a sentinel byte.  After the call every one of those
bytes must still hold it.  Shapes are ragged where the call allows, so the
tail paths of each kernel run, and one large weight takes the staged (ring)
kernels.  Values are not checked here; the parity tests do that."""
import pytest
import torch

import nm_inputs
import structured_sparsity_prune_b200 as nm

pytestmark = pytest.mark.gpu

G = 4096          # guard bytes on each side (keeps every view 16-byte aligned)
SENT = 0xA5


@pytest.fixture(scope="module", autouse=True)
def _built():
    from structured_sparsity_prune_b200 import build
    build.build()
    assert torch.cuda.is_available()


class Guarded:
    """A rows x cols view (row stride ld elements) or a flat view of n
    elements, inside a sentinel-filled byte buffer."""

    def __init__(self, dtype, rows, cols=None, ld=None):
        self.es = torch.empty((), dtype=dtype).element_size()
        self.rows, self.cols = rows, cols
        self.ld = cols if ld is None else ld
        n = rows * (self.ld if cols is not None else 1)
        self.nbytes = n * self.es
        self.big = torch.full((self.nbytes + 2 * G,), SENT, dtype=torch.uint8, device="cuda")
        inner = self.big[G:G + self.nbytes].view(dtype)
        self.t = inner if cols is None else inner.view(rows, self.ld)[:, :cols]

    def intact(self):
        ok = bool((self.big[:G] == SENT).all()) and bool((self.big[G + self.nbytes:] == SENT).all())
        if self.cols is not None and self.ld > self.cols:
            rows = self.big[G:G + self.nbytes].view(self.rows, self.ld * self.es)
            ok = ok and bool((rows[:, self.cols * self.es:] == SENT).all())
        return ok


def _done(*outs):
    torch.cuda.synchronize()
    assert nm.nm_last_device_status() == 0
    for o in outs:
        assert o.intact(), "a store landed outside its output"


def _weight(R, C, dtype, seed):
    if dtype == torch.int8:
        return nm_inputs.small_int8((R, C), seed).cuda()
    return nm_inputs.normal((R, C), seed, 0.02, dtype).cuda()


def _mask_input(W, N, M):
    """A mask to feed a compressing call: rows padded to 16 bytes, as masks must be."""
    R, C = W.shape
    buf = torch.empty((R, (C + 15) // 16 * 16), dtype=torch.uint8, device="cuda")
    return nm.nm_mask(W, N, M, mask=buf[:, :C])


def _compressed(R, C, dtype):
    _, mb, sb = nm.nm_sizes(R, C, 2, 4, dtype)
    return Guarded(dtype, R, C // 2), Guarded(torch.uint8, R, C // 8), Guarded(torch.uint8, sb)


@pytest.mark.parametrize("R,C,N,M,dtype", [(257, 96, 2, 4, torch.bfloat16), (257, 96, 4, 8, torch.bfloat16),
                                           (1000, 1040, 2, 4, torch.bfloat16), (129, 80, 1, 4, torch.float32),
                                           (257, 96, 2, 4, torch.int8), (130, 48, 3, 8, torch.float16)])
def test_mask(R, C, N, M, dtype):
    W = _weight(R, C, dtype, R + C)
    out = Guarded(torch.uint8, R, C, ld=C + 16)
    nm.nm_mask(W, N, M, mask=out.t)
    _done(out)


@pytest.mark.parametrize("R,C,dtype", [(257, 72, torch.bfloat16), (1000, 1056, torch.bfloat16),
                                       (16384, 8192, torch.bfloat16), (257, 96, torch.int8),
                                       (129, 40, torch.float32)])
def test_mask_compress_compress_decompress(R, C, dtype):
    W = _weight(R, C, dtype, 3 * R + C)
    v, m, img = _compressed(R, C, dtype)
    nm.nm_mask_compress(W, v.t, m.t, img.t)
    _done(v, m, img)
    mask = _mask_input(W, 2, 4)
    v2, m2, img2 = _compressed(R, C, dtype)
    nm.nm_compress(W, mask, v2.t, m2.t, img2.t)
    _done(v2, m2, img2)
    pad = 16 if dtype == torch.int8 else 8
    out = Guarded(dtype, R, C, ld=C + pad)              # strided rows
    nm.nm_decompress(v.t, m.t, C, out=out.t)
    dense = Guarded(dtype, R, C)                        # contiguous (the staged kernel where it applies)
    nm.nm_decompress(v.t, m.t, C, out=dense.t)
    _done(out, dense)
    if dtype == torch.int8:
        img8 = Guarded(torch.uint8, nm.nm_meta_s8_image_bytes(R, C))
        nm.nm_meta_to_sm100_s8(m.t, R, C, out=img8.t)
        _done(img8)
    else:
        img3 = Guarded(torch.uint8, img.t.numel())
        nm.nm_meta_to_sm100(m.t, R, C, out=img3.t)
        _done(img3)


@pytest.mark.parametrize("R,C,N,M", [(264, 72, 2, 4), (1000, 1040, 2, 4), (256, 96, 4, 8)])
def test_transposable_mask_and_compress_t(R, C, N, M):
    W = _weight(R, C, torch.bfloat16, R * C)
    out = Guarded(torch.uint8, R, C, ld=C + 16 - C % 16)
    nm.nm_mask_transposable(W, N, M, mask=out.t)
    _done(out)
    if (N, M) == (2, 4):
        v, m, img = _compressed(C, R, torch.bfloat16)
        nm.nm_compress_t(W, out.t, v.t, m.t, img.t)
        _done(v, m, img)


@pytest.mark.parametrize("R,C,dtype", [(257, 80, torch.float32), (1000, 1040, torch.float32),
                                       (130, 48, torch.bfloat16)])
def test_one_two_family(R, C, dtype):
    W = _weight(R, C, dtype, R + 7 * C)
    v = Guarded(dtype, R, C // 2)
    m = Guarded(torch.uint8, R, C // 16)
    nm.nm_mask_compress12(W, v.t, m.t)
    _done(v, m)
    mask = _mask_input(W, 1, 2)
    v2, m2 = Guarded(dtype, R, C // 2), Guarded(torch.uint8, R, C // 16)
    nm.nm_compress12(W, mask, v2.t, m2.t)
    _done(v2, m2)
    es = torch.empty((), dtype=dtype).element_size()
    out = Guarded(dtype, R, C, ld=C + 16 // es)
    nm.nm_decompress12(v.t, m.t, C, out=out.t)
    img = Guarded(torch.uint8, nm.nm_meta12_image_bytes(R, C))
    nm.nm_meta12_to_sm100(m.t, R, C, out=img.t)
    _done(out, img)


@pytest.mark.parametrize("R,C,dtype", [(257, 80, torch.bfloat16), (1000, 1024, torch.float32)])
def test_srste_step(R, C, dtype):
    ld = C + 16
    Wb = torch.zeros((R, ld), dtype=dtype, device="cuda")
    Gb = torch.zeros((R, ld), dtype=dtype, device="cuda")
    Wb[:, :C] = _weight(R, C, dtype, 11)
    Gb[:, :C] = _weight(R, C, dtype, 12)
    ws, go, mk = Guarded(dtype, R, C, ld=ld), Guarded(dtype, R, C, ld=ld), Guarded(torch.uint8, R, C, ld=ld)
    nm.nm_srste_step(Wb[:, :C], Gb[:, :C], 2, 4, 0.0002, W_sparse=ws.t, grad_out=go.t, mask=mk.t)
    _done(ws, go, mk)


def test_scored_mask():
    R, C = 257, 96
    W = _weight(R, C, torch.bfloat16, 21)
    d = (torch.rand(C, generator=torch.Generator().manual_seed(22)) + 0.5).cuda()
    out = Guarded(torch.uint8, R, C, ld=C + 16)
    nm.nm_mask_scored(W, d, 2, 4, mask=out.t)
    _done(out)


@pytest.mark.parametrize("R,K,T,kernel", [(1000, 512, 328, "default"), (384, 256, 45, "default"),
                                          (256, 256, 77, "pair128"), (2560, 2048, 2000, "default")])
def test_spmm(R, K, T, kernel):
    W = _weight(R, K, torch.bfloat16, 31)
    values, meta, img = nm.nm_mask_compress(W)
    Tp = (T + 7) // 8 * 8
    Xb = torch.zeros((K, Tp), dtype=torch.bfloat16, device="cuda")
    Xb[:, :T] = nm_inputs.normal((K, T), 32, 1.0, torch.bfloat16).cuda()
    for y_dtype in (torch.bfloat16, torch.float32):
        Y = Guarded(y_dtype, R, T)
        nm.nm_spmm_test(values, img, Xb[:, :T], Y=Y.t, y_dtype=y_dtype, kernel=kernel)
        _done(Y)


@pytest.mark.parametrize("R,K,T", [(257, 80, 100), (512, 256, 300)])
def test_spmm12(R, K, T):
    W = _weight(R, K, torch.float32, 41)
    v, m = nm.nm_mask_compress12(W)
    img = nm.nm_meta12_to_sm100(m, R, K)
    X = nm_inputs.normal((K, T), 42, 1.0, torch.float32).cuda()
    Y = Guarded(torch.float32, R, T)
    nm.nm_spmm12(v, img, X, Y=Y.t)
    _done(Y)


def test_int8_product():
    R, K, T = 700, 512, 500
    W = _weight(R, K, torch.int8, 51)
    v, m, _ = nm.nm_mask_compress(W, sm100=False)
    img = nm.nm_meta_to_sm100_s8(m, R, K)
    Xb = torch.zeros((K, 512), dtype=torch.int8, device="cuda")
    Xb[:, :T] = nm_inputs.small_int8((K, T), 52).cuda()
    for y_dtype in (torch.int32, torch.float32, torch.bfloat16):
        Y = Guarded(y_dtype, R, T)
        nm.nm_spmm(v, img, Xb[:, :T], Y=Y.t, y_dtype=y_dtype)
        _done(Y)
