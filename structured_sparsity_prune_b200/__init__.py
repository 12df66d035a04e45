"""Python binding of libnm (include/nm.h): N:M structured sparsity on B200.

Argument marshalling only: every step runs in the CUDA kernels of
``libnm.so``.  Functions keep the C names; tensors are torch CUDA tensors
(torch supplies device memory and streams), pointers and sizes are passed
straight through, and a non-zero status raises ``NMError``.  There is no CPU
fallback: if ``libnm.so`` is missing or fails to load, every call raises.

Element types: torch.float32 -> NM_F32, torch.bfloat16 -> NM_BF16,
torch.float16 -> NM_F16, torch.int8 -> NM_S8, torch.int32 -> NM_S32 (the
int8 product's exact output).
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libnm.so")

NM_F32, NM_BF16, NM_F16, NM_S8, NM_S32 = 0, 1, 2, 3, 4
STATUS = ["NM_OK", "NM_ERR_NULL", "NM_ERR_SHAPE", "NM_ERR_ALIGN", "NM_ERR_DTYPE", "NM_ERR_NM",
          "NM_ERR_UNSUPPORTED", "NM_ERR_CUDA", "NM_ERR_WORKSPACE", "NM_ERR_TIMEOUT"]
_DT = {torch.float32: NM_F32, torch.bfloat16: NM_BF16, torch.float16: NM_F16, torch.int8: NM_S8,
       torch.int32: NM_S32}


class NMError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__("%s: %s" % (what, _lib().nm_status_string(status).decode()))


_LIB = None


def _lib():
    global _LIB
    if _LIB is not None:
        return _LIB
    if not os.path.exists(LIB_PATH):
        raise ImportError("libnm.so not built (python -m structured_sparsity_prune_b200.build): " + LIB_PATH)
    lib = ctypes.CDLL(LIB_PATH)
    i64, i32, vp, sz, f32 = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_float
    sig = {
        "nm_status_string": ([i32], ctypes.c_char_p),
        "nm_version": ([], i32),
        "nm_sizes": ([i64, i64, i32, i32, i32, vp, vp, vp], i32),
        "nm_mask": ([vp, i32, i64, i64, i64, i32, i32, vp, i64, vp], i32),
        "nm_mask_scored": ([vp, i32, vp, i64, i64, i64, i32, i32, vp, i64, vp], i32),
        "nm_mask_transposable": ([vp, i32, i64, i64, i64, i32, i32, vp, i64, vp], i32),
        "nm_mask_compress12": ([vp, i32, i64, i64, i64, vp, vp, vp], i32),
        "nm_compress12": ([vp, vp, i32, i64, i64, i64, i64, vp, vp, vp, vp], i32),
        "nm_decompress12": ([vp, vp, i32, i64, i64, vp, i64, vp], i32),
        "nm_mask_compress": ([vp, i32, i64, i64, i64, vp, vp, vp, vp], i32),
        "nm_compress": ([vp, vp, i32, i64, i64, i64, i64, vp, vp, vp, vp, vp], i32),
        "nm_compress_t": ([vp, vp, i32, i64, i64, i64, i64, vp, vp, vp, vp, vp], i32),
        "nm_decompress": ([vp, vp, i32, i64, i64, vp, i64, vp], i32),
        "nm_meta_to_sm100": ([vp, i64, i64, vp, vp], i32),
        "nm_meta_s8_image_bytes": ([i64, i64], sz),
        "nm_meta_to_sm100_s8": ([vp, i64, i64, vp, vp], i32),
        "nm_meta12_image_bytes": ([i64, i64], sz),
        "nm_meta12_to_sm100": ([vp, i64, i64, vp, vp], i32),
        "nm_spmm12": ([vp, vp, vp, i64, vp, i32, i64, i64, i64, i64, f32, f32, vp], i32),
        "nm_spmm12_test": ([vp, vp, vp, i64, vp, i32, i64, i64, i64, i64, f32, f32, i32, i32, vp], i32),
        "nm_spmm_workspace_bytes": ([i32, i64, i64, i64], sz),
        "nm_spmm": ([vp, vp, i32, vp, i64, vp, i32, i64, i64, i64, i64, f32, f32, vp, sz, vp], i32),
        "nm_spmm_noalloc": ([vp, vp, i32, vp, i64, vp, i32, i64, i64, i64, i64, f32, f32, vp], i32),
        "nm_spmm_test": ([vp, vp, i32, vp, i64, vp, i32, i64, i64, i64, i64, f32, f32, vp, sz,
                          i32, i32, i64, i64, i32, i32, vp], i32),
        "nm_srste_step": ([vp, vp, i32, i64, i64, i64, i32, i32, f32, vp, vp, vp, vp], i32),
        "nm_last_device_status": ([vp], i32),
        "nm_spmm_peers": ([vp, vp, i32, vp, i64, vp, i32, i64, i64, i64, i64, i64, f32, vp], i32),
        "nm_peer_signal": ([vp, i32, i32, ctypes.c_uint64, vp], i32),
        "nm_peer_wait": ([vp, i32, ctypes.c_uint64, i64, vp], i32),
        "nm_ipc_handle": ([vp, vp, vp], i32),
        "nm_ipc_open": ([vp, i64, vp], i32),
        "nm_ipc_close": ([vp, i64], i32),
    }
    for name, (args, res) in sig.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = res
    _LIB = lib
    return lib


def load() -> ctypes.CDLL:
    """Load libnm.so (raises if it is missing)."""
    return _lib()


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _ld(t: torch.Tensor) -> int:
    assert t.dim() == 2 and t.stride(1) == 1, "row-major 2-D tensor with unit column stride expected"
    return t.stride(0)


def _check(st: int, what: str):
    if st != 0:
        raise NMError(st, what)


def _dtype(t: torch.Tensor) -> int:
    if t.dtype not in _DT:
        raise NMError(4, "dtype %s" % t.dtype)
    return _DT[t.dtype]


# ---------------------------------------------------------------------------
def nm_version() -> int:
    return _lib().nm_version()


def nm_status_string(status: int) -> str:
    return _lib().nm_status_string(status).decode()


def nm_sizes(R: int, C: int, N: int, M: int, dtype: torch.dtype):
    """-> (values_bytes, meta_bytes, meta_sm100_bytes)."""
    v, m, s = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    _check(_lib().nm_sizes(R, C, N, M, _DT[dtype], ctypes.byref(v), ctypes.byref(m), ctypes.byref(s)), "nm_sizes")
    return v.value, m.value, s.value


def nm_mask(W: torch.Tensor, N: int, M: int, mask: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    R, C = W.shape
    if mask is None:
        mask = torch.empty((R, C), dtype=torch.uint8, device=W.device)
    _check(_lib().nm_mask(_ptr(W), _dtype(W), R, C, _ld(W), N, M, _ptr(mask), _ld(mask), _stream(stream)), "nm_mask")
    return mask


def nm_mask_scored(W: torch.Tensor, d: torch.Tensor, N: int, M: int, mask: torch.Tensor | None = None,
                   stream=None) -> torch.Tensor:
    """Saliency-scored N:M mask; d: fp32 device vector of length W.shape[1]."""
    R, C = W.shape
    if d.dtype != torch.float32 or d.numel() != C or not d.is_contiguous():
        raise NMError(2, "nm_mask_scored: d must be a contiguous float32 vector of length C")
    if mask is None:
        mask = torch.empty((R, C), dtype=torch.uint8, device=W.device)
    _check(_lib().nm_mask_scored(_ptr(W), _dtype(W), _ptr(d), R, C, _ld(W), N, M, _ptr(mask), _ld(mask),
                                 _stream(stream)), "nm_mask_scored")
    return mask


def nm_mask_transposable(W: torch.Tensor, N: int, M: int, mask: torch.Tensor | None = None,
                         stream=None) -> torch.Tensor:
    """Greedy transposable N:M mask over M x M blocks (at most N kept per row
    and per column of every block)."""
    R, C = W.shape
    if mask is None:
        mask = torch.empty((R, C), dtype=torch.uint8, device=W.device)
    _check(_lib().nm_mask_transposable(_ptr(W), _dtype(W), R, C, _ld(W), N, M, _ptr(mask), _ld(mask),
                                       _stream(stream)), "nm_mask_transposable")
    return mask


def alloc_compressed12(R: int, C: int, dtype: torch.dtype, device):
    """Output buffers of the 1:2 compressing calls: (values R x C/2, meta R x C/16)."""
    return (torch.empty((R, C // 2), dtype=dtype, device=device),
            torch.empty((R, C // 16), dtype=torch.uint8, device=device))


def nm_mask_compress12(W: torch.Tensor, values=None, meta=None, stream=None):
    """1:2 compression keeping the larger magnitude of each pair -> (values, meta)."""
    R, C = W.shape
    if values is None:
        values, meta = alloc_compressed12(R, C, W.dtype, W.device)
    _check(_lib().nm_mask_compress12(_ptr(W), _dtype(W), R, C, _ld(W), _ptr(values), _ptr(meta), _stream(stream)),
           "nm_mask_compress12")
    return values, meta


def nm_compress12(W: torch.Tensor, mask: torch.Tensor, values=None, meta=None,
                  invalid_pairs: torch.Tensor | None = None, stream=None):
    """1:2 compression under a mask -> (values, meta)."""
    R, C = W.shape
    if values is None:
        values, meta = alloc_compressed12(R, C, W.dtype, W.device)
    _check(_lib().nm_compress12(_ptr(W), _ptr(mask), _dtype(W), R, C, _ld(W), _ld(mask), _ptr(values), _ptr(meta),
                                _ptr(invalid_pairs), _stream(stream)), "nm_compress12")
    return values, meta


def nm_decompress12(values: torch.Tensor, meta: torch.Tensor, C: int, out: torch.Tensor | None = None,
                    stream=None) -> torch.Tensor:
    R = values.shape[0]
    if out is None:
        out = torch.empty((R, C), dtype=values.dtype, device=values.device)
    _check(_lib().nm_decompress12(_ptr(values), _ptr(meta), _dtype(values), R, C, _ptr(out), _ld(out),
                                  _stream(stream)), "nm_decompress12")
    return out


def alloc_compressed(R: int, C: int, dtype: torch.dtype, device, sm100: bool = True):
    """Output buffers of the compressing calls: (values, meta, meta_sm100 or None)."""
    _, mb, sb = nm_sizes(R, C, 2, 4, dtype)
    values = torch.empty((R, C // 2), dtype=dtype, device=device)
    meta = torch.empty((R, C // 8), dtype=torch.uint8, device=device)
    img = torch.empty((sb,), dtype=torch.uint8, device=device) if sm100 else None
    return values, meta, img


def nm_mask_compress(W: torch.Tensor, values=None, meta=None, meta_sm100=None, sm100: bool = True, stream=None):
    """-> (values, meta, meta_sm100 or None)."""
    R, C = W.shape
    if values is None:
        values, meta, meta_sm100 = alloc_compressed(R, C, W.dtype, W.device, sm100)
    _check(_lib().nm_mask_compress(_ptr(W), _dtype(W), R, C, _ld(W), _ptr(values), _ptr(meta), _ptr(meta_sm100),
                                   _stream(stream)), "nm_mask_compress")
    return values, meta, meta_sm100


def nm_compress(W: torch.Tensor, mask: torch.Tensor, values=None, meta=None, meta_sm100=None, sm100: bool = True,
                invalid_groups: torch.Tensor | None = None, stream=None):
    """-> (values, meta, meta_sm100 or None); invalid_groups: optional int32 device counter."""
    R, C = W.shape
    if values is None:
        values, meta, meta_sm100 = alloc_compressed(R, C, W.dtype, W.device, sm100)
    _check(_lib().nm_compress(_ptr(W), _ptr(mask), _dtype(W), R, C, _ld(W), _ld(mask), _ptr(values), _ptr(meta),
                              _ptr(meta_sm100), _ptr(invalid_groups), _stream(stream)), "nm_compress")
    return values, meta, meta_sm100


def nm_compress_t(W: torch.Tensor, mask: torch.Tensor, values=None, meta=None, meta_sm100=None,
                  sm100: bool = True, invalid_groups: torch.Tensor | None = None, stream=None):
    """Compressed W^T (C x R, groups along R) under mask^T -> (values_t, meta_t, meta_t_sm100 or None)."""
    R, C = W.shape
    if values is None:
        values, meta, meta_sm100 = alloc_compressed(C, R, W.dtype, W.device, sm100)
    _check(_lib().nm_compress_t(_ptr(W), _ptr(mask), _dtype(W), R, C, _ld(W), _ld(mask), _ptr(values), _ptr(meta),
                                _ptr(meta_sm100), _ptr(invalid_groups), _stream(stream)), "nm_compress_t")
    return values, meta, meta_sm100


def nm_decompress(values: torch.Tensor, meta: torch.Tensor, C: int, out: torch.Tensor | None = None,
                  stream=None) -> torch.Tensor:
    R = values.shape[0]
    if out is None:
        out = torch.empty((R, C), dtype=values.dtype, device=values.device)
    _check(_lib().nm_decompress(_ptr(values), _ptr(meta), _dtype(values), R, C, _ptr(out), _ld(out),
                                _stream(stream)), "nm_decompress")
    return out


def nm_meta_to_sm100(meta: torch.Tensor, R: int, C: int, out: torch.Tensor | None = None, stream=None):
    if out is None:
        out = torch.empty((nm_sizes(R, C, 2, 4, torch.bfloat16)[2],), dtype=torch.uint8, device=meta.device)
    _check(_lib().nm_meta_to_sm100(_ptr(meta), R, C, _ptr(out), _stream(stream)), "nm_meta_to_sm100")
    return out


def nm_meta_s8_image_bytes(R: int, C: int) -> int:
    return int(_lib().nm_meta_s8_image_bytes(R, C))


def nm_meta12_image_bytes(R: int, C: int) -> int:
    return int(_lib().nm_meta12_image_bytes(R, C))


def nm_meta_to_sm100_s8(meta: torch.Tensor, R: int, C: int, out: torch.Tensor | None = None, stream=None):
    """Canonical 2:4 metadata of an int8 matrix -> the image the int8 product reads."""
    if out is None:
        out = torch.empty((nm_meta_s8_image_bytes(R, C),), dtype=torch.uint8, device=meta.device)
    _check(_lib().nm_meta_to_sm100_s8(_ptr(meta), R, C, _ptr(out), _stream(stream)), "nm_meta_to_sm100_s8")
    return out


def nm_meta12_to_sm100(meta: torch.Tensor, R: int, C: int, out: torch.Tensor | None = None, stream=None):
    """Canonical 1:2 metadata -> the image the TF32 1:2 product reads."""
    if out is None:
        out = torch.empty((nm_meta12_image_bytes(R, C),), dtype=torch.uint8, device=meta.device)
    _check(_lib().nm_meta12_to_sm100(_ptr(meta), R, C, _ptr(out), _stream(stream)), "nm_meta12_to_sm100")
    return out


def nm_spmm_workspace_bytes(ab_dtype: torch.dtype, R: int, K: int, T: int) -> int:
    return int(_lib().nm_spmm_workspace_bytes(_DT[ab_dtype], R, K, T))


def nm_spmm(values: torch.Tensor, meta_sm100: torch.Tensor, X: torch.Tensor, Y: torch.Tensor | None = None,
            y_dtype: torch.dtype = torch.bfloat16, alpha: float = 1.0, beta: float = 0.0,
            workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Y = alpha * (W (.) mask) X + beta * Y from the compressed W (values, meta_sm100).
    int8 values and X take the .kind::i8 image (nm_meta_to_sm100_s8) and may
    write torch.int32 (the exact sum)."""
    R, Kh = values.shape
    K = 2 * Kh
    Kx, T = X.shape
    assert Kx == K, "X must be K x T"
    if Y is None:
        Y = torch.empty((R, T), dtype=y_dtype, device=values.device)
    need = nm_spmm_workspace_bytes(values.dtype, R, K, T)
    if need and workspace is None:
        workspace = torch.empty((need,), dtype=torch.uint8, device=values.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(_lib().nm_spmm(_ptr(values), _ptr(meta_sm100), _dtype(values), _ptr(X), _ld(X), _ptr(Y), _dtype(Y),
                          _ld(Y), R, K, T, float(alpha), float(beta), _ptr(workspace), ws_bytes, _stream(stream)),
           "nm_spmm")
    return Y


# nm_spmm_test's kernel choices (include/nm_testing.h)
SPMM_KERNELS = {"default": 0, "pair256": 1, "pair192": 2, "pair128": 3, "single256": 4, "single128": 5,
                "single64": 6, "single64x2": 7, "single32x2": 8, "single16x2": 9}


def nm_spmm_test(values: torch.Tensor, meta_sm100: torch.Tensor, X: torch.Tensor, Y: torch.Tensor | None = None,
                 y_dtype: torch.dtype = torch.bfloat16, alpha: float = 1.0, beta: float = 0.0,
                 workspace: torch.Tensor | None = None, kernel: str = "default", tail_split: bool = True,
                 wait_limit_ns: int = 0, skip_step: int = -1, raster_group: int = 0, raster_m_inner: int = 0,
                 stream=None) -> torch.Tensor:
    """nm_spmm with the test hooks of include/nm_testing.h: a forced tile
    configuration, the half-width last wave on or off, a shorter limit for the
    kernel's bounded waits, and a pipeline step the producer never fills."""
    R, Kh = values.shape
    K = 2 * Kh
    Kx, T = X.shape
    assert Kx == K, "X must be K x T"
    if Y is None:
        Y = torch.empty((R, T), dtype=y_dtype, device=values.device)
    need = nm_spmm_workspace_bytes(values.dtype, R, K, T)
    if need and workspace is None:
        workspace = torch.empty((need,), dtype=torch.uint8, device=values.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(_lib().nm_spmm_test(_ptr(values), _ptr(meta_sm100), _dtype(values), _ptr(X), _ld(X), _ptr(Y), _dtype(Y),
                               _ld(Y), R, K, T, float(alpha), float(beta), _ptr(workspace), ws_bytes,
                               SPMM_KERNELS[kernel], 1 if tail_split else 0, int(wait_limit_ns), int(skip_step),
                               int(raster_group), int(raster_m_inner), _stream(stream)), "nm_spmm_test")
    return Y


def _spmm12_args(values, meta12_sm100, X, Y, y_dtype, alpha, beta):
    R, Kh = values.shape
    K = 2 * Kh
    Kx, T = X.shape
    assert Kx == K, "X must be K x T"
    if Y is None:
        Y = torch.empty((R, T), dtype=y_dtype, device=values.device)
    return Y, (_ptr(values), _ptr(meta12_sm100), _ptr(X), _ld(X), _ptr(Y), _dtype(Y), _ld(Y), R, K, T,
               float(alpha), float(beta))


def nm_spmm12(values: torch.Tensor, meta12_sm100: torch.Tensor, X: torch.Tensor, Y: torch.Tensor | None = None,
              y_dtype: torch.dtype = torch.float32, alpha: float = 1.0, beta: float = 0.0, stream=None) -> torch.Tensor:
    """Y = alpha * (W (.) mask) X + beta * Y for a 1:2-sparse fp32 W (values R x K/2,
    the nm_meta12_to_sm100 image) on the TF32 sparse tensor cores."""
    Y, args = _spmm12_args(values, meta12_sm100, X, Y, y_dtype, alpha, beta)
    _check(_lib().nm_spmm12(*args, _stream(stream)), "nm_spmm12")
    return Y


def nm_spmm12_test(values: torch.Tensor, meta12_sm100: torch.Tensor, X: torch.Tensor, Y: torch.Tensor | None = None,
                   y_dtype: torch.dtype = torch.float32, alpha: float = 1.0, beta: float = 0.0,
                   kernel: str = "default", tail_split: bool = True, stream=None) -> torch.Tensor:
    """nm_spmm12 with a forced tile configuration and the half-width last wave on or off."""
    Y, args = _spmm12_args(values, meta12_sm100, X, Y, y_dtype, alpha, beta)
    _check(_lib().nm_spmm12_test(*args, SPMM_KERNELS[kernel], 1 if tail_split else 0, _stream(stream)),
           "nm_spmm12_test")
    return Y


def nm_spmm_noalloc(values: torch.Tensor, meta_sm100: torch.Tensor, X: torch.Tensor, Y: torch.Tensor | None = None,
                    y_dtype: torch.dtype = torch.bfloat16, alpha: float = 1.0, beta: float = 0.0,
                    stream=None) -> torch.Tensor:
    """nm_spmm without a workspace: fp32 inputs are staged in the library's fixed device array."""
    R, Kh = values.shape
    K = 2 * Kh
    Kx, T = X.shape
    assert Kx == K, "X must be K x T"
    if Y is None:
        Y = torch.empty((R, T), dtype=y_dtype, device=values.device)
    _check(_lib().nm_spmm_noalloc(_ptr(values), _ptr(meta_sm100), _dtype(values), _ptr(X), _ld(X), _ptr(Y),
                                  _dtype(Y), _ld(Y), R, K, T, float(alpha), float(beta), _stream(stream)),
           "nm_spmm_noalloc")
    return Y


# ---------------------------------------------------------------------------
# Row-split product over several GPUs (include/nm.h: nm_spmm_peers,
# nm_peer_signal, nm_peer_wait, nm_ipc_*).  Destination buffers and flag
# arrays are given as torch tensors (this process's memory) or as integer
# device addresses (another process's memory, mapped with nm_ipc_open).
NM_IPC_HANDLE_BYTES = 64
NM_MAX_PEERS = 8


def _addr(x) -> int:
    return x.data_ptr() if isinstance(x, torch.Tensor) else int(x)


def _ptr_array(xs):
    return (ctypes.c_void_p * len(xs))(*[_addr(x) for x in xs])


def nm_spmm_peers(values: torch.Tensor, meta_sm100: torch.Tensor, X: torch.Tensor, peer_Y, row0: int, ldy: int,
                  alpha: float = 1.0, stream=None) -> None:
    """(W (.) mask) X * alpha in bf16, written into rows [row0, row0 + R) of
    every buffer of peer_Y (leading dim ldy)."""
    R, Kh = values.shape
    K = 2 * Kh
    Kx, T = X.shape
    assert Kx == K, "X must be K x T"
    ys = list(peer_Y)
    _check(_lib().nm_spmm_peers(_ptr(values), _ptr(meta_sm100), _dtype(values), _ptr(X), _ld(X), _ptr_array(ys),
                                len(ys), int(row0), int(ldy), R, K, T, float(alpha), _stream(stream)),
           "nm_spmm_peers")


def nm_peer_signal(peer_flags, rank: int, epoch: int, stream=None) -> None:
    """Store epoch into slot `rank` of every flag array of peer_flags."""
    fs = list(peer_flags)
    _check(_lib().nm_peer_signal(_ptr_array(fs), len(fs), int(rank), int(epoch), _stream(stream)), "nm_peer_signal")


def nm_peer_wait(flags: torch.Tensor, epoch: int, timeout_ns: int = 2_000_000_000, stream=None) -> None:
    """Make the stream wait (bounded) until every slot of flags holds >= epoch."""
    assert flags.dtype in (torch.int64, torch.uint64) and flags.dim() == 1
    _check(_lib().nm_peer_wait(_ptr(flags), flags.numel(), int(epoch), int(timeout_ns), _stream(stream)),
           "nm_peer_wait")


def nm_ipc_handle(t: torch.Tensor):
    """-> (64-byte handle, byte offset of t's first element in its allocation)."""
    h = ctypes.create_string_buffer(NM_IPC_HANDLE_BYTES)
    off = ctypes.c_int64()
    _check(_lib().nm_ipc_handle(_ptr(t), h, ctypes.byref(off)), "nm_ipc_handle")
    return h.raw, off.value


def nm_ipc_open(handle: bytes, offset: int) -> int:
    """Map another process's buffer; -> its device address in this process."""
    assert len(handle) == NM_IPC_HANDLE_BYTES
    p = ctypes.c_void_p()
    _check(_lib().nm_ipc_open(ctypes.c_char_p(handle), int(offset), ctypes.byref(p)), "nm_ipc_open")
    return int(p.value)


def nm_ipc_close(addr: int, offset: int) -> None:
    _check(_lib().nm_ipc_close(ctypes.c_void_p(addr), int(offset)), "nm_ipc_close")


def nm_last_device_status(stream=None) -> int:
    return int(_lib().nm_last_device_status(_stream(stream)))


def nm_srste_step(W: torch.Tensor, grad: torch.Tensor, N: int = 2, M: int = 4, decay: float = 0.0002,
                  W_sparse: torch.Tensor | None = None, grad_out: torch.Tensor | None = None,
                  mask: torch.Tensor | None = None, want_mask: bool = False, stream=None):
    """SR-STE step -> (W_sparse, grad_out, mask or None).  W, grad and the outputs
    share one leading dimension (that of W)."""
    R, C = W.shape
    ld = _ld(W)
    assert _ld(grad) == ld
    if W_sparse is None:
        W_sparse = torch.empty_strided((R, C), (ld, 1), dtype=W.dtype, device=W.device)
    if grad_out is None:
        grad_out = torch.empty_strided((R, C), (ld, 1), dtype=W.dtype, device=W.device)
    if mask is None and want_mask:
        mask = torch.empty_strided((R, C), (ld, 1), dtype=torch.uint8, device=W.device)
    _check(_lib().nm_srste_step(_ptr(W), _ptr(grad), _dtype(W), R, C, ld, N, M, float(decay), _ptr(W_sparse),
                                _ptr(grad_out), _ptr(mask), _stream(stream)), "nm_srste_step")
    return W_sparse, grad_out, mask
