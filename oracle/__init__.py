"""CPU oracle for N:M structured sparsity -- TEST INFRASTRUCTURE ONLY.

Thin ctypes binding over ``nm_oracle.c`` (plain C, fp64 where there is any
floating-point arithmetic).  Only the test suite, ``__graft_entry__.smoke``
and the CPU-baseline leg of ``bench.py`` may import this package; the
product library never does, and this package never imports the product.

What each function follows (page title and section):

* ``mask_rank`` -- "SR-STE sparse training", SR-STE forward (argsort of
  |w| inside each group of M, the M-N smallest zeroed) and "Accelerating
  Sparse Deep Neural Networks" review, Step-2 (drop the smallest of each
  group of 4).  Stable tie rule: equal |w| keeps the lower index.
* ``mask_exhaustive`` -- "SR-STE sparse training", the Apex static-mask
  listing (mn_1d_best / m4n2_1d): best of all C(M,N) patterns by kept L1
  sum, with exact sums and lexicographic pattern order.
* ``compress24`` / ``decompress24`` -- "Accelerating Sparse Deep Neural
  Networks" review, "Benefits of 2:4 sparsity": R*C/2 values, 2-bit index
  per kept value, two values stored even for emptier groups.
* ``meta_sm100`` -- PTX ISA, tcgen05 sparse-matrix metadata layout
  (the pages give none).
* ``spmm`` -- same review, "Structured sparse GEMM on tensor cores":
  sparse x dense = dense; computed in double.
* ``spmm12`` -- the 1:2 (sparse TF32) product of the same section, in double.
* ``meta_sm100_s8`` / ``meta12_sm100`` -- PTX ISA, tcgen05 sparse metadata of
  the .kind::i8 and .kind::tf32 MMAs.
* ``srste`` -- "SR-STE sparse training", SR-STE forward / backward:
  masked weight and grad + decay * (1 - mask) * w.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "nm_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

F32, BF16, F16, S8 = 0, 1, 2, 3
_OK, _BAD_ARG, _NONFINITE, _BAD_MASK = 0, 1, 2, 3

_lib = None


def build(force: bool = False) -> str:
    """Compile nm_oracle.c into liboracle.so next to it (gcc, -O2)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp.%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fPIC", "-shared", "-pthread",
                               "-Wall", "-Wextra", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is not None:
        return _lib
    lib = ctypes.CDLL(build())
    i64, i32, vp, dbl = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p, ctypes.c_double
    lib.oracle_decode.argtypes = [ctypes.c_uint32, i32]
    lib.oracle_decode.restype = dbl
    lib.oracle_encode.argtypes = [dbl, i32]
    lib.oracle_encode.restype = ctypes.c_uint32
    lib.oracle_mag.argtypes = [ctypes.c_uint32, i32]
    lib.oracle_mag.restype = ctypes.c_uint32
    for name in ("oracle_mask_rank", "oracle_mask_exhaustive"):
        f = getattr(lib, name)
        f.argtypes = [vp, i32, i64, i64, i64, i32, i32, vp, i64]
        f.restype = i32
    lib.oracle_compress12.argtypes = [vp, vp, i32, i64, i64, vp, vp]
    lib.oracle_compress12.restype = i32
    lib.oracle_decompress12.argtypes = [vp, vp, i32, i64, i64, vp]
    lib.oracle_decompress12.restype = i32
    lib.oracle_compress24.argtypes = [vp, vp, i32, i64, i64, vp, vp]
    lib.oracle_compress24.restype = i32
    lib.oracle_decompress24.argtypes = [vp, vp, i32, i64, i64, vp]
    lib.oracle_decompress24.restype = i32
    lib.oracle_meta_sm100_bytes.argtypes = [i64, i64]
    lib.oracle_meta_sm100_bytes.restype = i64
    lib.oracle_meta_sm100.argtypes = [vp, i64, i64, vp]
    lib.oracle_meta_sm100.restype = i32
    lib.oracle_spmm.argtypes = [vp, vp, i32, vp, i64, vp, i32, i64, i64, dbl, dbl, vp, i64, i32, vp]
    lib.oracle_spmm.restype = i32
    lib.oracle_spmm12.argtypes = [vp, vp, i32, vp, i64, vp, i32, i64, i64, dbl, dbl, vp, i64, i32, vp]
    lib.oracle_spmm12.restype = i32
    for name in ("oracle_meta_sm100_s8", "oracle_meta12_sm100"):
        getattr(lib, name + "_bytes").argtypes = [i64, i64]
        getattr(lib, name + "_bytes").restype = i64
        getattr(lib, name).argtypes = [vp, i64, i64, vp]
        getattr(lib, name).restype = i32
    lib.oracle_rows_parallel.argtypes = [i32, vp, i32, i64, i64, i32, i32, vp, vp, vp, i32]
    lib.oracle_rows_parallel.restype = i32
    lib.oracle_mask_transposable.argtypes = [vp, i32, i64, i64, i64, i32, i32, vp, i64]
    lib.oracle_mask_transposable.restype = i32
    lib.oracle_mask_scored.argtypes = [vp, i32, vp, i64, i64, i64, i32, i32, vp, i64]
    lib.oracle_mask_scored.restype = i32
    lib.oracle_srste.argtypes = [vp, vp, i32, i64, i64, i32, i32, ctypes.c_float, vp, vp, vp]
    lib.oracle_srste.restype = i32
    _lib = lib
    return lib


# ---------------------------------------------------------------------------
# helpers: the oracle works on raw bit patterns; arrays are numpy
#   f32  -> np.float32 (or its uint32 view)
#   bf16 -> np.uint16 bit patterns
#   f16  -> np.float16 (or its uint16 view)
# ---------------------------------------------------------------------------
def dtype_code(a: np.ndarray, hint: int | None = None) -> int:
    if hint is not None:
        return hint
    if a.dtype in (np.float32, np.uint32):
        return F32
    if a.dtype == np.float16:
        return F16
    if a.dtype in (np.int8, np.uint8):
        return S8
    raise ValueError("pass dtype= for bf16 bit patterns (np.uint16)")


def _bits(a: np.ndarray, code: int) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if code == S8:
        return a.view(np.uint8)
    return a.view(np.uint32) if code == F32 else a.view(np.uint16)


def _check(st: int, what: str):
    if st != _OK:
        raise ValueError("%s failed with oracle status %d" % (what, st))


def decode(bits: int, code: int) -> float:
    return _load().oracle_decode(int(bits), code)


def encode(x: float, code: int) -> int:
    """Round-to-nearest-even encode of a double into the format `code`."""
    return int(_load().oracle_encode(float(x), code))


def encode_array(x: np.ndarray, code: int) -> np.ndarray:
    lib = _load()
    flat = np.asarray(x, dtype=np.float64).ravel()
    out = np.empty(flat.shape, dtype=np.uint32 if code == F32 else np.uint16)
    for i, v in enumerate(flat):
        out[i] = lib.oracle_encode(float(v), code)
    return out.reshape(np.shape(x))


def decode_array(bits: np.ndarray, code: int) -> np.ndarray:
    """Exact decode of bit patterns to float64 (elementwise oracle_decode)."""
    lib = _load()
    b = np.asarray(bits)
    if code != F32:
        table = np.array([lib.oracle_decode(i, code) for i in range(65536)], dtype=np.float64)
        return table[b.astype(np.int64)]
    flat = b.astype(np.uint32).ravel()
    out = np.array([lib.oracle_decode(int(v), code) for v in flat], dtype=np.float64)
    return out.reshape(b.shape)


def mask_rank(W: np.ndarray, N: int, M: int, dtype: int | None = None) -> np.ndarray:
    code = dtype_code(W, dtype)
    Wb = _bits(W, code)
    R, C = Wb.shape
    mask = np.zeros((R, C), dtype=np.uint8)
    _check(_load().oracle_mask_rank(Wb.ctypes.data, code, R, C, C, N, M, mask.ctypes.data, C),
           "mask_rank")
    return mask


def mask_scored(W: np.ndarray, d: np.ndarray, N: int, M: int, dtype: int | None = None) -> np.ndarray:
    """Saliency-scored N:M mask: keep the N largest binary32 scores w^2 / d^2
    of each group ("sparsegpt.py", fasterprune, semi-structured branch)."""
    code = dtype_code(W, dtype)
    Wb = _bits(W, code)
    R, C = Wb.shape
    dv = np.ascontiguousarray(d, dtype=np.float32).ravel()
    assert dv.size == C
    mask = np.zeros((R, C), dtype=np.uint8)
    _check(_load().oracle_mask_scored(Wb.ctypes.data, code, dv.ctypes.data, R, C, C, N, M, mask.ctypes.data, C),
           "mask_scored")
    return mask


def mask_transposable(W: np.ndarray, N: int, M: int, dtype: int | None = None) -> np.ndarray:
    """Greedy transposable N:M mask over MxM blocks (at most N kept per row
    and per column of every block), as described in the oracle source."""
    code = dtype_code(W, dtype)
    Wb = _bits(W, code)
    R, C = Wb.shape
    mask = np.zeros((R, C), dtype=np.uint8)
    _check(_load().oracle_mask_transposable(Wb.ctypes.data, code, R, C, C, N, M, mask.ctypes.data, C),
           "mask_transposable")
    return mask


def mask_exhaustive(W: np.ndarray, N: int, M: int, dtype: int | None = None) -> np.ndarray:
    code = dtype_code(W, dtype)
    Wb = _bits(W, code)
    R, C = Wb.shape
    mask = np.zeros((R, C), dtype=np.uint8)
    _check(_load().oracle_mask_exhaustive(Wb.ctypes.data, code, R, C, C, N, M, mask.ctypes.data, C),
           "mask_exhaustive")
    return mask


def compress24(W: np.ndarray, mask: np.ndarray, dtype: int | None = None):
    """-> (values R x C/2 same bit type as W, meta R x C/8 uint8)."""
    code = dtype_code(W, dtype)
    Wb = _bits(W, code)
    R, C = Wb.shape
    m = np.ascontiguousarray(mask, dtype=np.uint8)
    values = np.zeros((R, C // 2), dtype=Wb.dtype)
    meta = np.zeros((R, C // 8), dtype=np.uint8)
    _check(_load().oracle_compress24(Wb.ctypes.data, m.ctypes.data, code, R, C,
                                     values.ctypes.data, meta.ctypes.data), "compress24")
    return values.view(W.dtype) if W.dtype != np.uint16 else values, meta


def decompress24(values: np.ndarray, meta: np.ndarray, C: int, dtype: int | None = None) -> np.ndarray:
    code = dtype_code(values, dtype)
    vb = _bits(values, code)
    R = vb.shape[0]
    out = np.zeros((R, C), dtype=vb.dtype)
    mt = np.ascontiguousarray(meta, dtype=np.uint8)
    _check(_load().oracle_decompress24(vb.ctypes.data, mt.ctypes.data, code, R, C, out.ctypes.data),
           "decompress24")
    return out.view(values.dtype) if values.dtype != np.uint16 else out


def compress12(W: np.ndarray, mask: np.ndarray, dtype: int | None = None):
    """1:2 compression -> (values R x C/2 same bit type as W, meta R x C/16 uint8:
    bit p%8 of byte p/8 is the kept index of pair p)."""
    code = dtype_code(W, dtype)
    Wb = _bits(W, code)
    R, C = Wb.shape
    m = np.ascontiguousarray(mask, dtype=np.uint8)
    values = np.zeros((R, C // 2), dtype=Wb.dtype)
    meta = np.zeros((R, C // 16), dtype=np.uint8)
    _check(_load().oracle_compress12(Wb.ctypes.data, m.ctypes.data, code, R, C,
                                     values.ctypes.data, meta.ctypes.data), "compress12")
    return values.view(W.dtype) if W.dtype != np.uint16 else values, meta


def decompress12(values: np.ndarray, meta: np.ndarray, C: int, dtype: int | None = None) -> np.ndarray:
    code = dtype_code(values, dtype)
    vb = _bits(values, code)
    R = vb.shape[0]
    out = np.zeros((R, C), dtype=vb.dtype)
    mt = np.ascontiguousarray(meta, dtype=np.uint8)
    _check(_load().oracle_decompress12(vb.ctypes.data, mt.ctypes.data, code, R, C, out.ctypes.data),
           "decompress12")
    return out.view(values.dtype) if values.dtype != np.uint16 else out


def meta_sm100_bytes(R: int, C: int) -> int:
    return int(_load().oracle_meta_sm100_bytes(R, C))


def meta_sm100(meta: np.ndarray, R: int, C: int) -> np.ndarray:
    mt = np.ascontiguousarray(meta, dtype=np.uint8)
    out = np.zeros(meta_sm100_bytes(R, C), dtype=np.uint8)
    _check(_load().oracle_meta_sm100(mt.ctypes.data, R, C, out.ctypes.data), "meta_sm100")
    return out


def meta_sm100_s8(meta: np.ndarray, R: int, C: int) -> np.ndarray:
    """Tensor-core metadata image of a 2:4 int8 matrix (.kind::i8 layout)."""
    lib = _load()
    mt = np.ascontiguousarray(meta, dtype=np.uint8)
    out = np.zeros(int(lib.oracle_meta_sm100_s8_bytes(R, C)), dtype=np.uint8)
    _check(lib.oracle_meta_sm100_s8(mt.ctypes.data, R, C, out.ctypes.data), "meta_sm100_s8")
    return out


def meta12_sm100(meta: np.ndarray, R: int, C: int) -> np.ndarray:
    """Tensor-core metadata image of a 1:2 fp32 matrix (.kind::tf32 layout)."""
    lib = _load()
    mt = np.ascontiguousarray(meta, dtype=np.uint8)
    out = np.zeros(int(lib.oracle_meta12_sm100_bytes(R, C)), dtype=np.uint8)
    _check(lib.oracle_meta12_sm100(mt.ctypes.data, R, C, out.ctypes.data), "meta12_sm100")
    return out


def spmm(values: np.ndarray, meta: np.ndarray, X: np.ndarray, ab_dtype: int,
         alpha: float = 1.0, beta: float = 0.0, Y_in: np.ndarray | None = None,
         y_dtype: int = F32, rows: np.ndarray | None = None, threads: int | None = None) -> np.ndarray:
    """fp64 Y = alpha * (W (.) mask) X + beta * Y_in, from the compressed 2:4 form
    (int8 inputs summed exactly in int64).

    values: R x K/2, meta: R x K/8 (canonical), X: K x T; returns float64
    (len(rows) or R) x T."""
    return _spmm("oracle_spmm", 8, values, meta, X, ab_dtype, alpha, beta, Y_in, y_dtype, rows, threads)


def spmm12(values: np.ndarray, meta: np.ndarray, X: np.ndarray, ab_dtype: int = F32,
           alpha: float = 1.0, beta: float = 0.0, Y_in: np.ndarray | None = None,
           y_dtype: int = F32, rows: np.ndarray | None = None, threads: int | None = None) -> np.ndarray:
    """fp64 Y = alpha * (W (.) mask) X + beta * Y_in, from the compressed 1:2 form.

    values: R x K/2, meta: R x K/16 (one index bit per pair), X: K x T."""
    return _spmm("oracle_spmm12", 16, values, meta, X, ab_dtype, alpha, beta, Y_in, y_dtype, rows, threads)


def _spmm(fn, meta_div, values, meta, X, ab_dtype, alpha, beta, Y_in, y_dtype, rows, threads):
    vb = _bits(values, ab_dtype)
    xb = _bits(X, ab_dtype)
    R, Kh = vb.shape
    K = 2 * Kh
    T = xb.shape[1]
    assert xb.shape[0] == K
    mt = np.ascontiguousarray(meta, dtype=np.uint8)
    ybits = None
    if beta != 0.0:
        assert Y_in is not None
        ybits = _bits(Y_in, y_dtype)
    rows_arr = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    nrows = R if rows_arr is None else len(rows_arr)
    out = np.zeros((nrows, T), dtype=np.float64)
    nthr = threads or os.cpu_count() or 1
    assert mt.size == R * K // meta_div, "metadata size does not match the values"
    _check(getattr(_load(), fn)(vb.ctypes.data, mt.ctypes.data, ab_dtype, xb.ctypes.data, T,
                                None if ybits is None else ybits.ctypes.data, y_dtype, R, K,
                                float(alpha), float(beta),
                                None if rows_arr is None else rows_arr.ctypes.data, nrows,
                                int(nthr), out.ctypes.data), fn)
    return out


def rows_parallel(what: int, W: np.ndarray, N: int, M: int, dtype: int, threads: int):
    """Multi-threaded mask (what=0) or 2:4 mask+compress (what=1) over rows:
    the single-row oracle run on row ranges in parallel, for the CPU baseline
    and for the whole-matrix parity tests.  Mode 1 also fills the mask."""
    Wb = _bits(W, dtype)
    R, C = Wb.shape
    mask = np.zeros((R, C), dtype=np.uint8)
    values = np.zeros((R, C // 2), dtype=Wb.dtype)
    meta = np.zeros((R, C // 8), dtype=np.uint8)
    _check(_load().oracle_rows_parallel(what, Wb.ctypes.data, dtype, R, C, N, M, mask.ctypes.data,
                                        values.ctypes.data, meta.ctypes.data, int(threads)),
           "rows_parallel")
    return mask, values, meta


def srste(W: np.ndarray, grad: np.ndarray, N: int, M: int, decay: float, dtype: int | None = None):
    """SR-STE step -> (W_sparse, grad_out, mask); arrays of W's bit type."""
    code = dtype_code(W, dtype)
    Wb, Gb = _bits(W, code), _bits(grad, code)
    R, C = Wb.shape
    ws = np.zeros_like(Wb)
    go = np.zeros_like(Wb)
    mask = np.zeros((R, C), dtype=np.uint8)
    _check(_load().oracle_srste(Wb.ctypes.data, Gb.ctypes.data, code, R, C, N, M, float(decay),
                                ws.ctypes.data, go.ctypes.data, mask.ctypes.data), "srste")
    if W.dtype != np.uint16:
        return ws.view(W.dtype), go.view(W.dtype), mask
    return ws, go, mask
