"""The C-ABI library: it builds, loads, exports every symbol the headers in
include/ declare, and validates arguments on the host (no GPU needed: every
case here fails validation before any CUDA call)."""
import ctypes
import os
import re

import pytest

import structured_sparsity_prune_b200 as nm
from structured_sparsity_prune_b200 import build as nm_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", h) for h in sorted(os.listdir(os.path.join(ROOT, "include")))
           if h.endswith(".h")]


def _declared():
    text = ""
    for h in HEADERS:
        with open(h) as f:
            text += f.read()
    return sorted(set(re.findall(r"NM_API\s+[\w\s\*]*?\b(nm_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    nm_build.build()
    return nm.load()


def test_header_declares_the_hot_path():
    names = _declared()
    for want in ["nm_mask", "nm_mask_compress", "nm_compress", "nm_decompress", "nm_meta_to_sm100", "nm_spmm",
                 "nm_sizes", "nm_status_string", "nm_spmm_workspace_bytes", "nm_last_device_status"]:
        assert want in names


def test_every_declared_symbol_is_exported(lib):
    for name in _declared():
        assert hasattr(lib, name), name


def test_status_strings(lib):
    for code, name in enumerate(nm.STATUS):
        assert nm.nm_status_string(code).startswith(name)
    assert "unknown" in nm.nm_status_string(99)


def test_version(lib):
    assert nm.nm_version() >= 10000


def test_sizes_match_the_pages_counts(lib):
    import torch
    # 2:4: R*C/2 values and R*C/2 2-bit fields; image padded to 128 x 128 blocks
    v, m, s = nm.nm_sizes(4096, 4096, 2, 4, torch.bfloat16)
    assert v == 4096 * 4096 // 2 * 2 and m == 4096 * 4096 // 2 * 2 // 8 and s == 4096 * 4096 // 8
    v, m, s = nm.nm_sizes(200, 72, 2, 4, torch.float32)
    assert v == 200 * 36 * 4 and m == 200 * 9 and s == 256 * 128 // 8
    # 36 of 64 bits per four 16-bit weights
    v16, m16, _ = nm.nm_sizes(8, 64, 2, 4, torch.float16)
    assert (v16 + m16) * 8 * 64 == 8 * 64 * 16 * 36
    # other N:M: values only
    v, m, s = nm.nm_sizes(10, 80, 2, 8, torch.float32)
    assert v == 10 * 20 * 4 and m == 0 and s == 0


@pytest.mark.parametrize("N,M,code", [(0, 4, 5), (4, 4, 5), (2, 9, 5), (2, 1, 5)])
def test_sizes_bad_nm(lib, N, M, code):
    import torch
    with pytest.raises(nm.NMError) as e:
        nm.nm_sizes(8, 64, N, M, torch.float32)
    assert e.value.status == code


def test_host_validation_before_any_launch(lib):
    fake = ctypes.c_void_p(0x10000)          # never dereferenced: validation fails first
    odd = ctypes.c_void_p(0x10008)
    s = ctypes.c_void_p(0)
    L = lib
    assert L.nm_mask(fake, 7, 4, 64, 64, 2, 4, fake, 64, s) == 4          # bad dtype
    assert L.nm_mask(fake, 0, 4, 64, 64, 4, 4, fake, 64, s) == 5          # N == M
    assert L.nm_mask(fake, 0, 4, 66, 66, 2, 4, fake, 66, s) == 2          # C % M
    assert L.nm_mask(fake, 0, 4, 64, 32, 2, 4, fake, 64, s) == 2          # ldw < C
    assert L.nm_mask(None, 0, 4, 64, 64, 2, 4, fake, 64, s) == 1          # NULL
    assert L.nm_mask(odd, 0, 4, 64, 64, 2, 4, fake, 64, s) == 3           # misaligned
    assert L.nm_mask(fake, 1, 4, 64, 68, 2, 4, fake, 64, s) == 3          # ldw*2 not 16B
    assert L.nm_mask(fake, 0, 0, 64, 64, 2, 4, fake, 64, s) == 0          # R == 0: no-op
    assert L.nm_mask_compress(fake, 1, 4, 12, 12, fake, fake, None, s) == 2   # C % 8
    assert L.nm_mask_compress(fake, 1, 4, 64, 64, None, fake, None, s) == 1
    assert L.nm_mask_compress(fake, 1, 4, 64, 64, fake, odd, None, s) == 3
    assert L.nm_compress(fake, fake, 1, 4, 64, 64, 32, fake, fake, None, None, s) == 2  # ldm < C
    assert L.nm_compress(fake, None, 1, 4, 64, 64, 64, fake, fake, None, None, s) == 1
    # compress of the transpose: R % 8, ldw / ldm < C, dtype, NULL, misaligned, empty
    assert L.nm_compress_t(fake, fake, 1, 12, 64, 64, 64, fake, fake, None, None, s) == 2
    assert L.nm_compress_t(fake, fake, 1, 16, 64, 32, 64, fake, fake, None, None, s) == 2
    assert L.nm_compress_t(fake, fake, 1, 16, 64, 64, 32, fake, fake, None, None, s) == 2
    assert L.nm_compress_t(fake, fake, 9, 16, 64, 64, 64, fake, fake, None, None, s) == 4
    assert L.nm_compress_t(fake, None, 1, 16, 64, 64, 64, fake, fake, None, None, s) == 1
    assert L.nm_compress_t(fake, fake, 1, 16, 64, 64, 64, fake, odd, None, None, s) == 3
    assert L.nm_compress_t(fake, fake, 1, 16, 64, 68, 64, fake, fake, None, None, s) == 3   # ldw*2 not 16B
    assert L.nm_compress_t(fake, fake, 1, 16, 64, 64, 64, fake, fake, None, ctypes.c_void_p(0x10002), s) == 3
    assert L.nm_compress_t(fake, fake, 1, 0, 64, 64, 64, fake, fake, None, None, s) == 0    # R == 0: no-op
    assert L.nm_compress_t(fake, fake, 1, 16, 0, 0, 0, fake, fake, None, None, s) == 0      # C == 0: no-op
    # transposable mask: dtype, N:M, R % M, ldm < C, NULL, misaligned, empty
    assert L.nm_mask_transposable(fake, 9, 8, 8, 8, 4, 8, fake, 8, s) == 4
    assert L.nm_mask_transposable(fake, 1, 8, 8, 8, 8, 8, fake, 8, s) == 5
    assert L.nm_mask_transposable(fake, 1, 12, 16, 16, 4, 8, fake, 16, s) == 2
    assert L.nm_mask_transposable(fake, 1, 16, 16, 16, 4, 8, fake, 8, s) == 2
    assert L.nm_mask_transposable(None, 1, 16, 16, 16, 4, 8, fake, 16, s) == 1
    assert L.nm_mask_transposable(fake, 1, 16, 16, 16, 4, 8, odd, 16, s) == 3
    assert L.nm_mask_transposable(fake, 1, 0, 16, 16, 4, 8, fake, 16, s) == 0
    # saliency mask: int8 refused (floating-point call), NULL d, N:M
    assert L.nm_mask_scored(fake, 3, fake, 4, 64, 64, 2, 4, fake, 64, s) == 4
    assert L.nm_mask_scored(fake, 1, None, 4, 64, 64, 2, 4, fake, 64, s) == 1
    assert L.nm_mask_scored(fake, 1, fake, 4, 64, 64, 0, 4, fake, 64, s) == 5
    # 1:2 calls: C % 16, int8 refused
    assert L.nm_mask_compress12(fake, 0, 4, 40, 40, fake, fake, s) == 2
    assert L.nm_mask_compress12(fake, 3, 4, 64, 64, fake, fake, s) == 4
    assert L.nm_decompress12(fake, fake, 0, 4, 40, fake, 40, s) == 2
    assert L.nm_decompress(fake, fake, 1, 4, 64, fake, 60, s) == 2
    assert L.nm_meta_to_sm100(fake, 4, 60, fake, s) == 2
    assert L.nm_meta_to_sm100(None, 4, 64, fake, s) == 1
    f = ctypes.c_float
    # spmm: K % 16, dtype of Y, ldx < T, NULL, misaligned, workspace
    assert L.nm_spmm(fake, fake, 1, fake, 8, fake, 1, 8, 128, 40, 8, f(1), f(0), None, 0, s) == 2
    assert L.nm_spmm(fake, fake, 1, fake, 8, fake, 2, 8, 128, 64, 8, f(1), f(0), None, 0, s) == 4
    assert L.nm_spmm(fake, fake, 1, fake, 4, fake, 1, 8, 128, 64, 8, f(1), f(0), None, 0, s) == 2
    assert L.nm_spmm(fake, None, 1, fake, 8, fake, 1, 8, 128, 64, 8, f(1), f(0), None, 0, s) == 1
    assert L.nm_spmm(fake, fake, 1, odd, 8, fake, 1, 8, 128, 64, 8, f(1), f(0), None, 0, s) == 3
    assert L.nm_spmm(fake, fake, 1, fake, 12, fake, 1, 16, 128, 64, 12, f(1), f(0), None, 0, s) == 3
    assert L.nm_spmm(fake, fake, 0, fake, 8, fake, 0, 8, 128, 64, 8, f(1), f(0), None, 0, s) == 8
    assert L.nm_spmm(fake, fake, 1, fake, 8, fake, 1, 8, 0, 64, 8, f(1), f(0), None, 0, s) == 0
    # maximum sizes: tile coordinates are 32-bit, so R, K and T must stay below 2^31 - 256
    big = 2 ** 31 - 256
    assert L.nm_spmm(fake, fake, 1, fake, 8, fake, 1, 8, big, 64, 8, f(1), f(0), None, 0, s) == 2
    assert L.nm_spmm(fake, fake, 1, fake, 8, fake, 1, 8, 128, big // 16 * 16 + 16, 8, f(1), f(0), None, 0, s) == 2
    assert L.nm_spmm(fake, fake, 1, fake, big, fake, 1, big, 128, 64, big, f(1), f(0), None, 0, s) == 2
    # K == 0 with rows and columns to write has no product to form
    assert L.nm_spmm(fake, fake, 1, fake, 8, fake, 1, 8, 128, 0, 8, f(1), f(0), None, 0, s) == 2
    # the no-allocation product checks its arguments before its scratch limit: fp32 at 4096^3
    # needs 48 MiB of staging, more than its 16 MiB array, yet a malformed call reports its fault
    n = 4096
    assert L.nm_spmm_noalloc(fake, fake, 0, fake, n, fake, 0, n, n, n + 8, n, f(1), f(0), s) == 2   # K % 16
    assert L.nm_spmm_noalloc(fake, fake, 0, odd, n, fake, 0, n, n, n, n, f(1), f(0), s) == 3        # misaligned X
    assert L.nm_spmm_noalloc(fake, fake, 0, fake, n - 8, fake, 0, n, n, n, n, f(1), f(0), s) == 2   # ldx < T
    assert L.nm_spmm_noalloc(fake, fake, 0, fake, n, fake, 0, n, n, n, n, f(1), f(0), s) == 8       # too large
    assert L.nm_spmm_noalloc(fake, fake, 0, fake, n, fake, 0, n, 0, n, n, f(1), f(0), s) == 0       # R == 0
    # the test entry point: its own arguments, then nm_spmm's checks
    # int8 product: K % 32, output types, exact s32 output only with alpha 1 and beta 0
    assert L.nm_spmm(fake, fake, 3, fake, 16, fake, 4, 16, 128, 48, 16, f(1), f(0), None, 0, s) == 2
    assert L.nm_spmm(fake, fake, 3, fake, 16, fake, 2, 16, 128, 64, 16, f(1), f(0), None, 0, s) == 4
    assert L.nm_spmm(fake, fake, 3, fake, 16, fake, 4, 16, 128, 64, 16, f(2), f(0), None, 0, s) == 6
    assert L.nm_spmm(fake, fake, 3, fake, 16, fake, 4, 16, 128, 64, 16, f(1), f(1), None, 0, s) == 6
    assert L.nm_spmm(fake, fake, 3, fake, 8, fake, 4, 16, 128, 64, 8, f(1), f(0), None, 0, s) == 3   # ldx bytes % 16
    assert L.nm_spmm(fake, fake, 1, fake, 8, fake, 4, 8, 128, 64, 8, f(1), f(0), None, 0, s) == 4    # s32 out of bf16
    assert L.nm_spmm(fake, fake, 3, fake, 16, fake, 4, 16, 0, 64, 16, f(1), f(0), None, 0, s) == 0
    # TF32 1:2 product: K % 16, output types, X row stride, NULL, empty
    assert L.nm_spmm12(fake, fake, fake, 8, fake, 0, 8, 128, 40, 8, f(1), f(0), s) == 2
    assert L.nm_spmm12(fake, fake, fake, 8, fake, 3, 8, 128, 64, 8, f(1), f(0), s) == 4
    assert L.nm_spmm12(fake, fake, fake, 6, fake, 0, 8, 128, 64, 6, f(1), f(0), s) == 3
    assert L.nm_spmm12(fake, None, fake, 8, fake, 0, 8, 128, 64, 8, f(1), f(0), s) == 1
    assert L.nm_spmm12(fake, fake, fake, 8, fake, 0, 8, 128, 64, 0, f(1), f(0), s) == 0
    assert L.nm_spmm12_test(fake, fake, fake, 8, fake, 0, 8, 128, 64, 8, f(1), f(0), 10, 1, s) == 2
    # the two metadata images
    assert L.nm_meta_to_sm100_s8(fake, 4, 60, fake, s) == 2
    assert L.nm_meta_to_sm100_s8(None, 4, 64, fake, s) == 1
    assert L.nm_meta_to_sm100_s8(fake, 4, 64, odd, s) == 3
    assert L.nm_meta12_to_sm100(fake, 4, 40, fake, s) == 2
    assert L.nm_meta12_to_sm100(fake, 4, 64, None, s) == 1
    assert L.nm_meta12_to_sm100(fake, 0, 64, fake, s) == 0
    t = lambda kern, split, wait, skip, K=64, rg=0, rm=0: L.nm_spmm_test(
        fake, fake, 1, fake, 8, fake, 1, 8, 128, K, 8, f(1), f(0), None, 0, kern, split, wait, skip, rg, rm, s)
    assert t(10, 1, 0, -1) == 2 and t(-1, 1, 0, -1) == 2
    assert t(0, 1, -5, -1) == 2 and t(0, 1, 0, -2) == 2
    assert t(1, 1, 0, -1, K=40) == 2
    assert t(0, 1, 0, -1, rg=-1) == 2 and t(0, 1, 0, -1, rg=4, rm=2) == 2


def test_image_sizes(lib):
    """.kind::i8: 128-row x 256-column stages, one bit per column; .kind::tf32:
    2048 bytes per 128 rows x 64 fp32 columns."""
    assert lib.nm_meta_s8_image_bytes(200, 300) == 256 * 512 // 8
    assert lib.nm_meta_s8_image_bytes(128, 256) == 128 * 256 // 8
    assert lib.nm_meta12_image_bytes(200, 100) == 2 * 2 * 2048
    assert lib.nm_meta12_image_bytes(128, 64) == 2048
    assert lib.nm_meta12_image_bytes(0, 64) == 0


def test_workspace_size(lib):
    import torch
    assert nm.nm_spmm_workspace_bytes(torch.bfloat16, 256, 256, 128) == 0
    need = nm.nm_spmm_workspace_bytes(torch.float32, 256, 256, 128)
    assert need >= 256 * 128 * 2 + 256 * 128 * 2


def test_no_cpu_fallback_in_the_binding():
    """The product binding must not reach the oracle or any CPU path."""
    with open(os.path.join(ROOT, "structured_sparsity_prune_b200", "__init__.py")) as f:
        src = f.read()
    assert "oracle" not in src.replace("no CPU\nfallback", "")
    assert "import numpy" not in src


def test_binding_has_every_declared_call():
    """The Python binding keeps the C names: one function per declared call."""
    missing = [name for name in _declared() if not callable(getattr(nm, name, None))]
    assert missing == []


def test_peer_calls_validate_on_the_host(lib):
    """nm_spmm_peers, nm_peer_signal, nm_peer_wait and the IPC calls reject
    malformed arguments before any CUDA call."""
    fake = 0x10000
    s = ctypes.c_void_p(0)
    vp = ctypes.c_void_p
    f = ctypes.c_float

    def arr(*xs):
        return (ctypes.c_void_p * len(xs))(*xs)

    def peers(ptrs, n, row0=0, ldy=256, dtype=1, R=256, K=64, T=256, n_override=None):
        return lib.nm_spmm_peers(vp(fake), vp(fake), dtype, vp(fake), 256, arr(*ptrs) if ptrs is not None else None,
                                 n if n_override is None else n_override, row0, ldy, R, K, T, f(1), s)

    assert peers([fake], 1, dtype=0) == 4                     # fp32 operands: no peer path
    assert peers([fake], 1, dtype=3) == 4                     # int8 operands: no peer path
    assert peers([fake], 0, n_override=0) == 2                # no destination
    assert peers([fake] * 9, 9) == 2                          # more than NM_MAX_PEERS
    assert peers([fake], 1, row0=-1) == 2
    assert peers(None, 1) == 1                                # NULL array
    assert peers([fake, 0], 2) == 1                           # NULL destination
    assert peers([fake], 1, K=40) == 2                        # K % 16
    assert peers([fake], 1, ldy=200) == 2                     # ldy < T
    assert peers([fake], 1, ldy=260) == 3                     # ldy * 2 not a multiple of 16
    assert peers([fake, fake + 8], 2) == 3                    # destination rows not 16-byte aligned
    assert peers([fake], 1, R=0) == 0                         # nothing to compute
    assert lib.nm_peer_signal(arr(fake, fake), 2, 2, 1, s) == 2       # rank outside [0, n)
    assert lib.nm_peer_signal(arr(fake), 0, 0, 1, s) == 2
    assert lib.nm_peer_signal(arr(*([fake] * 9)), 9, 0, 1, s) == 2
    assert lib.nm_peer_signal(None, 2, 0, 1, s) == 1
    assert lib.nm_peer_signal(arr(fake, 0), 2, 0, 1, s) == 1
    assert lib.nm_peer_signal(arr(fake, fake + 4), 2, 0, 1, s) == 3   # flags not 8-byte aligned
    assert lib.nm_peer_wait(vp(fake), 2, 1, 0, s) == 2                # no time limit
    assert lib.nm_peer_wait(vp(fake), 9, 1, 1000, s) == 2
    assert lib.nm_peer_wait(None, 2, 1, 1000, s) == 1
    assert lib.nm_peer_wait(vp(fake + 4), 2, 1, 1000, s) == 3
    h = ctypes.create_string_buffer(64)
    off = ctypes.c_int64()
    assert lib.nm_ipc_handle(None, h, ctypes.byref(off)) == 1
    assert lib.nm_ipc_handle(vp(fake), None, ctypes.byref(off)) == 1
    p = ctypes.c_void_p()
    assert lib.nm_ipc_open(None, 0, ctypes.byref(p)) == 1
    assert lib.nm_ipc_open(h, -1, ctypes.byref(p)) == 2
    assert lib.nm_ipc_close(None, 0) == 1
    assert lib.nm_ipc_close(vp(fake), -1) == 2
