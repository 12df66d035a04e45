"""Seeded synthetic inputs shared by the tests, the smoke check and the bench.

This module holds only random-number recipes: it contains none of the
sparsity method's arithmetic, so both the CPU oracle and the CUDA library
can be fed from it without sharing any of the method.  Everything is drawn
on the CPU with torch's Philox-free default CPU generator (``torch.Generator``
seeded per tensor) and returned as CPU tensors; callers copy to the device.

The workloads stand in for the pages' models (vision and transformer
linear/conv weights; the pages' datasets and trained weights are not used):

* ``small_fp32``      W 256x256 ~N(0,1) (seed 0), X 256x128 ~N(0,1) (seed 100)
* ``linear_4096``     W bf16 4096x4096 = bf16(0.02 * N(0,1)) (seed 1),
                      X bf16 4096x4096 ~N(0,1) (seed 101)
* ``mlp_pair``        W_up bf16 14336x4096 (seed 2), W_down bf16 4096x14336
                      (seed 3), both bf16(0.02 * N(0,1)); X bf16 4096x8192 (seed 102)
* ``mlp_hidden``      a bf16 14336x8192 ~N(0,1) stand-in for the MLP pair's
                      hidden activation (seed 104), the down product's input in
                      its full-size parity test
* ``linear_4096_grad`` dY bf16 4096x4096 ~N(0,1) (seed 103), the backward
                      product's input in the transposable 2:4 step
* ``ties_fp32``       W fp32 8192x8192 = fp32(k/100), k ~ U{-8..7} (seed 4)
* ``decode_skinny``   W bf16 28672x8192 = bf16(0.02 * N(0,1)) (seed 5),
                      X bf16 8192xT ~N(0,1) (seed 105+T), T in {16,64,256,1024}
* ``srste``           the linear_4096 weight and a gradient bf16(1e-3 * N(0,1))
                      of the same shape (seed 6)
* ``int8_decode``     the decode_skinny weight quantised to int8:
                      clamp(round(w / 0.02 * 32), -128, 127)
* ``decode_X_int8``   the decode_skinny X (8192xT, seed 105+T) quantised to
                      int8: clamp(round(x * 32), -128, 127), the int8 product's
                      activations
* ``fp32_linear``     W fp32 8192x8192 = fp32(0.02 * N(0,1)) (seed 8), for the
                      1:2 pattern of sparse TF32; X fp32 8192xT ~N(0,1)
                      (seed 109), the TF32 product's activations
* ``saliency``        the linear_4096 weight and d of length 4096: the diagonal
                      of the upper Cholesky factor of H^-1, H = (2/n) X^T X +
                      0.01 * mean(diag) * I from n = 512 synthetic calibration
                      rows X ~ N(0,1) (seed 7), prepared in float64 the way
                      "sparsegpt.py" prepares its inverse Hessian, then
                      rounded to float32.  This stands in for calibration data.
"""
from __future__ import annotations

import torch

SEEDS = {
    "small_fp32.W": 0, "small_fp32.X": 100,
    "linear_4096.W": 1, "linear_4096.X": 101,
    "mlp_pair.W_up": 2, "mlp_pair.W_down": 3, "mlp_pair.X": 102,
    "ties_fp32.W": 4,
    "decode_skinny.W": 5,
    "srste.grad": 6,
    "saliency.X": 7,
    "fp32_linear.W": 8,
    "linear_4096.dY": 103,
    "mlp_pair.H": 104,
    "fp32_linear.X": 109,
}


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return g


def normal(shape, seed: int, std: float = 1.0, dtype=torch.float32) -> torch.Tensor:
    """N(0, std^2) drawn in fp32 then rounded (RNE) to `dtype`."""
    x = torch.randn(*shape, generator=_gen(seed), dtype=torch.float32)
    if std != 1.0:
        x = x * std
    return x.to(dtype)


def ties(shape, seed: int) -> torch.Tensor:
    """fp32(k/100), k uniform on the integers -8..7 (computed in fp64, rounded once)."""
    k = torch.randint(-8, 8, shape, generator=_gen(seed), dtype=torch.int64)
    return (k.to(torch.float64) / 100.0).to(torch.float32)


def small_int(shape, seed: int, lo: int = -8, hi: int = 8, dtype=torch.bfloat16) -> torch.Tensor:
    """Integer values in [lo, hi], exactly representable in bf16/f16/f32."""
    k = torch.randint(lo, hi + 1, shape, generator=_gen(seed), dtype=torch.int64)
    return k.to(torch.float32).to(dtype)


# ---- the named workloads ---------------------------------------------------
def small_fp32():
    return normal((256, 256), SEEDS["small_fp32.W"]), normal((256, 128), SEEDS["small_fp32.X"])


def linear_4096():
    return (normal((4096, 4096), SEEDS["linear_4096.W"], 0.02, torch.bfloat16),
            normal((4096, 4096), SEEDS["linear_4096.X"], 1.0, torch.bfloat16))


def linear_4096_grad():
    """Output gradient dY of the transformer linear (R x T = 4096 x 4096), bf16 ~N(0,1)."""
    return normal((4096, 4096), SEEDS["linear_4096.dY"], 1.0, torch.bfloat16)


def mlp_pair():
    return (normal((14336, 4096), SEEDS["mlp_pair.W_up"], 0.02, torch.bfloat16),
            normal((4096, 14336), SEEDS["mlp_pair.W_down"], 0.02, torch.bfloat16),
            normal((4096, 8192), SEEDS["mlp_pair.X"], 1.0, torch.bfloat16))


def mlp_hidden():
    """A 14336 x 8192 bf16 ~N(0,1) stand-in for the MLP pair's hidden activation
    (the down projection's input), drawn from its own seed."""
    return normal((14336, 8192), SEEDS["mlp_pair.H"], 1.0, torch.bfloat16)


def ties_fp32(R: int = 8192, C: int = 8192):
    return ties((R, C), SEEDS["ties_fp32.W"])


def decode_skinny_W():
    return normal((28672, 8192), SEEDS["decode_skinny.W"], 0.02, torch.bfloat16)


def decode_skinny_X(T: int):
    return normal((8192, T), 105 + T, 1.0, torch.bfloat16)


def bits_u16(t: torch.Tensor):
    """numpy uint16 view of a bf16/f16 CPU tensor (bit patterns)."""
    return t.contiguous().view(torch.int16).numpy().view("uint16")


def srste_grad(shape=(4096, 4096)):
    return normal(shape, SEEDS["srste.grad"], 1e-3, torch.bfloat16)


def saliency_d(C: int = 4096, n: int = 512, seed: int | None = None) -> torch.Tensor:
    """float32 vector of length C: diag of the upper Cholesky factor of the
    inverse of a damped synthetic Gram matrix (see the module docstring)."""
    g = _gen(SEEDS["saliency.X"] if seed is None else seed)
    X = torch.randn(n, C, generator=g, dtype=torch.float64)
    H = (2.0 / n) * (X.T @ X)
    H.diagonal().add_(0.01 * H.diagonal().mean())
    Hinv = torch.cholesky_inverse(torch.linalg.cholesky(H))
    U = torch.linalg.cholesky(Hinv, upper=True)
    return U.diagonal().to(torch.float32).contiguous()


def fp32_linear(R: int = 8192, C: int = 8192) -> torch.Tensor:
    return normal((R, C), SEEDS["fp32_linear.W"], 0.02, torch.float32)


def int8_decode() -> torch.Tensor:
    w = decode_skinny_W().float()
    return torch.clamp(torch.round(w / 0.02 * 32), -128, 127).to(torch.int8)


def decode_X_int8(T: int) -> torch.Tensor:
    x = decode_skinny_X(T).float()
    return torch.clamp(torch.round(x * 32), -128, 127).to(torch.int8)


def fp32_linear_X(T: int = 4096, K: int = 8192) -> torch.Tensor:
    return normal((K, T), SEEDS["fp32_linear.X"], 1.0, torch.float32)


def small_int8(shape, seed: int, lo: int = -128, hi: int = 127) -> torch.Tensor:
    """int8 values uniform on the integers lo..hi."""
    return torch.randint(lo, hi + 1, shape, generator=_gen(seed), dtype=torch.int64).to(torch.int8)
