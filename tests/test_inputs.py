"""The seeded input recipes (nm_inputs), on CPU: what both the oracle and the
CUDA path are fed must be what the recipes state, and the same on every call."""
import os
import sys

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import nm_inputs  # noqa: E402


def test_every_recipe_has_its_own_seed():
    seeds = list(nm_inputs.SEEDS.values())
    assert len(seeds) == len(set(seeds))
    decode_x = {105 + T for T in (16, 64, 256, 1024)}          # the skinny activations' seeds
    assert not decode_x & set(seeds)


def test_draws_repeat_and_seeds_differ():
    a = nm_inputs.normal((32, 48), 9, 0.02, torch.bfloat16)
    assert torch.equal(a, nm_inputs.normal((32, 48), 9, 0.02, torch.bfloat16))
    assert not torch.equal(a, nm_inputs.normal((32, 48), 10, 0.02, torch.bfloat16))


def test_low_precision_draws_are_the_rounded_fp32_draw():
    """bf16(0.02 * N(0,1)): one fp32 product, then one rounding to the target type."""
    for dtype in (torch.bfloat16, torch.float16):
        got = nm_inputs.normal((64, 64), 11, 0.02, dtype)
        ref = (nm_inputs.normal((64, 64), 11, 1.0, torch.float32) * 0.02).to(dtype)
        assert got.dtype == dtype and torch.equal(got, ref)


def test_ties_are_hundredths_from_minus_eight_to_seven():
    W = nm_inputs.ties((256, 256), nm_inputs.SEEDS["ties_fp32.W"])
    assert W.dtype == torch.float32
    allowed = np.array([np.float32(np.float64(k) / 100.0) for k in range(-8, 8)], dtype=np.float32)
    vals, counts = np.unique(W.numpy(), return_counts=True)
    assert np.array_equal(vals, np.sort(allowed))                # every value, nothing else
    assert counts.min() > 256 * 256 // 16 // 2                    # heavy exact ties throughout


def test_saliency_d_is_the_diagonal_of_the_inverse_factor():
    """d = diag(U), U upper with U^T U = H^-1.  Its ends have closed forms:
    U[0,0]^2 = (H^-1)[0,0], and U[C-1,C-1] = 1 / sqrt(H[C-1,C-1])."""
    C, n = 48, 512
    d = nm_inputs.saliency_d(C, n).double().numpy()
    g = torch.Generator().manual_seed(nm_inputs.SEEDS["saliency.X"])
    X = torch.randn(n, C, generator=g, dtype=torch.float64)
    H = (2.0 / n) * (X.T @ X)
    H.diagonal().add_(0.01 * H.diagonal().mean())
    H = H.numpy()
    assert d.shape == (C,) and np.all(d > 0)
    assert abs(d[0] - np.sqrt(np.linalg.inv(H)[0, 0])) <= 1e-6 * d[0]
    assert abs(d[-1] - 1.0 / np.sqrt(H[-1, -1])) <= 1e-6 * d[-1]
