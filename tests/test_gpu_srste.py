"""GPU parity of the fused SR-STE step against the CPU oracle, bit for bit."""
import numpy as np
import pytest
import torch

import oracle
import nm_inputs
import structured_sparsity_prune_b200 as nm

pytestmark = pytest.mark.gpu

CODE = {torch.float32: oracle.F32, torch.bfloat16: oracle.BF16, torch.float16: oracle.F16}


def _bits(t):
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.float32:
        return t.view(torch.int32).numpy().view(np.uint32)
    if t.dtype == torch.uint8:
        return t.numpy()
    return t.view(torch.int16).numpy().view(np.uint16)


@pytest.fixture(scope="module", autouse=True)
def _built():
    from structured_sparsity_prune_b200 import build
    build.build()
    oracle.build()


def _case(R, C, dtype, seed, ties=False):
    if ties:
        W = nm_inputs.ties((R, C), seed).to(dtype)
    else:
        W = nm_inputs.normal((R, C), seed, 1.0, dtype)
    G = nm_inputs.normal((R, C), seed + 1, 1e-3, dtype)
    return W, G


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16, torch.float16])
@pytest.mark.parametrize("N,M", [(2, 4), (1, 4), (3, 4), (4, 8), (2, 8), (2, 3)])
@pytest.mark.parametrize("R,C", [(64, 96), (33, 48), (128, 528)])
def test_srste_matches_oracle(dtype, N, M, R, C):
    if C % M:
        pytest.skip("C must be a multiple of M")
    W, G = _case(R, C, dtype, R + C + N * 7 + M, ties=(R == 33))
    ws, go, mask = nm.nm_srste_step(W.cuda(), G.cuda(), N, M, 0.0002, want_mask=True)
    e_ws, e_go, e_mask = oracle.srste(_bits(W), _bits(G), N, M, 0.0002, dtype=CODE[dtype])
    assert np.array_equal(_bits(mask), e_mask)
    assert np.array_equal(_bits(ws), np.ascontiguousarray(e_ws).view(_bits(ws).dtype))
    assert np.array_equal(_bits(go), np.ascontiguousarray(e_go).view(_bits(go).dtype))


def test_srste_strided_without_mask_and_large_decay():
    R, C, ld = 40, 256, 320
    dtype = torch.bfloat16
    Wf, Gf = _case(R, ld, dtype, 5)
    W, G = Wf.cuda()[:, :C], Gf.cuda()[:, :C]
    ws, go, mask = nm.nm_srste_step(W, G, 2, 4, 0.5)
    assert mask is None
    e_ws, e_go, _ = oracle.srste(_bits(Wf[:, :C]), _bits(Gf[:, :C]), 2, 4, 0.5, dtype=oracle.BF16)
    assert np.array_equal(_bits(ws), e_ws)
    assert np.array_equal(_bits(go), e_go)


def test_srste_full_size_linear_weight():
    """The 4096 x 4096 bf16 transformer-linear weight with a bf16 gradient."""
    W, _ = nm_inputs.linear_4096()
    G = nm_inputs.normal((4096, 4096), nm_inputs.SEEDS["srste.grad"], 1e-3, torch.bfloat16)
    ws, go, mask = nm.nm_srste_step(W.cuda(), G.cuda(), 2, 4, 0.0002, want_mask=True)
    e_ws, e_go, e_mask = oracle.srste(_bits(W), _bits(G), 2, 4, 0.0002, dtype=oracle.BF16)
    assert np.array_equal(_bits(mask), e_mask)
    assert np.array_equal(_bits(ws), e_ws)
    assert np.array_equal(_bits(go), e_go)
