"""GPU parity of the dense bf16 few-column projection (the paired GDN A/B
projection, N = 96, K = 5120, M = 1 and 4) through the C ABI, against the
CPU oracle."""
import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import assert_parity, bf16_tensor, to_f64

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda", 0)


@pytest.fixture(scope="module")
def mxg():
    import __graft_entry__
    __graft_entry__.build()
    import mxfp8_gemm_speculative_b200 as m
    return m


@pytest.mark.parametrize("M,N,K", [(1, 96, 5120), (4, 96, 5120), (8, 96, 5120), (3, 16, 64),
                                   (5, 256, 1024), (2, 48, 17408), (4, 96, 37888), (1, 2048, 320)])
def test_bf16_small_parity(mxg, M, N, K):
    lay = synth.bf16_layer(M, K, N, seed=M + N + K)
    y = mxg.bf16_gemm_small(bf16_tensor(lay.X, DEV), bf16_tensor(lay.W, DEV))
    assert_parity(to_f64(y), oracle.bf16_gemm(lay.X, lay.W, M, N, K), f"bf16 small {M}x{N}x{K}")


def test_bf16_small_exact_identity(mxg):
    """Identity weights: every output is one product, so Y is X bit for bit."""
    M, K = 4, 128
    lay = synth.bf16_layer(M, K, K, seed=9)
    eye = torch.eye(K, dtype=torch.bfloat16, device=DEV)
    y = mxg.bf16_gemm_small(bf16_tensor(lay.X, DEV), eye)
    assert torch.equal(y.view(torch.int16).cpu(), torch.from_numpy(lay.X.view(np.int16)))


def test_bf16_small_deterministic(mxg):
    M, N, K = 4, 96, 5120
    lay = synth.bf16_layer(M, K, N, seed=11)
    x, w = bf16_tensor(lay.X, DEV), bf16_tensor(lay.W, DEV)
    ws = torch.zeros(mxg.raw_lib().bf16_gemm_small_workspace_bytes(M, N, K), dtype=torch.uint8,
                     device=DEV)
    outs = [mxg.bf16_gemm_small(x, w, workspace_buf=ws, late_weights=late)
            for late in (False, False, True)]
    torch.cuda.synchronize()
    assert torch.equal(outs[0].view(torch.int16), outs[1].view(torch.int16))
    assert torch.equal(outs[0].view(torch.int16), outs[2].view(torch.int16))
    assert mxg.mxg_workspace_status(ws) == 0
