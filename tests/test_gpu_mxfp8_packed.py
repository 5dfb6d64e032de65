"""Re-packed MXFP8 weight streaming (mxfp8_repack + mxfp8_gemm_packed)
against the fp64 oracle, through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import (assert_parity, assert_sampled_parity, bf16_tensor, bits_of_bf16, to_f64)

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.fixture(scope="module")
def mxg():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    import mxfp8_gemm_speculative_b200 as m
    return m


def packed_call(mxg, lay):
    wq = torch.from_numpy(lay.Wq).to(DEV)
    ws = torch.from_numpy(lay.Ws).to(DEV)
    packed = mxg.mxfp8_repack(wq, ws)
    return mxg.mxfp8_gemm_packed(bf16_tensor(lay.X, DEV), packed, lay.N, lay.K)


# N: one group, a group and a ragged group of two tiles, several groups;
# K: whole 128-row stages, a last stage of one 64-row chunk, long rows
@pytest.mark.parametrize("M", [1, 4, 5, 8, 9, 16])
@pytest.mark.parametrize("N,K", [(256, 512), (320, 640), (512, 2048), (1024, 5120)])
def test_packed_parity(mxg, M, N, K):
    lay = synth.mxfp8_layer(M, K, N, seed=3 * M + N + K)
    y = packed_call(mxg, lay)
    ref = oracle.mxfp8_gemm(lay.X, lay.Wq, lay.Ws, M, N, K)
    assert_parity(to_f64(y), ref, f"mxfp8 packed M={M} N={N} K={K}")


def test_packed_matches_unpacked_path(mxg):
    M, N, K = 5, 768, 1536
    lay = synth.mxfp8_layer(M, K, N, seed=11)
    yp = to_f64(packed_call(mxg, lay))
    yu = to_f64(mxg.mxfp8_gemm(bf16_tensor(lay.X, DEV), torch.from_numpy(lay.Wq).to(DEV),
                               torch.from_numpy(lay.Ws).to(DEV)))
    ref = oracle.mxfp8_gemm(lay.X, lay.Wq, lay.Ws, M, N, K)
    assert_parity(yp, ref, "packed")
    assert_parity(yu, ref, "unpacked")


def test_packed_identity_is_exact(mxg):
    # W = I * 1.0 (E4M3 0x38) with block scale 2^-3: Y = X / 8 exactly
    K = N = 256
    Wq = np.zeros((N, K), dtype=np.uint8)
    np.fill_diagonal(Wq, 0x38)
    Ws = np.full((N, K // 32), 124, dtype=np.uint8)
    X = synth.mxfp8_layer(3, K, N, seed=2).X
    packed = mxg.mxfp8_repack(torch.from_numpy(Wq).to(DEV), torch.from_numpy(Ws).to(DEV))
    y = mxg.mxfp8_gemm_packed(bf16_tensor(X, DEV), packed, N, K)
    xin = torch.from_numpy(X.view(np.int16)).view(torch.bfloat16).float() * 0.125
    assert np.array_equal(bits_of_bf16(y), bits_of_bf16(xin.to(torch.bfloat16)))


def test_packed_wide_activation_range(mxg):
    # every 64-row group of X at its own magnitude, 2^-90 .. 2^90: the
    # power-of-two factor per (group, token) keeps each group exact in fp16
    M, N, K = 4, 256, 1024
    lay = synth.mxfp8_layer(M, K, N, seed=4)
    x = torch.from_numpy(lay.X.view(np.int16)).view(torch.bfloat16).float()
    rng = np.random.default_rng(9)
    ex = rng.integers(-90, 91, size=(M, K // 64))
    x = x * torch.from_numpy(np.repeat(np.exp2(ex.astype(np.float64)), 64, axis=1)).float()
    xb = x.to(torch.bfloat16)
    X = bits_of_bf16(xb)
    packed = mxg.mxfp8_repack(torch.from_numpy(lay.Wq).to(DEV), torch.from_numpy(lay.Ws).to(DEV))
    y = to_f64(mxg.mxfp8_gemm_packed(xb.to(DEV), packed, N, K))
    ref = oracle.mxfp8_gemm(X, lay.Wq, lay.Ws, M, N, K)
    assert_parity(y, ref, "wide activation range")


def test_packed_m4_full_size_sampled(mxg):
    M, K, N = 4, 5120, 17408
    lay = synth.mxfp8_layer(M, K, N, seed=0)
    yf = to_f64(packed_call(mxg, lay))
    rng = np.random.default_rng(6)
    rows = rng.integers(0, M, size=512)
    cols = rng.integers(0, N, size=512)
    ref = oracle.mxfp8_gemm_at(lay.X, lay.Wq, lay.Ws, M, N, K, rows, cols,
                               nthreads=oracle.threads(64))
    rms = float(np.sqrt(np.mean(ref ** 2)))
    assert_sampled_parity(yf[rows, cols], ref, rms, "mxfp8 packed M=4 full size")
    assert np.isfinite(yf).all()


def test_packed_rejects_shapes(mxg):
    assert mxg.raw_lib().mxfp8_packed_bytes(96, 512) == 0      # N % 64
    assert mxg.raw_lib().mxfp8_packed_bytes(256, 96) == 0      # K % 64
    assert mxg.mxfp8_packed_workspace_bytes(17, 256, 512) == 0  # M > 16
    lay = synth.mxfp8_layer(17, 512, 256, seed=1)
    packed = mxg.mxfp8_repack(torch.from_numpy(lay.Wq).to(DEV), torch.from_numpy(lay.Ws).to(DEV))
    with pytest.raises(mxg.MxgError) as e:
        mxg.mxfp8_gemm_packed(bf16_tensor(lay.X, DEV), packed, 256, 512,
                              workspace_buf=torch.zeros(1 << 20, dtype=torch.uint8, device=DEV))
    assert e.value.status == mxg.MXG_ERR_UNSUPPORTED_SHAPE
