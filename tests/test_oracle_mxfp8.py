"""Pins for the oracle's MXFP8 dequantization and GEMM.

* identity weights (E4M3 1.0 on the diagonal, scale 2^0 or 2^-3): Y is X
  (or X * 2^-3) exactly;
* exact-integer regime with integer-valued E4M3 codes and power-of-two block
  scales: the sum is an integer computed with Python integers;
* brute force on tiny shapes against an independent numpy/torch
  implementation (torch's float8_e4m3fn / float8_e8m0fnu decoders);
* the block index: scale (n, b) multiplies exactly k = 32b .. 32b+31 of row n;
* NaN codes and scales are rejected.
"""
import numpy as np
import pytest
import torch

import synth


def _bf16_to_f64(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(
        torch.bfloat16).double().numpy()


def _f64_to_bf16_bits(v):
    return torch.from_numpy(np.ascontiguousarray(v, dtype=np.float32)).to(
        torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _torch_dense(Wq, Ws, N, K):
    v = torch.from_numpy(np.ascontiguousarray(Wq)).view(torch.float8_e4m3fn).double()
    s = torch.from_numpy(np.ascontiguousarray(Ws)).view(torch.float8_e8m0fnu).double()
    return (v * s.repeat_interleave(32, dim=1)).numpy()


@pytest.mark.parametrize("E,factor", [(127, 1.0), (124, 0.125)])
def test_identity(orc, E, factor):
    K = N = 256
    Wq = np.zeros((N, K), dtype=np.uint8)
    np.fill_diagonal(Wq, 0x38)
    Ws = np.full((N, K // 32), E, dtype=np.uint8)
    X = synth.mxfp8_layer(4, K, N, seed=9).X
    Y = orc.mxfp8_gemm(X, Wq, Ws, 4, N, K)
    assert np.array_equal(Y, _bf16_to_f64(X) * factor)


def test_block_index(orc):
    N, K = 4, 128
    Wq = np.full((N, K), 0x38, dtype=np.uint8)
    Ws = np.zeros((N, K // 32), dtype=np.uint8)
    for n in range(N):
        for b in range(K // 32):
            Ws[n, b] = 120 + 2 * b + n
    w = orc.mxfp8_dequant(Wq, Ws, N, K)
    for n in range(N):
        for k in range(K):
            assert w[n, k] == 2.0 ** (120 + 2 * (k // 32) + n - 127)


def test_exact_integer_regime(orc):
    rng = np.random.default_rng(3)
    M, K, N = 5, 256, 128
    # E4M3 codes of the integers -4..4 (from the format: 1.f * 2^(e-7))
    int_codes = {0: 0x00, 1: 0x38, 2: 0x40, 3: 0x44, 4: 0x48}
    vals = rng.integers(-4, 5, size=(N, K))
    Wq = np.array([[int_codes[abs(v)] | (0x80 if v < 0 else 0) for v in row] for row in vals],
                  dtype=np.uint8)
    e = rng.integers(125, 130, size=(N, K // 32))
    Ws = e.astype(np.uint8)
    xi = rng.integers(-3, 4, size=(M, K))
    X = _f64_to_bf16_bits(xi.astype(np.float64))
    Y = orc.mxfp8_gemm(X, Wq, Ws, M, N, K)
    for m in range(M):
        for n in range(N):
            tot = 0   # 4 * sum (scale exponents >= -2)
            for k in range(K):
                tot += int(xi[m, k]) * int(vals[n, k]) * 2 ** (int(e[n, k // 32]) - 127 + 2)
            assert Y[m, n] == tot / 4.0


@pytest.mark.parametrize("M", [1, 4, 5, 17, 33])
@pytest.mark.parametrize("N,K", [(128, 64), (130, 96), (256, 320)])
def test_brute_force_vs_torch(orc, M, N, K):
    lay = synth.mxfp8_layer(M, K, N, seed=M + N + K)
    Y = orc.mxfp8_gemm(lay.X, lay.Wq, lay.Ws, M, N, K)
    W = _torch_dense(lay.Wq, lay.Ws, N, K)
    assert np.array_equal(orc.mxfp8_dequant(lay.Wq, lay.Ws, N, K), W)
    ref = _bf16_to_f64(lay.X) @ W.T
    err = np.abs(Y - ref).max() / max(np.abs(ref).max(), 1e-300)
    assert err <= 1e-12
    rows = [0, M - 1]
    cols = [N - 1, 0]
    assert np.array_equal(orc.mxfp8_gemm_at(lay.X, lay.Wq, lay.Ws, M, N, K, rows, cols),
                          Y[rows, cols])


def test_all_codes_dequant(orc):
    """Every finite code at several block scales: value = e4m3 * 2^(E-127)."""
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    K = 32 * ((codes.size + 31) // 32)
    for E in (100, 119, 123, 127, 140):
        Wq = np.zeros((1, K), dtype=np.uint8)
        Wq[0, :codes.size] = codes
        Ws = np.full((1, K // 32), E, dtype=np.uint8)
        w = orc.mxfp8_dequant(Wq, Ws, 1, K)
        ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy() * 2.0 ** (E - 127)
        assert np.array_equal(w[0, :codes.size], ref)


def test_nan_inputs_rejected(orc):
    lay = synth.mxfp8_layer(1, 64, 128, seed=0)
    Wq = lay.Wq.copy()
    Wq[3, 5] = 0x7F
    with pytest.raises(ValueError):
        orc.mxfp8_gemm(lay.X, Wq, lay.Ws, 1, 128, 64)
    Ws = lay.Ws.copy()
    Ws[0, 0] = 0xFF
    with pytest.raises(ValueError):
        orc.mxfp8_dequant(lay.Wq, Ws, 128, 64)
