"""Pins for the oracle's dense bf16 GEMM (few output columns).

* identity weights: Y is X exactly;
* a single non-zero weight at (n0, k0): only column n0 is non-zero and it
  equals X[:, k0] times that weight (catches a transposed or reversed index);
* exact-integer regime: small integer activations and weights, the sum
  computed with Python integers;
* brute force against torch's bf16 decoder and a float64 matmul.
"""
import numpy as np
import pytest
import torch

import synth


def _bits(v):
    return torch.tensor(np.asarray(v, dtype=np.float32)).to(torch.bfloat16).view(
        torch.int16).numpy().view(np.uint16)


def _f64(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(
        torch.bfloat16).double().numpy()


def test_identity(orc):
    M, K = 3, 96
    lay = synth.bf16_layer(M, K, K, seed=1)
    W = _bits(np.eye(K))
    Y = orc.bf16_gemm(lay.X, W, M, K, K)
    assert np.array_equal(Y, _f64(lay.X))


@pytest.mark.parametrize("n0,k0", [(0, 0), (5, 63), (47, 17), (95, 127)])
def test_single_weight_index(orc, n0, k0):
    M, K, N = 4, 128, 96
    lay = synth.bf16_layer(M, K, N, seed=2)
    w = np.zeros((N, K), dtype=np.float32)
    w[n0, k0] = 2.0
    Y = orc.bf16_gemm(lay.X, _bits(w), M, N, K)
    expect = np.zeros((M, N))
    expect[:, n0] = 2.0 * _f64(lay.X)[:, k0]
    assert np.array_equal(Y, expect)


def test_exact_integer_regime(orc):
    rng = np.random.default_rng(3)
    M, K, N = 4, 256, 48
    xi = rng.integers(-8, 9, size=(M, K))
    wi = rng.integers(-8, 9, size=(N, K))
    Y = orc.bf16_gemm(_bits(xi), _bits(wi), M, N, K)
    want = [[sum(int(xi[m, k]) * int(wi[n, k]) for k in range(K)) for n in range(N)]
            for m in range(M)]
    assert np.array_equal(Y, np.array(want, dtype=np.float64))


@pytest.mark.parametrize("M,K,N", [(1, 64, 16), (4, 320, 96), (8, 5120, 32)])
def test_brute_force_vs_torch(orc, M, K, N):
    lay = synth.bf16_layer(M, K, N, seed=M + K + N)
    Y = orc.bf16_gemm(lay.X, lay.W, M, N, K)
    ref = _f64(lay.X) @ _f64(lay.W).T
    assert np.allclose(Y, ref, rtol=1e-12, atol=1e-12)


def test_invalid_arguments(orc):
    with pytest.raises(Exception):
        orc.bf16_gemm(np.zeros((1, 64), np.uint16), np.zeros((16, 64), np.uint16), 0, 16, 64)
