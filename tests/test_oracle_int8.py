"""Pins for the oracle's INT8 W8A16 unpack and GEMM (the vocabulary head).

* hand-packed words: byte j of word (i, n) is the code of row 4i + j of
  column n, least significant byte first, weight (q - 128) * scale;
* the scale index: scale (g, n) multiplies exactly rows gG .. gG+G-1 of n;
* identity weights (code 129 on the diagonal, 128 elsewhere, scale 1): Y is X
  exactly;
* exact-integer regime: small integer activations and weights, power-of-two
  scales, the sum computed with Python integers;
* brute force against an independent numpy decode and a float64 matmul.
"""
import numpy as np
import pytest
import torch

import synth


def _f64(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(
        torch.bfloat16).double().numpy()


def _bf16_bits(v):
    return torch.tensor(np.asarray(v, dtype=np.float32)).to(torch.bfloat16).view(
        torch.int16).numpy().view(np.uint16)


def test_hand_packed_words(orc):
    K, N, G = 32, 2, 32
    qw = np.full((K // 4, N), np.uint32(0x80808080).view(np.int32), dtype=np.int32)
    qw[0, 0] = np.uint32(0x83828180).view(np.int32)       # rows 0..3 of column 0
    qw[2, 1] = np.uint32(0x7F00FF01).view(np.int32)       # rows 8..11 of column 1
    sc = np.array([[0x3C00, 0x4000]], dtype=np.uint16)      # 1.0, 2.0
    codes, w = orc.w8a16_unpack(qw, sc, K, N, G)
    assert codes[0, :4].tolist() == [128, 129, 130, 131]
    assert codes[1, 8:12].tolist() == [1, 255, 0, 127]
    assert w[0, :4].tolist() == [0.0, 1.0, 2.0, 3.0]
    assert w[1, 8:12].tolist() == [-254.0, 254.0, -256.0, -2.0]
    assert np.count_nonzero(w) == 7


def test_scale_index(orc):
    K, N = 256, 3
    for G in (32, 64, 128):
        for n in range(N):
            for g in range(K // G):
                qw = np.full((K // 4, N), np.uint32(0x81818181).view(np.int32), dtype=np.int32)
                sc = np.full((K // G, N), 0x3C00, dtype=np.uint16)
                sc[g, n] = 0x4400                                        # 4.0
                _, w = orc.w8a16_unpack(qw, sc, K, N, G)
                expect = np.ones((N, K))
                expect[n, g * G:(g + 1) * G] = 4.0
                assert np.array_equal(w, expect)


def test_identity(orc):
    M, K = 3, 128
    lay = synth.int8_layer(M, K, K, 32, seed=4)
    codes = np.full((K, K), 128, dtype=np.uint8)
    np.fill_diagonal(codes, 129)
    qw = np.ascontiguousarray(codes.T).reshape(K // 4, 4, K).transpose(0, 2, 1)
    qw = np.ascontiguousarray(qw).view(np.uint32).reshape(K // 4, K).view(np.int32)
    sc = np.full((K // 32, K), 0x3C00, dtype=np.uint16)
    Y = orc.w8a16_gemm(lay.X, qw, sc, M, K, K, 32)
    assert np.array_equal(Y, _f64(lay.X))


def test_exact_integer_regime(orc):
    rng = np.random.default_rng(6)
    M, K, N, G = 3, 128, 8, 64
    lay = synth.int8_layer(M, K, N, G, seed=6)
    xi = rng.integers(-4, 5, size=(M, K))
    sc = np.full((K // G, N), 0x4000, dtype=np.uint16)                 # 2.0
    Y = orc.w8a16_gemm(_bf16_bits(xi), lay.qweight, sc, M, N, K, G)
    want = [[sum(int(xi[m, k]) * (int(lay.codes[n, k]) - 128) * 2 for k in range(K))
             for n in range(N)] for m in range(M)]
    assert np.array_equal(Y, np.array(want, dtype=np.float64))


@pytest.mark.parametrize("M,K,N,G", [(1, 64, 8, 32), (5, 256, 24, 64), (4, 512, 16, 128)])
def test_brute_force_vs_numpy(orc, M, K, N, G):
    lay = synth.int8_layer(M, K, N, G, seed=M + K + N + G)
    words = np.ascontiguousarray(lay.qweight).view(np.uint32)           # [K/4][N]
    shifts = np.arange(4, dtype=np.uint32) * np.uint32(8)
    q = ((words[:, None, :] >> shifts[None, :, None]) & np.uint32(0xFF)).reshape(K, N)
    s = np.ascontiguousarray(lay.scales).view(np.float16).astype(np.float64)
    W = (q.astype(np.float64) - 128.0) * np.repeat(s, G, axis=0)        # [K][N]
    Y = orc.w8a16_gemm(lay.X, lay.qweight, lay.scales, M, N, K, G)
    assert np.allclose(Y, _f64(lay.X) @ W, rtol=1e-12, atol=1e-12)
    codes, w = orc.w8a16_unpack(lay.qweight, lay.scales, K, N, G)
    assert np.array_equal(codes, lay.codes)
    assert np.array_equal(w, W.T)


def test_invalid_arguments(orc):
    with pytest.raises(Exception):
        orc.w8a16_gemm(np.zeros((1, 64), np.uint16), np.zeros((16, 8), np.int32),
                       np.zeros((2, 8), np.uint16), 1, 8, 64, 48)


def test_int8_with_int4_codes_equals_int4(orc):
    """INT8 codes q + 120 for INT4 codes q (so q8 - 128 = q - 8) with the same
    scales give the INT4 layer's Y exactly: the two formats' oracles agree."""
    M, K, N, G = 3, 256, 32, 64
    lay4 = synth.int4_layer(M, K, N, G, seed=21)
    codes8 = (lay4.codes.astype(np.int32) + 120).astype(np.uint8)
    qw8 = np.ascontiguousarray(codes8.T).reshape(K // 4, 4, N).transpose(0, 2, 1)
    qw8 = np.ascontiguousarray(qw8).view(np.uint32).reshape(K // 4, N).view(np.int32)
    y8 = orc.w8a16_gemm(lay4.X, qw8, lay4.scales, M, N, K, G)
    y4 = orc.w4a16_gemm(lay4.X, lay4.qweight, lay4.scales, M, N, K, G)
    assert np.array_equal(y8, y4)
