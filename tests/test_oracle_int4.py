"""Pins for the oracle's INT4 W4A16 unpack, dequantization and GEMM.

Pins (none of them re-types the oracle's own formula):
* hand-packed worked examples (tests/golden/w4a16_worked_examples.txt);
* the pack/unpack round trip, and agreement with the input generator's packer;
* identity and permutation weights, where Y is X (or a scaled or permuted X)
  exactly;
* the exact-integer regime, where the sum is an integer computed with Python
  integers;
* brute force on tiny shapes against an independent numpy implementation
  (vectorised bit operations, float64 matmul).
"""
import os

import numpy as np
import pytest
import torch

import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(
        torch.bfloat16).double().numpy()


def _f64_to_bf16_bits(v: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(v, dtype=np.float32)).to(
        torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _numpy_dense_weights(qweight, scales, K, N, G):
    """Independent W[K][N] in float64 from GPTQ words (vectorised)."""
    words = np.ascontiguousarray(qweight).view(np.uint32)            # [K/8][N]
    shifts = np.arange(8, dtype=np.uint32) * np.uint32(4)
    q = (words[:, None, :] >> shifts[None, :, None]) & np.uint32(0xF)  # [K/8][8][N]
    q = q.reshape(K, N).astype(np.float64)
    s = np.ascontiguousarray(scales).view(np.float16).astype(np.float64)  # [K/G][N]
    return (q - 8.0) * np.repeat(s, G, axis=0)


def test_worked_examples(orc):
    with open(os.path.join(GOLDEN, "w4a16_worked_examples.txt")) as f:
        rows = [l.split() for l in f if l.strip() and not l.startswith("#")]
    assert len(rows) >= 10
    for r in rows:
        word = int(r[0], 16)
        scale_bits = int(r[1], 16)
        scale = float(r[2])
        q_want = [int(v) for v in r[3:11]]
        w_want = [float(v) for v in r[11:19]]
        assert orc.decode_fp16(scale_bits) == scale
        # one column (N=1), K=8, G=8: a single word and a single scale
        qw = np.array([[np.uint32(word).view(np.int32)]], dtype=np.int32)
        sc = np.array([[scale_bits]], dtype=np.uint16)
        codes, w = orc.w4a16_unpack(qw, sc, K=8, N=1, group_size=8)
        assert codes[0].tolist() == q_want, r[0]
        assert w[0].tolist() == w_want, r[0]


def test_nibble_order_and_column_index(orc):
    """Word (i, n) feeds rows 8i..8i+7 of column n and nothing else."""
    K, N, G = 32, 6, 32
    for i in range(K // 8):
        for n in range(N):
            qw = np.full((K // 8, N), np.uint32(0x88888888).view(np.int32), dtype=np.int32)
            qw[i, n] = np.uint32(0x76543210).view(np.int32)
            sc = np.full((K // G, N), 0x3C00, dtype=np.uint16)
            codes, w = orc.w4a16_unpack(qw, sc, K, N, G)
            expect = np.full((N, K), 8, dtype=np.uint8)
            expect[n, 8 * i:8 * i + 8] = np.arange(8)
            assert np.array_equal(codes, expect)
            assert np.array_equal(w, expect.astype(np.float64) - 8.0)


def test_group_index(orc):
    """Scale (g, n) multiplies exactly rows g*G .. g*G+G-1 of column n."""
    for G in (32, 64, 128):
        K, N = 256, 3
        qw = np.full((K // 8, N), np.uint32(0x99999999).view(np.int32), dtype=np.int32)  # q=9 -> 1
        sc = np.zeros((K // G, N), dtype=np.uint16)
        for g in range(K // G):
            for n in range(N):
                sc[g, n] = np.float16(2.0 ** (g - n)).view(np.uint16)
        _, w = orc.w4a16_unpack(qw, sc, K, N, G)
        for n in range(N):
            for k in range(K):
                assert w[n, k] == 2.0 ** (k // G - n)


def test_round_trip_random_words(orc):
    rng = np.random.default_rng(7)
    K, N = 64, 48
    words = rng.integers(0, 2**32, size=(K // 8, N), dtype=np.uint64).astype(np.uint32).view(np.int32)
    codes, _ = orc.w4a16_unpack(words, None, K, N, 8, want_weights=False)
    assert np.array_equal(orc.w4a16_pack(codes), words)
    # the input generator's packer is an independent implementation
    assert np.array_equal(synth.pack_codes_gptq(codes), words)
    big = rng.integers(0, 16, size=(40, 8 * 3125), dtype=np.uint8)   # 10^6 codes
    qw = synth.pack_codes_gptq(big)
    back, _ = orc.w4a16_unpack(qw, None, big.shape[1], big.shape[0], 8, want_weights=False)
    assert np.array_equal(back, big)


@pytest.mark.parametrize("scale_bits,factor", [(0x3C00, 1.0), (0x3000, 0.125)])
def test_identity(orc, scale_bits, factor):
    K = N = 512
    G = 128
    codes = np.full((N, K), 8, dtype=np.uint8)
    np.fill_diagonal(codes, 9)
    qw = orc.w4a16_pack(codes)
    sc = np.full((K // G, N), scale_bits, dtype=np.uint16)
    lay = synth.int4_layer(4, K, N, G, seed=3)
    Y = orc.w4a16_gemm(lay.X, qw, sc, 4, N, K, G)
    assert np.array_equal(Y, _bf16_to_f64(lay.X) * factor)


def test_permutation(orc):
    K = N = 256
    G = 64
    perm = np.random.default_rng(5).permutation(N)
    codes = np.full((N, K), 8, dtype=np.uint8)
    codes[np.arange(N), perm] = 9          # column n picks row perm[n] of X^T
    qw = orc.w4a16_pack(codes)
    sc = np.full((K // G, N), 0x3C00, dtype=np.uint16)
    lay = synth.int4_layer(3, K, N, G, seed=4)
    Y = orc.w4a16_gemm(lay.X, qw, sc, 3, N, K, G)
    assert np.array_equal(Y, _bf16_to_f64(lay.X)[:, perm])


def test_exact_integer_regime(orc):
    rng = np.random.default_rng(11)
    M, K, N, G = 5, 384, 64, 64
    xi = rng.integers(-3, 4, size=(M, K))
    X = _f64_to_bf16_bits(xi.astype(np.float64))
    codes = rng.integers(0, 16, size=(N, K), dtype=np.uint8)
    e = rng.integers(-2, 3, size=(K // G, N))               # scale 2^e
    sc = np.array([[np.float16(2.0 ** v) for v in row] for row in e]).view(np.uint16)
    Y = orc.w4a16_gemm(X, orc.w4a16_pack(codes), sc, M, N, K, G)
    for m in range(M):
        for n in range(N):
            # 4 * sum_k x * (q - 8) * 2^e as a Python integer (e >= -2)
            tot = 0
            for k in range(K):
                tot += int(xi[m, k]) * (int(codes[n, k]) - 8) * (2 ** (int(e[k // G, n]) + 2))
            assert Y[m, n] == tot / 4.0


@pytest.mark.parametrize("M", [1, 2, 3, 5, 8, 17, 33])
@pytest.mark.parametrize("N", [64, 128, 192])
@pytest.mark.parametrize("K,G", [(128, 32), (256, 64), (384, 128), (256, 128)])
def test_brute_force_vs_numpy(orc, M, N, K, G):
    lay = synth.int4_layer(M, K, N, G, seed=M * 1000 + N + K + G)
    Y = orc.w4a16_gemm(lay.X, lay.qweight, lay.scales, M, N, K, G)
    W = _numpy_dense_weights(lay.qweight, lay.scales, K, N, G)
    ref = _bf16_to_f64(lay.X) @ W
    err = np.abs(Y - ref).max() / max(np.abs(ref).max(), 1e-300)
    assert err <= 1e-12
    _, w = orc.w4a16_unpack(lay.qweight, lay.scales, K, N, G, want_codes=False)
    assert np.array_equal(w, W.T)


def test_threads_and_sampled_outputs_agree(orc):
    lay = synth.int4_layer(7, 512, 256, 128, seed=21)
    Y1 = orc.w4a16_gemm(lay.X, lay.qweight, lay.scales, 7, 256, 512, 128, nthreads=1)
    Y4 = orc.w4a16_gemm(lay.X, lay.qweight, lay.scales, 7, 256, 512, 128, nthreads=4)
    assert np.array_equal(Y1, Y4)
    rows = [0, 6, 3, 3]
    cols = [0, 255, 17, 128]
    at = orc.w4a16_gemm_at(lay.X, lay.qweight, lay.scales, 7, 256, 512, 128, rows, cols)
    assert np.array_equal(at, Y1[rows, cols])


def test_invalid_arguments(orc):
    lay = synth.int4_layer(1, 128, 64, 64, seed=0)
    with pytest.raises(ValueError):
        orc.w4a16_gemm(lay.X, lay.qweight, lay.scales, 1, 64, 128, 48)   # K % G != 0
    with pytest.raises(ValueError):
        orc.w4a16_gemm_at(lay.X, lay.qweight, lay.scales, 1, 64, 128, 64, [1], [0])  # row out of range


# ------------------------------------------- compressed-tensors export
def test_ct_nibble_order_and_row_index(orc):
    """Word (n, i) of weight_packed[N][K/8] feeds rows 8i..8i+7 of column n,
    least significant nibble first, and nothing else."""
    K, N, G = 32, 6, 32
    for n in range(N):
        for i in range(K // 8):
            wp = np.full((N, K // 8), np.uint32(0x88888888).view(np.int32), dtype=np.int32)
            wp[n, i] = np.uint32(0xFEDCBA98).view(np.int32)
            sc = np.full((N, K // G), 0x3C00, dtype=np.uint16)
            codes, w = orc.w4a16_unpack_ct(wp, sc, K, N, G)
            expect = np.full((N, K), 8, dtype=np.uint8)
            expect[n, 8 * i:8 * i + 8] = [8, 9, 10, 11, 12, 13, 14, 15]
            assert np.array_equal(codes, expect)
            assert np.array_equal(w, expect.astype(np.float64) - 8.0)


def test_ct_scale_index(orc):
    """weight_scale[n][g] multiplies exactly rows g*G .. g*G+G-1 of column n."""
    K, N = 256, 4
    for G in (32, 64, 128):
        for n in range(N):
            for g in range(K // G):
                wp = np.full((N, K // 8), np.uint32(0x99999999).view(np.int32), dtype=np.int32)
                sc = np.full((N, K // G), 0x3C00, dtype=np.uint16)   # 1.0
                sc[n, g] = 0x4400                                   # 4.0
                _, w = orc.w4a16_unpack_ct(wp, sc, K, N, G)
                expect = np.ones((N, K))
                expect[n, g * G:(g + 1) * G] = 4.0
                assert np.array_equal(w, expect)


def test_ct_equals_gptq_of_transposed_words(orc):
    """The export is the GPTQ words and scales transposed: both unpackers
    (written separately) agree on random words."""
    rng = np.random.default_rng(5)
    for K, N, G in [(64, 64, 32), (256, 96, 64), (512, 40, 128)]:
        qw = rng.integers(0, 2**32, size=(K // 8, N), dtype=np.uint64).astype(np.uint32).view(np.int32)
        sc = (np.abs(rng.standard_normal((K // G, N))) * 0.01 + 1e-3).astype(np.float16).view(np.uint16)
        c1, w1 = orc.w4a16_unpack(qw, sc, K, N, G)
        c2, w2 = orc.w4a16_unpack_ct(np.ascontiguousarray(qw.T), np.ascontiguousarray(sc.T), K, N, G)
        assert np.array_equal(c1, c2) and np.array_equal(w1, w2)
        assert np.array_equal(w2, _numpy_dense_weights(qw, sc, K, N, G).T)
