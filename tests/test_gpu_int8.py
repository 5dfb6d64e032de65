"""GPU parity of the INT8 W8A16 weight-streaming path (the vocabulary head)
through the C ABI, against the CPU oracle."""
import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import assert_parity, assert_sampled_parity, bits_of_bf16, bf16_tensor, to_f64

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda", 0)


@pytest.fixture(scope="module")
def mxg():
    import __graft_entry__
    __graft_entry__.build()
    import mxfp8_gemm_speculative_b200 as m
    return m


def _run(mxg, lay, X=None):
    qw = torch.from_numpy(lay.qweight).to(DEV)
    sc = torch.from_numpy(lay.scales.view(np.int16)).to(DEV)
    packed = mxg.w8a16_repack(qw, sc, lay.group_size)
    assert packed.numel() == mxg.raw_lib().w8a16_packed_bytes(lay.K, lay.N, lay.group_size)
    x = bf16_tensor(lay.X if X is None else X, DEV)
    return mxg.w8a16_gemm(x, packed, lay.N, lay.K, lay.group_size)


@pytest.mark.parametrize("M", [1, 5, 8, 16, 17, 32])
@pytest.mark.parametrize("K,N,G", [(512, 512, 128), (1024, 192, 64), (256, 320, 32)])
def test_int8_stream_parity(mxg, M, K, N, G):
    lay = synth.int8_layer(M, K, N, G, seed=M + K + N + G)
    y = _run(mxg, lay)
    ref = oracle.w8a16_gemm(lay.X, lay.qweight, lay.scales, M, N, K, G)
    assert_parity(to_f64(y), ref, f"int8 M={M} K={K} N={N} G={G}")


@pytest.mark.parametrize("M", [1, 5, 32])
@pytest.mark.parametrize("G", [32, 128])
def test_int8_exact_integer_regime(mxg, M, G):
    """Small-integer activations, power-of-two scales: every product and
    partial sum is exact in fp32, so Y equals the rounded oracle bit for bit."""
    rng = np.random.default_rng(M + 3 * G)
    K, N = 512, 128
    lay = synth.int8_layer(M, K, N, G, seed=G)
    xi = rng.integers(-3, 4, size=(M, K)).astype(np.float32)
    X = torch.from_numpy(xi).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    e = rng.integers(-9, -6, size=(K // G, N))
    sc = np.array([[np.float16(2.0 ** v) for v in row] for row in e]).view(np.uint16)
    lay = synth.Int8Layer(M, K, N, G, X, lay.codes, lay.qweight, sc)
    y = _run(mxg, lay)
    ref = oracle.w8a16_gemm(X, lay.qweight, sc, M, N, K, G)
    assert np.array_equal(bits_of_bf16(y), oracle.round_bf16_array(ref).reshape(M, N))


def test_int8_vocab_head_sampled(mxg):
    """The vocabulary head at full size (M = 5, K = 5120, N = 248320, g128):
    sampled outputs against the oracle, every output finite."""
    M, K, N, G = 5, 5120, 248320, 128
    lay = synth.int8_layer(M, K, N, G, seed=0)
    y = to_f64(_run(mxg, lay))
    rng = np.random.default_rng(8)
    cols = np.unique(rng.integers(0, N, size=256))
    ref = oracle.w8a16_gemm(lay.X, np.ascontiguousarray(lay.qweight[:, cols]),
                            np.ascontiguousarray(lay.scales[:, cols]), M, len(cols), K, G,
                            nthreads=oracle.threads(64))
    rms = float(np.sqrt(np.mean(ref ** 2)))
    assert_sampled_parity(y[:, cols].ravel(), ref.ravel(), rms, "INT8 head")
    assert np.isfinite(y).all()


@pytest.mark.parametrize("K,N,G", [(512, 512, 128), (1024, 192, 64), (256, 320, 32)])
def test_int8_repack_ct_matches(mxg, K, N, G):
    """The compressed-tensors export ([N][K/4] words, [N][K/G] scales: the
    GPTQ-style ones transposed) re-packs to the same bytes."""
    lay = synth.int8_layer(3, K, N, G, seed=K + N)
    qw = torch.from_numpy(lay.qweight).to(DEV)
    sc = torch.from_numpy(lay.scales.view(np.int16)).to(DEV)
    ref = mxg.w8a16_repack(qw, sc, G)
    wp = torch.from_numpy(np.ascontiguousarray(lay.qweight.T)).to(DEV)
    ws = torch.from_numpy(np.ascontiguousarray(lay.scales.T).view(np.int16)).to(DEV)
    packed = mxg.w8a16_repack_ct(wp, ws, G)
    torch.cuda.synchronize()
    assert torch.equal(packed, ref)
