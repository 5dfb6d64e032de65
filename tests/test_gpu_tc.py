"""GPU parity of the tensor-core (tcgen05) path, through the C ABI, against
the CPU oracle."""
import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import assert_parity, assert_sampled_parity, bf16_tensor, bits_of_bf16, to_f64

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda", 0)


@pytest.fixture(scope="module")
def mxg():
    import __graft_entry__
    __graft_entry__.build()
    import mxfp8_gemm_speculative_b200 as m
    return m


def int4_gemm(mxg, lay, path):
    qw = torch.from_numpy(lay.qweight).to(DEV)
    sc = torch.from_numpy(lay.scales.view(np.int16)).to(DEV)
    packed = mxg.w4a16_repack(qw, sc, lay.group_size)
    y = mxg.w4a16_gemm(bf16_tensor(lay.X, DEV), packed, lay.N, lay.K, lay.group_size, path=path)
    assert mxg.mxg_workspace_status(mxg.workspace(0)) == 0
    return y


def mxfp8_gemm(mxg, lay, path):
    y = mxg.mxfp8_gemm(bf16_tensor(lay.X, DEV), torch.from_numpy(lay.Wq).to(DEV),
                       torch.from_numpy(lay.Ws).to(DEV), path=path)
    assert mxg.mxg_workspace_status(mxg.workspace(0)) == 0
    return y


@pytest.mark.parametrize("M", [1, 5, 33, 64, 100, 128, 129, 256, 300])
@pytest.mark.parametrize("K,N,G", [(512, 512, 128), (1024, 768, 64), (256, 320, 32), (640, 1280, 128)])
def test_int4_tc_parity(mxg, M, K, N, G):
    lay = synth.int4_layer(M, K, N, G, seed=11 * M + K + N + G)
    y = int4_gemm(mxg, lay, path=2)
    ref = oracle.w4a16_gemm(lay.X, lay.qweight, lay.scales, M, N, K, G)
    assert_parity(to_f64(y), ref, f"int4 tc M={M} K={K} N={N} G={G}")


@pytest.mark.parametrize("M", [7, 128, 200])
@pytest.mark.parametrize("G", [32, 64, 128])
def test_int4_tc_exact_integer_regime(mxg, M, G):
    rng = np.random.default_rng(100 + M + G)
    K, N = 1024, 512
    xi = rng.integers(-3, 4, size=(M, K)).astype(np.float32)
    X = torch.from_numpy(xi).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    codes = rng.integers(0, 16, size=(N, K), dtype=np.uint8)
    e = rng.integers(-2, 3, size=(K // G, N))
    sc = np.array([[np.float16(2.0 ** v) for v in row] for row in e]).view(np.uint16)
    lay = synth.Int4Layer(M, K, N, G, X, codes, synth.pack_codes_gptq(codes), sc)
    y = int4_gemm(mxg, lay, path=2)
    ref = oracle.w4a16_gemm(X, lay.qweight, sc, M, N, K, G)
    assert np.array_equal(bits_of_bf16(y), oracle.round_bf16_array(ref).reshape(M, N))


def test_int4_tc_identity_is_exact(mxg):
    K = N = 512
    M = 160
    codes = np.full((N, K), 8, dtype=np.uint8)
    np.fill_diagonal(codes, 9)
    sc = np.full((K // 128, N), 0x3C00, dtype=np.uint16)
    X = synth.int4_layer(M, K, N, 128, seed=4).X
    lay = synth.Int4Layer(M, K, N, 128, X, codes, synth.pack_codes_gptq(codes), sc)
    y = int4_gemm(mxg, lay, path=2)
    assert np.array_equal(bits_of_bf16(y), X)


@pytest.mark.parametrize("li", [0, 1])
def test_int4_c32_mtp3_layers_sampled(mxg, li):
    """M = 128 (32 streams x (1 + 3)) on both C32 layers, full size, sampled."""
    K, N = synth.C32_MTP3_LAYERS[li]
    lay = synth.int4_layer(128, K, N, 128, seed=0, layer=li)
    y = to_f64(int4_gemm(mxg, lay, path=0))
    rng = np.random.default_rng(li)
    rows = rng.integers(0, 128, size=512)
    cols = rng.integers(0, N, size=512)
    ref = oracle.w4a16_gemm_at(lay.X, lay.qweight, lay.scales, 128, N, K, 128, rows, cols,
                               nthreads=oracle.threads(64))
    assert_sampled_parity(y[rows, cols], ref, float(np.sqrt(np.mean(ref ** 2))), f"C32 layer {li}")
    assert np.isfinite(y).all()


def test_int4_prefill_chunk_sampled(mxg):
    """M = 8192, K = 5120, N = 17408: the tensor-core-bound prefill chunk, sampled."""
    M, K, N = 8192, 5120, 17408
    lay = synth.int4_layer(M, K, N, 128, seed=0)
    y = int4_gemm(mxg, lay, path=0)
    rng = np.random.default_rng(8192)
    rows = rng.integers(0, M, size=256)
    cols = rng.integers(0, N, size=256)
    # corners of the output: first/last tile rows and columns
    rows = np.concatenate([rows, [0, 0, M - 1, M - 1, 127, 128]])
    cols = np.concatenate([cols, [0, N - 1, 0, N - 1, 255, 256]])
    ref = oracle.w4a16_gemm_at(lay.X, lay.qweight, lay.scales, M, N, K, 128, rows, cols,
                               nthreads=oracle.threads(64))
    ys = to_f64(y[torch.from_numpy(rows).to(DEV), torch.from_numpy(cols).to(DEV)])
    assert_sampled_parity(ys, ref, float(np.sqrt(np.mean(ref ** 2))), "prefill")
    assert bool(torch.isfinite(y.float()).all())


@pytest.mark.parametrize("M", [1, 33, 128, 200])
@pytest.mark.parametrize("N,K", [(128, 64), (130, 96), (256, 512), (1000, 2080)])
def test_mxfp8_tc_parity(mxg, M, N, K):
    lay = synth.mxfp8_layer(M, K, N, seed=3 * M + N + K)
    y = mxfp8_gemm(mxg, lay, path=2)
    ref = oracle.mxfp8_gemm(lay.X, lay.Wq, lay.Ws, M, N, K)
    assert_parity(to_f64(y), ref, f"mxfp8 tc M={M} N={N} K={K}")


def test_mxfp8_m128_full_size_sampled(mxg):
    M, K, N = 128, 5120, 17408
    lay = synth.mxfp8_layer(M, K, N, seed=0)
    y = to_f64(mxfp8_gemm(mxg, lay, path=0))
    rng = np.random.default_rng(128)
    rows = rng.integers(0, M, size=512)
    cols = rng.integers(0, N, size=512)
    ref = oracle.mxfp8_gemm_at(lay.X, lay.Wq, lay.Ws, M, N, K, rows, cols,
                               nthreads=oracle.threads(64))
    assert_sampled_parity(y[rows, cols], ref, float(np.sqrt(np.mean(ref ** 2))), "mxfp8 M=128")
    assert np.isfinite(y).all()


def test_paths_agree_at_crossover(mxg):
    """M = 32 on both paths: the two paths differ only in rounding order."""
    lay = synth.int4_layer(32, 2048, 1024, 128, seed=32)
    ys = to_f64(int4_gemm(mxg, lay, path=1))
    yt = to_f64(int4_gemm(mxg, lay, path=2))
    ref = oracle.w4a16_gemm(lay.X, lay.qweight, lay.scales, 32, 1024, 2048, 128)
    assert_parity(ys, ref, "stream at M=32")
    assert_parity(yt, ref, "tc at M=32")


@pytest.mark.parametrize("M,K,N", [(128, 4096, 512), (64, 8192, 256), (200, 2048, 768)])
def test_int4_tc_split_k_parity_and_reproducible(mxg, M, K, N):
    """Few output tiles and a long K: the plan splits K across CTA pairs and the
    last split adds the fp32 partials in split order, so two calls give the
    same bits and both are within tolerance."""
    lay = synth.int4_layer(M, K, N, 128, seed=11)
    y1 = int4_gemm(mxg, lay, path=2)
    y2 = int4_gemm(mxg, lay, path=2)
    torch.cuda.synchronize()
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))
    ref = oracle.w4a16_gemm(lay.X, lay.qweight, lay.scales, M, N, K, 128)
    assert_parity(to_f64(y1), ref, f"split-K M={M} K={K} N={N}")
