"""Full-size parity of the measured configurations, through the C ABI,
against the CPU oracle on all host cores (the oracle's per-element arithmetic
does not depend on the thread count).

Every output of every layer is compared (the C32 MTP3 chunk, the MTP4
verify layers, MXFP8 at M = 4 and 128, the INT8 vocabulary head); for the
M = 8192 prefill chunk every column of 256 rows that take both sides of every
128-row tile boundary.  Each output buffer is filled with NaN before the
GEMM, so an element the kernels never write fails the comparison.  The
device decode of the re-packed 5120 x 17408 layer is compared with the
oracle's unpack bit for bit.
"""
import os

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


@pytest.fixture(scope="module")
def nthreads():
    oracle.build()
    return oracle.threads(os.cpu_count() or 1)


def poisoned(M, N):
    return torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=DEV)


def int4_packed(mxg, lay):
    return mxg.w4a16_repack(torch.from_numpy(lay.qweight).to(DEV),
                            torch.from_numpy(lay.scales.view(np.int16)).to(DEV), lay.group_size)


@pytest.mark.parametrize("M,K,N", [(5, 5120, 5120), (5, 5120, 17408), (5, 17408, 5120),
                                   (128, 5120, 17408), (128, 17408, 5120)])
def test_int4_every_output(mxg, nthreads, M, K, N):
    lay = synth.int4_layer(M, K, N, 128, seed=100 + M + K // 64 + N // 64)
    y = poisoned(M, N)
    mxg.w4a16_gemm(bf16_tensor(lay.X, DEV), int4_packed(mxg, lay), N, K, 128, out=y)
    ref = oracle.w4a16_gemm(lay.X, lay.qweight, lay.scales, M, N, K, 128, nthreads=nthreads)
    assert_parity(to_f64(y), ref, f"int4 M={M} K={K} N={N} (every output)")


@pytest.mark.parametrize("M", [4, 128])
def test_mxfp8_every_output(mxg, nthreads, M):
    K, N = 5120, 17408
    lay = synth.mxfp8_layer(M, K, N, seed=200 + M)
    y = poisoned(M, N)
    mxg.mxfp8_gemm(bf16_tensor(lay.X, DEV), torch.from_numpy(lay.Wq).to(DEV),
                   torch.from_numpy(lay.Ws).to(DEV), out=y)
    ref = oracle.mxfp8_gemm(lay.X, lay.Wq, lay.Ws, M, N, K, nthreads=nthreads)
    assert_parity(to_f64(y), ref, f"mxfp8 M={M} (every output)")


def test_int8_head_every_output(mxg, nthreads):
    M, K, N, G = 5, 5120, 248320, 128
    lay = synth.int8_layer(M, K, N, G, seed=300)
    packed = mxg.w8a16_repack(torch.from_numpy(lay.qweight).to(DEV),
                              torch.from_numpy(lay.scales.view(np.int16)).to(DEV), G)
    y = poisoned(M, N)
    mxg.w8a16_gemm(bf16_tensor(lay.X, DEV), packed, N, K, G, out=y)
    ref = oracle.w8a16_gemm(lay.X, lay.qweight, lay.scales, M, N, K, G, nthreads=nthreads)
    assert_parity(to_f64(y), ref, "int8 head (every output)")


def prefill_rows(M, tile=128, seed=5):
    """Both rows at every tile boundary, the first and last row, and seeded
    rows in between: 256 rows of the M = 8192 chunk."""
    rows = {0, M - 1}
    for b in range(tile, M, tile):
        rows.update((b - 1, b))
    rng = np.random.default_rng(seed)
    while len(rows) < 256:
        rows.add(int(rng.integers(0, M)))
    return np.array(sorted(rows), dtype=np.int64)


def test_prefill_rows_every_column(mxg, nthreads):
    M, K, N, G = 8192, 5120, 17408, 128
    lay = synth.int4_layer(M, K, N, G, seed=400)
    y = poisoned(M, N)
    mxg.w4a16_gemm(bf16_tensor(lay.X, DEV), int4_packed(mxg, lay), N, K, G, out=y)
    rows = prefill_rows(M)
    assert len(rows) == 256
    xs = np.ascontiguousarray(lay.X[rows])
    ref = oracle.w4a16_gemm(xs, lay.qweight, lay.scales, len(rows), N, K, G, nthreads=nthreads)
    got = to_f64(y[torch.from_numpy(rows).to(DEV)])
    assert_parity(got, ref, "prefill M=8192, 256 rows x every column")
    # the rows not compared were written too
    assert not torch.isnan(y.float()).any()


def test_unpack_config_shape_bit_exact(mxg):
    K, N, G = 5120, 17408, 128
    lay = synth.int4_layer(1, K, N, G, seed=500)
    codes, w32, w16 = mxg.w4a16_unpack(int4_packed(mxg, lay), K, N, G)
    ocodes, ow = oracle.w4a16_unpack(lay.qweight, lay.scales, K, N, G)
    assert np.array_equal(codes.cpu().numpy(), ocodes)
    ow32 = ow.astype(np.float32)
    assert np.array_equal(ow32.astype(np.float64), ow)        # exact in fp32
    assert np.array_equal(w32.cpu().numpy().view(np.uint32), ow32.view(np.uint32))
    # bf16 nearest (ties to even) of the exact weight; the oracle's own
    # rounding routine agrees with torch's cast (pinned in the oracle tests)
    want16 = torch.from_numpy(ow32).to(torch.bfloat16).view(torch.int16).numpy()
    assert np.array_equal(w16.view(torch.int16).cpu().numpy(), want16)
