"""GPU parity of the weight tools and the small-M (weight-streaming) path,
through the C ABI, against the CPU oracle."""
import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import (assert_parity, assert_sampled_parity, bf16_tensor, bits_of_bf16, to_f64)

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda", 0)


@pytest.fixture(scope="module")
def mxg():
    import __graft_entry__
    __graft_entry__.build()
    import mxfp8_gemm_speculative_b200 as m
    return m


def int4_device(lay):
    qw = torch.from_numpy(lay.qweight).to(DEV)
    sc = torch.from_numpy(lay.scales.view(np.int16)).to(DEV)
    return qw, sc


def run_int4(mxg, lay, path=0):
    qw, sc = int4_device(lay)
    packed = mxg.w4a16_repack(qw, sc, lay.group_size)
    y = mxg.w4a16_gemm(bf16_tensor(lay.X, DEV), packed, lay.N, lay.K, lay.group_size, path=path)
    return y, packed


# --------------------------------------------------------------- weight tools
@pytest.mark.parametrize("K,N,G", [(512, 512, 128), (1024, 192, 64), (256, 320, 32), (384, 64, 128)])
def test_repack_unpack_bit_exact(mxg, K, N, G):
    lay = synth.int4_layer(1, K, N, G, seed=K + N + G)
    qw, sc = int4_device(lay)
    packed = mxg.w4a16_repack(qw, sc, G)
    assert packed.numel() == mxg.w4a16_packed_bytes(K, N, G)
    codes, w32, w16 = mxg.w4a16_unpack(packed, K, N, G)
    ocodes, ow = oracle.w4a16_unpack(lay.qweight, lay.scales, K, N, G)
    assert np.array_equal(codes.cpu().numpy(), ocodes)
    assert np.array_equal(w32.cpu().numpy().astype(np.float64), ow)     # exact in fp32
    want16 = oracle.round_bf16_array(ow)
    assert np.array_equal(bits_of_bf16(w16), want16)


def test_unpack_every_scale_pattern(mxg):
    """All finite positive fp16 scales, every code: the bf16 dequant rounds once."""
    K, N, G = 64, 64, 32
    rng = np.random.default_rng(0)
    all_pos = np.arange(1, 0x7C00, dtype=np.uint16)           # positive finite fp16
    for start in range(0, all_pos.size, (K // G) * N):
        chunk = all_pos[start:start + (K // G) * N]
        sc = np.resize(chunk, (K // G) * N).reshape(K // G, N).astype(np.uint16)
        codes = rng.integers(0, 16, size=(N, K), dtype=np.uint8)
        lay = synth.Int4Layer(1, K, N, G, np.zeros((1, K), np.uint16), codes,
                              synth.pack_codes_gptq(codes), sc)
        qw, scd = int4_device(lay)
        packed = mxg.w4a16_repack(qw, scd, G)
        _, w32, w16 = mxg.w4a16_unpack(packed, K, N, G)
        _, ow = oracle.w4a16_unpack(lay.qweight, sc, K, N, G)
        assert np.array_equal(w32.cpu().numpy().astype(np.float64), ow)
        assert np.array_equal(bits_of_bf16(w16), oracle.round_bf16_array(ow)), start


@pytest.mark.parametrize("E", [100, 119, 121, 123, 127, 140])
def test_mxfp8_dequant_bit_exact(mxg, E):
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    N, K = 128, 256
    Wq = np.resize(codes, N * K).reshape(N, K).astype(np.uint8)
    Ws = np.full((N, K // 32), E, dtype=np.uint8)
    Ws[::3] = np.uint8(E - 2)
    w16 = mxg.mxfp8_dequant(torch.from_numpy(Wq).to(DEV), torch.from_numpy(Ws).to(DEV))
    ow = oracle.mxfp8_dequant(Wq, Ws, N, K)
    assert np.array_equal(bits_of_bf16(w16), oracle.round_bf16_array(ow))


# ------------------------------------------------------------ INT4 streaming
M_STREAM = [1, 2, 3, 4, 5, 8, 16, 17, 31, 32]


@pytest.mark.parametrize("M", M_STREAM)
@pytest.mark.parametrize("K,N,G", [(512, 512, 128), (1024, 192, 64), (256, 320, 32), (1280, 640, 128)])
def test_int4_stream_parity(mxg, M, K, N, G):
    lay = synth.int4_layer(M, K, N, G, seed=7 * M + K + N + G)
    y, _ = run_int4(mxg, lay, path=1)
    ref = oracle.w4a16_gemm(lay.X, lay.qweight, lay.scales, M, N, K, G)
    assert_parity(to_f64(y), ref, f"int4 stream M={M} K={K} N={N} G={G}")


@pytest.mark.parametrize("M", [1, 5, 8, 13, 32])
@pytest.mark.parametrize("G", [32, 64, 128])
def test_int4_stream_exact_integer_regime(mxg, M, G):
    rng = np.random.default_rng(M + G)
    K, N = 1024, 256
    xi = rng.integers(-3, 4, size=(M, K)).astype(np.float32)
    X = torch.from_numpy(xi).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    codes = rng.integers(0, 16, size=(N, K), dtype=np.uint8)
    e = rng.integers(-2, 3, size=(K // G, N))
    sc = np.array([[np.float16(2.0 ** v) for v in row] for row in e]).view(np.uint16)
    lay = synth.Int4Layer(M, K, N, G, X, codes, synth.pack_codes_gptq(codes), sc)
    y, _ = run_int4(mxg, lay, path=1)
    ref = oracle.w4a16_gemm(X, lay.qweight, sc, M, N, K, G)
    want = oracle.round_bf16_array(ref).reshape(M, N)
    assert np.array_equal(bits_of_bf16(y), want)


def test_int4_identity_is_exact(mxg):
    """W = identity / 8 with small-integer activations: every product and
    every partial sum of the weight-streaming path is exact in fp32, so Y is
    X / 8 bit for bit (no weight is rounded anywhere on the path)."""
    K = N = 512
    codes = np.full((N, K), 8, dtype=np.uint8)
    np.fill_diagonal(codes, 9)
    sc = np.full((K // 128, N), 0x3000, dtype=np.uint16)   # 2^-3
    rng = np.random.default_rng(np.random.SeedSequence([1, 7]))
    xi = rng.integers(-8, 9, size=(7, K)).astype(np.float32)
    X = (torch.from_numpy(xi).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16))
    lay = synth.Int4Layer(7, K, N, 128, X, codes, synth.pack_codes_gptq(codes), sc)
    y, _ = run_int4(mxg, lay, path=1)
    xin = torch.from_numpy(X.view(np.int16)).view(torch.bfloat16).float() * 0.125
    assert np.array_equal(bits_of_bf16(y), bits_of_bf16(xin.to(torch.bfloat16)))


def test_int4_tiny_layer_config(mxg):
    """M=1, K=N=512, group 128, seed 0: the tiny workload, in full."""
    lay = synth.int4_layer(1, 512, 512, 128, seed=0)
    y, _ = run_int4(mxg, lay)
    ref = oracle.w4a16_gemm(lay.X, lay.qweight, lay.scales, 1, 512, 512, 128)
    assert_parity(to_f64(y), ref, "tiny layer")


def test_int4_deterministic_and_workspace_restored(mxg):
    lay = synth.int4_layer(5, 2048, 1024, 128, seed=3)
    qw, sc = int4_device(lay)
    packed = mxg.w4a16_repack(qw, sc, 128)
    ws = torch.zeros(mxg.w4a16_workspace_bytes(5, 1024, 2048, 128), dtype=torch.uint8, device=DEV)
    x = bf16_tensor(lay.X, DEV)
    y1 = mxg.w4a16_gemm(x, packed, 1024, 2048, 128, workspace_buf=ws)
    y2 = mxg.w4a16_gemm(x, packed, 1024, 2048, 128, workspace_buf=ws)
    torch.cuda.synchronize()
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))
    # the header (status word) and the arrival counters are zero again; the
    # partial-sum region after them is scratch
    counters_end = 256 + ((1024 // 16) * 4 + 255) // 256 * 256
    assert int(ws[:counters_end].count_nonzero()) == 0
    assert mxg.mxg_workspace_status(ws) == 0
    # scratch left over from another shape does not leak into the result
    ws[counters_end:] = 0x7F
    y3 = mxg.w4a16_gemm(x, packed, 1024, 2048, 128, workspace_buf=ws)
    assert torch.equal(y1.view(torch.int16), y3.view(torch.int16))


@pytest.mark.parametrize("li", [0, 1, 2])
def test_int4_mtp4_verify_layers_sampled(mxg, li):
    """The three MTP4 verify-chunk layers at full size (M=5): sampled outputs."""
    K, N = synth.MTP4_VERIFY_LAYERS[li]
    lay = synth.int4_layer(5, K, N, 128, seed=0, layer=li)
    y, _ = run_int4(mxg, lay)
    yf = to_f64(y)
    rng = np.random.default_rng(li)
    rows = rng.integers(0, 5, size=512)
    cols = rng.integers(0, N, size=512)
    ref = oracle.w4a16_gemm_at(lay.X, lay.qweight, lay.scales, 5, N, K, 128, rows, cols,
                               nthreads=oracle.threads(64))
    rms = float(np.sqrt(np.mean(ref ** 2)))
    assert_sampled_parity(yf[rows, cols], ref, rms, f"MTP4 layer {li}")
    # every column tile is written: no output left unset
    assert np.isfinite(yf).all()


# ------------------------------------------------------------ MXFP8 streaming
@pytest.mark.parametrize("M", [1, 4, 5, 16, 17, 32])
@pytest.mark.parametrize("N,K", [(128, 64), (130, 96), (256, 512), (1000, 2080)])
def test_mxfp8_stream_parity(mxg, M, N, K):
    lay = synth.mxfp8_layer(M, K, N, seed=M + N + K)
    y = mxg.mxfp8_gemm(bf16_tensor(lay.X, DEV), torch.from_numpy(lay.Wq).to(DEV),
                       torch.from_numpy(lay.Ws).to(DEV), path=1)
    ref = oracle.mxfp8_gemm(lay.X, lay.Wq, lay.Ws, M, N, K)
    assert_parity(to_f64(y), ref, f"mxfp8 stream M={M} N={N} K={K}")


def test_mxfp8_identity_is_exact(mxg):
    K = N = 256
    Wq = np.zeros((N, K), dtype=np.uint8)
    np.fill_diagonal(Wq, 0x38)
    Ws = np.full((N, K // 32), 124, dtype=np.uint8)
    X = synth.mxfp8_layer(3, K, N, seed=2).X
    y = mxg.mxfp8_gemm(bf16_tensor(X, DEV), torch.from_numpy(Wq).to(DEV), torch.from_numpy(Ws).to(DEV))
    xin = torch.from_numpy(X.view(np.int16)).view(torch.bfloat16).float() * 0.125
    assert np.array_equal(bits_of_bf16(y), bits_of_bf16(xin.to(torch.bfloat16)))


def test_mxfp8_m4_full_size_sampled(mxg):
    M, K, N = 4, 5120, 17408
    lay = synth.mxfp8_layer(M, K, N, seed=0)
    y = mxg.mxfp8_gemm(bf16_tensor(lay.X, DEV), torch.from_numpy(lay.Wq).to(DEV),
                       torch.from_numpy(lay.Ws).to(DEV))
    yf = to_f64(y)
    rng = np.random.default_rng(5)
    rows = rng.integers(0, M, size=512)
    cols = rng.integers(0, N, size=512)
    ref = oracle.mxfp8_gemm_at(lay.X, lay.Wq, lay.Ws, M, N, K, rows, cols,
                               nthreads=oracle.threads(64))
    rms = float(np.sqrt(np.mean(ref ** 2)))
    assert_sampled_parity(yf[rows, cols], ref, rms, "mxfp8 M=4 full size")
    assert np.isfinite(yf).all()


# --------------------------------------------------------- failure handling
def test_bounded_wait_reports_timeout(mxg):
    ws = torch.zeros(4096, dtype=torch.uint8, device=DEV)
    mxg.mxg_selftest_wait_timeout(ws, 2000)       # 2 ms limit on a wait nothing completes
    assert mxg.mxg_workspace_status(ws) == mxg.MXG_ERR_TIMEOUT
    # the context is still usable
    lay = synth.int4_layer(2, 512, 512, 128, seed=9)
    y, _ = run_int4(mxg, lay)
    ref = oracle.w4a16_gemm(lay.X, lay.qweight, lay.scales, 2, 512, 512, 128)
    assert_parity(to_f64(y), ref, "after timeout")


def test_workspace_too_small_rejected(mxg):
    lay = synth.int4_layer(5, 1024, 512, 128, seed=1)
    qw, sc = int4_device(lay)
    packed = mxg.w4a16_repack(qw, sc, 128)
    ws = torch.zeros(256, dtype=torch.uint8, device=DEV)
    with pytest.raises(mxg.MxgError) as e:
        mxg.w4a16_gemm(bf16_tensor(lay.X, DEV), packed, 512, 1024, 128, workspace_buf=ws)
    assert e.value.status == mxg.MXG_ERR_WORKSPACE


def test_prepared_calls_match_direct_calls(mxg):
    """prepare_w4a16_gemm / prepare_mxfp8_gemm marshal once; each call reads the
    buffers' current contents, so refilling x between calls behaves like a
    fresh direct call."""
    lay = synth.int4_layer(5, 1024, 512, 128, seed=21)
    qw, sc = int4_device(lay)
    packed = mxg.w4a16_repack(qw, sc, 128)
    x = bf16_tensor(lay.X, DEV)
    call, y = mxg.prepare_w4a16_gemm(x, packed, 512, 1024, 128)
    for step in range(2):
        if step:
            x.copy_(torch.randn_like(x, dtype=torch.float32).to(torch.bfloat16))
        call()
        ref = mxg.w4a16_gemm(x, packed, 512, 1024, 128)
        torch.cuda.synchronize()
        assert torch.equal(y.view(torch.int16), ref.view(torch.int16))
    mlay = synth.mxfp8_layer(4, 512, 256, seed=22)
    wq, ws = torch.from_numpy(mlay.Wq).to(DEV), torch.from_numpy(mlay.Ws).to(DEV)
    xm = bf16_tensor(mlay.X, DEV)
    mcall, ym = mxg.prepare_mxfp8_gemm(xm, wq, ws)
    mcall()
    mref = mxg.mxfp8_gemm(xm, wq, ws)
    torch.cuda.synchronize()
    assert torch.equal(ym.view(torch.int16), mref.view(torch.int16))


def test_early_weight_loads_match_late_loads(mxg):
    """Weight tiles loaded before the wait for the previous kernel give the
    same bits as loads after it; a GEMM issued right after w4a16_repack
    re-packs new weights into a reused buffer and sees the new weights."""
    lay = synth.int4_layer(5, 2048, 1024, 128, seed=31)
    lay2 = synth.int4_layer(5, 2048, 1024, 128, seed=32)
    qw, sc = int4_device(lay)
    qw2, sc2 = int4_device(lay2)
    x = bf16_tensor(lay.X, DEV)
    packed = mxg.w4a16_repack(qw, sc, 128)
    outs = {}
    for early in (1, 0):
        late = not early
        y1 = mxg.w4a16_gemm(x, packed, 1024, 2048, 128, late_weights=late)
        # re-pack other weights into the same buffer, GEMM right after
        mxg.w4a16_repack(qw2, sc2, 128, out=packed)
        y2 = mxg.w4a16_gemm(x, packed, 1024, 2048, 128, late_weights=late)
        mxg.w4a16_repack(qw, sc, 128, out=packed)
        torch.cuda.synchronize()
        outs[early] = (y1, y2)
    for a, b in zip(outs[1], outs[0]):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    ref2 = oracle.w4a16_gemm(lay.X, lay2.qweight, lay2.scales, 5, 1024, 2048, 128)
    assert_parity(to_f64(outs[1][1]), ref2, "GEMM right after re-pack")
    mlay = synth.mxfp8_layer(4, 512, 256, seed=33)
    wq, ws = torch.from_numpy(mlay.Wq).to(DEV), torch.from_numpy(mlay.Ws).to(DEV)
    xm = bf16_tensor(mlay.X, DEV)
    mouts = [mxg.mxfp8_gemm(xm, wq, ws, late_weights=late) for late in (False, True)]
    torch.cuda.synchronize()
    assert torch.equal(mouts[0].view(torch.int16), mouts[1].view(torch.int16))


@pytest.mark.parametrize("K,N,G", [(512, 512, 128), (1024, 192, 64), (256, 320, 32)])
def test_repack_ct_matches_gptq_repack(mxg, K, N, G):
    """The compressed-tensors export (words [N][K/8], scales [N][K/G]: the
    GPTQ ones transposed) re-packs to the same bytes, and a GEMM on it
    matches the oracle's unpack of the export."""
    lay = synth.int4_layer(4, K, N, G, seed=K + 3 * N + G)
    qw, sc = int4_device(lay)
    ref = mxg.w4a16_repack(qw, sc, G)
    wp = torch.from_numpy(np.ascontiguousarray(lay.qweight.T)).to(DEV)
    ws = torch.from_numpy(np.ascontiguousarray(lay.scales.T).view(np.int16)).to(DEV)
    packed = mxg.w4a16_repack_ct(wp, ws, G)
    torch.cuda.synchronize()
    assert torch.equal(packed, ref)
    _, w = oracle.w4a16_unpack_ct(np.ascontiguousarray(lay.qweight.T),
                                  np.ascontiguousarray(lay.scales.T), K, N, G)
    y = mxg.w4a16_gemm(bf16_tensor(lay.X, DEV), packed, N, K, G)
    x64 = (lay.X.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    assert_parity(to_f64(y), x64 @ w.T, "compressed-tensors GEMM")


@pytest.mark.parametrize("K,Ns,G,M", [(512, (256, 128, 128), 128, 5), (1024, (192, 192), 64, 16),
                                      (256, (64, 320), 32, 40)])
def test_repack_fused_matches_concatenated_repack(mxg, K, Ns, G, M):
    """A fused buffer of several projections (same K) is byte for byte the
    re-pack of their words and scales concatenated along N, and one GEMM on it
    (weight streaming, or tensor cores for M = 40) matches the oracle for
    every part."""
    lays = [synth.int4_layer(M, K, n, G, seed=100 * i + n + K) for i, n in enumerate(Ns)]
    parts = [int4_device(lay) for lay in lays]
    fused = mxg.w4a16_repack_fused(parts, G)
    qcat = torch.cat([qw for qw, _ in parts], dim=1).contiguous()
    scat = torch.cat([sc for _, sc in parts], dim=1).contiguous()
    ref = mxg.w4a16_repack(qcat, scat, G)
    torch.cuda.synchronize()
    assert torch.equal(fused, ref)
    N = sum(Ns)
    y = to_f64(mxg.w4a16_gemm(bf16_tensor(lays[0].X, DEV), fused, N, K, G))
    n0 = 0
    for lay, n in zip(lays, Ns):
        want = oracle.w4a16_gemm(lays[0].X, lay.qweight, lay.scales, M, n, K, G)
        assert_parity(y[:, n0:n0 + n], want, f"fused part at column {n0}")
        n0 += n


def test_tensor_parallel_shards_on_one_gpu(mxg):
    """Column and row shards of one layer (as two ranks would hold them),
    re-packed and run one after the other on this GPU: the column blocks are
    the layer's columns, the row partials add up to the layer (the sum that
    the row-parallel all-reduce does across GPUs is done here on the host)."""
    from mxfp8_gemm_speculative_b200 import tp
    M, K, N, G, P = 5, 2048, 1024, 128, 2
    lay = synth.int4_layer(M, K, N, G, seed=12)
    qw, sc = int4_device(lay)
    x = bf16_tensor(lay.X, DEV)
    ref = oracle.w4a16_gemm(lay.X, lay.qweight, lay.scales, M, N, K, G)
    cols = []
    for r in range(P):
        q, s, n0, n1 = tp.column_shard(qw, sc, r, P)
        packed = mxg.w4a16_repack(q.contiguous(), s.contiguous(), G)
        cols.append(to_f64(mxg.w4a16_gemm(x, packed, n1 - n0, K, G)))
    assert_parity(np.concatenate(cols, axis=1), ref, "column-parallel shards")
    total = np.zeros((M, N))
    for r in range(P):
        q, s, k0, k1 = tp.row_shard(qw, sc, G, r, P)
        packed = mxg.w4a16_repack(q.contiguous(), s.contiguous(), G)
        y = tp.row_parallel_w4a16_gemm(x[:, k0:k1].contiguous(), packed, N, k1 - k0, G)
        total += to_f64(y)
    assert_parity(total, ref, "row-parallel shards")
