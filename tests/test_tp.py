"""Tensor-parallel sharding of the INT4 layer (host logic), on CPU with two
gloo ranks (127.0.0.1) and the oracle as each rank's local GEMM.

* column-parallel: the ranks' column blocks of Y, side by side, are the full
  layer's Y exactly (same sums, same order);
* row-parallel: the ranks' partial outputs summed by one all-reduce equal the
  full layer's Y (fp64, to rounding);
* shard boundaries keep the kernels' shape rules (multiples of 64 and of G).
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _load_tp():
    # the sharding helpers need no GPU and no compiled library
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "mxg_tp", os.path.join(ROOT, "mxfp8_gemm_speculative_b200", "tp.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def _worker(rank, world, port, out):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import oracle
    import synth
    tp = _load_tp()
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        M, K, N, G = 5, 1024, 512, 128
        lay = synth.int4_layer(M, K, N, G, seed=3)
        # column-parallel
        qc, sc, n0, n1 = tp.column_shard(lay.qweight, lay.scales, rank, world)
        yc = oracle.w4a16_gemm(lay.X, np.ascontiguousarray(qc), np.ascontiguousarray(sc), M,
                               n1 - n0, K, G)
        # row-parallel: the rank's rows of W and columns of X, then one all-reduce
        qr, sr, k0, k1 = tp.row_shard(lay.qweight, lay.scales, G, rank, world)
        xr = np.ascontiguousarray(lay.X[:, k0:k1])
        yr = oracle.w4a16_gemm(xr, np.ascontiguousarray(qr), np.ascontiguousarray(sr), M, N,
                               k1 - k0, G)
        t = torch.from_numpy(yr.copy())
        tp.all_reduce_sum(t)
        # the same partial as the GEMM returns it (bf16), reduced in fp32
        tb = torch.from_numpy(yr.copy()).to(torch.bfloat16)
        tp.all_reduce_sum(tb)
        out[rank] = (n0, n1, yc, t.numpy(), k0, k1, tb.float().numpy(), yr)
    finally:
        dist.destroy_process_group()


def test_column_and_row_parallel_gloo():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_worker, args=(world, port, out), nprocs=world, join=True,
                           start_method="spawn")
        res = dict(out)
    sys.path.insert(0, ROOT)
    import oracle
    import synth
    M, K, N, G = 5, 1024, 512, 128
    lay = synth.int4_layer(M, K, N, G, seed=3)
    full = oracle.w4a16_gemm(lay.X, lay.qweight, lay.scales, M, N, K, G)
    cols = np.concatenate([res[r][2] for r in range(world)], axis=1)
    assert [(res[r][0], res[r][1]) for r in range(world)] == [(0, 256), (256, 512)]
    assert np.array_equal(cols, full)
    assert [(res[r][4], res[r][5]) for r in range(world)] == [(0, 512), (512, 1024)]
    for r in range(world):
        assert np.allclose(res[r][3], full, rtol=1e-12, atol=1e-12)
    # bf16 partials: the all-reduce adds them in fp32 and rounds once, so the
    # result is the bf16 nearest of the exact sum of the rounded partials
    parts = [torch.from_numpy(res[r][7]).to(torch.bfloat16).double() for r in range(world)]
    expect = (parts[0] + parts[1]).to(torch.bfloat16).float().numpy()
    for r in range(world):
        assert np.array_equal(res[r][6], expect)


def test_shard_boundaries_follow_the_shape_rules():
    tp = _load_tp()
    qw = np.zeros((17408 // 8, 5120), dtype=np.int32)
    sc = np.zeros((17408 // 128, 5120), dtype=np.uint16)
    for world in (1, 2, 4, 8):
        for r in range(world):
            q, s, n0, n1 = tp.column_shard(qw, sc, r, world)
            assert (n1 - n0) % 64 == 0 and q.shape == (17408 // 8, n1 - n0)
    # K = 17408 = 136 groups of 128: 2, 4 and 8 ranks get whole groups
    for world in (2, 4, 8):
        q, s, k0, k1 = tp.row_shard(qw, sc, 128, world - 1, world)
        assert (k1 - k0) % 128 == 0 and k1 == 17408 and s.shape[0] == (k1 - k0) // 128
    with pytest.raises(ValueError):
        tp.column_shard(qw[:, :96], sc[:, :96], 0, 2)          # 48 columns per rank
    with pytest.raises(ValueError):
        tp.row_shard(qw[:64], sc[:4], 128, 0, 3)              # 512 rows into 3 ranks
