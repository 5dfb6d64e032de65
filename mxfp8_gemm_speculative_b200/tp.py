"""Tensor parallelism for the INT4 layer across the GPUs of one node.

The Eole Qwen3.8 recipe (section "INT4 tensor parallelism") partitions the
packed GPTQ weights before the kernel re-pack and shards the attention and
MLP projections.  Two partitionings, each followed by w4a16_repack on every
rank:

* column-parallel (split N; e.g. gate/up 5120 -> 17408): rank r owns the
  columns [r N/P, (r+1) N/P) of W and computes those columns of Y; there is
  no exchange for this GEMM (Y stays distributed by columns);
* row-parallel (split K; e.g. down 17408 -> 5120): rank r owns the rows
  [r K/P, (r+1) K/P) of W, its activations are the matching columns of X
  (in a layer pair, exactly the columns the previous column-parallel layer
  left on it), and the partial outputs are summed with one all-reduce of
  M x N (torch.distributed: NCCL over NVLink on GPUs, gloo on CPU).

Shards must keep the kernels' shape rules: N/P a multiple of 64, K/P a
multiple of 64 and of the group size.  The functions take and return plain
tensors (numpy arrays work too for the sharding helpers); only
``row_parallel_w4a16_gemm`` launches the library's kernel.
"""
from __future__ import annotations

import math


def _split(total: int, world: int, quantum: int, what: str) -> int:
    if world < 1 or total % world != 0 or (total // world) % quantum != 0:
        raise ValueError(f"{what}={total} does not split into {world} shards of a multiple of "
                         f"{quantum}")
    return total // world


def column_shard(qweight, scales, rank: int, world: int):
    """Rank ``rank``'s columns of GPTQ qweight[K/8][N] and scales[K/G][N]:
    (qweight_r, scales_r, n0, n1), the shard being columns [n0, n1)."""
    N = qweight.shape[1]
    n = _split(N, world, 64, "N")
    n0, n1 = rank * n, (rank + 1) * n
    return qweight[:, n0:n1], scales[:, n0:n1], n0, n1


def row_shard(qweight, scales, group_size: int, rank: int, world: int):
    """Rank ``rank``'s rows of GPTQ qweight[K/8][N] and scales[K/G][N]:
    (qweight_r, scales_r, k0, k1), the shard being rows [k0, k1) of W (and
    columns [k0, k1) of X)."""
    K = qweight.shape[0] * 8
    quantum = 64 * group_size // math.gcd(64, group_size)
    k = _split(K, world, quantum, "K")
    k0, k1 = rank * k, (rank + 1) * k
    return qweight[k0 // 8:k1 // 8], scales[k0 // group_size:k1 // group_size], k0, k1


def all_reduce_sum(y, group=None):
    """Sum a partial output over the ranks of ``group`` in place (no-op
    without an initialised process group of more than one rank).

    16-bit partials are summed in fp32 and rounded once: each rank's partial
    carries one bf16 rounding from its GEMM's output (at most 2^-9 of its
    magnitude), and a reduction in bf16 would add one rounding per step of
    the collective's reduction tree; in fp32 the sum of P <= 8 bf16 values is
    exact unless their exponents span more than 16 binades."""
    import torch
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        if y.dtype in (torch.bfloat16, torch.float16):
            y32 = y.float()
            dist.all_reduce(y32, op=dist.ReduceOp.SUM, group=group)
            y.copy_(y32)
        else:
            dist.all_reduce(y, op=dist.ReduceOp.SUM, group=group)
    return y


def row_parallel_w4a16_gemm(x_r, packed_r, N: int, K_r: int, group_size: int = 128, group=None,
                            out=None, stream=None):
    """Row-parallel layer: this rank's partial Y = x_r * dequant(W_r)^T over
    its K_r rows (one w4a16_gemm launch), summed over the ranks with one
    all-reduce.  ``x_r`` is bf16 [M][K_r], ``packed_r`` the rank's re-packed
    rows."""
    from . import w4a16_gemm
    y = w4a16_gemm(x_r, packed_r, N, K_r, group_size, out=out, stream=stream)
    return all_reduce_sum(y, group)
