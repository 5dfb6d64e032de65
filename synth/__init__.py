"""Seeded synthetic inputs for the weight-quantized linear layer.

This module is the only code shared by the CPU oracle side (tests) and the
CUDA side (tests, bench).  It draws random numbers and stores them in the
formats the layer consumes; it holds none of the layer's arithmetic (no
dequantization, no products, no sums).  Rounding into storage formats uses
library casts only: numpy float16 (round to nearest even), torch bfloat16 and
torch float8_e4m3fn (round to nearest even).

Recipes (value distributions of the workloads the layer is measured on):

* INT4 W4A16, symmetric, group G along K: codes q uniform in 0..15, packed 8
  per int32 word along K (code of row k = 8i + j in bits [4j, 4j+3] of word
  (i, n)); scales fp16(1e-3 + 0.01*|z|) per (group, column); X bf16(z);
  z ~ N(0, 1) drawn in float32.
* MXFP8: z ~ N(0, 1) in float32, code = e4m3(z) (round to nearest even), one
  E8M0 exponent per (row, 32-block) uniform in 119..123 (2^-8 .. 2^-4); X as
  above.

* Dense bf16 (the paired GDN A/B projection): W bf16(0.02*z) [N][K], X as
  above.
* INT8 W8A16 (the vocabulary head): codes uniform in 0..255, packed 4 per
  int32 word along K (code of row k = 4i + j in bits [8j, 8j+7] of word
  (i, n)); scales fp16(1e-4 + 0.001*|z|) per (group, column); X as above.

RNG: numpy ``Generator(PCG64)`` seeded from ``SeedSequence([seed, layer])``,
spawned into three independent streams (codes, scales, X).
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch


def _streams(seed: int, layer: int):
    ss = np.random.SeedSequence([int(seed), int(layer)])
    return [np.random.Generator(np.random.PCG64(s)) for s in ss.spawn(3)]


def bf16_bits_of_normals(rng: np.random.Generator, shape) -> np.ndarray:
    """bf16 bit patterns of float32 N(0,1) samples (torch RNE cast)."""
    z = rng.standard_normal(size=shape, dtype=np.float32)
    t = torch.from_numpy(z).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def pack_codes_gptq(codes: np.ndarray) -> np.ndarray:
    """Pack codes[N][K] (0..15) into GPTQ words qweight[K/8][N] (int32)."""
    codes = np.asarray(codes, dtype=np.uint8)
    N, K = codes.shape
    c = codes.T.reshape(K // 8, 8, N).astype(np.uint32)
    words = np.zeros((K // 8, N), dtype=np.uint32)
    for j in range(8):
        words |= c[:, j, :] << np.uint32(4 * j)
    return words.view(np.int32)


@dataclass
class Int4Layer:
    M: int
    K: int
    N: int
    group_size: int
    X: np.ndarray        # uint16 bf16 bits [M][K]
    codes: np.ndarray    # uint8 [N][K], 0..15
    qweight: np.ndarray  # int32 [K/8][N]
    scales: np.ndarray   # uint16 fp16 bits [K/G][N]


@dataclass
class Mxfp8Layer:
    M: int
    K: int
    N: int
    X: np.ndarray        # uint16 bf16 bits [M][K]
    Wq: np.ndarray       # uint8 E4M3 codes [N][K]
    Ws: np.ndarray       # uint8 E8M0 exponents [N][K/32]


def int4_layer(M: int, K: int, N: int, group_size: int = 128, seed: int = 0,
               layer: int = 0) -> Int4Layer:
    r_codes, r_scales, r_x = _streams(seed, layer)
    codes = r_codes.integers(0, 16, size=(N, K), dtype=np.uint8)
    z = r_scales.standard_normal(size=(K // group_size, N), dtype=np.float32)
    scales = (1e-3 + 0.01 * np.abs(z.astype(np.float64))).astype(np.float16)
    X = bf16_bits_of_normals(r_x, (M, K))
    return Int4Layer(M, K, N, group_size, X, codes, pack_codes_gptq(codes),
                     scales.view(np.uint16).copy())


def mxfp8_layer(M: int, K: int, N: int, seed: int = 0, layer: int = 0,
                exp_lo: int = 119, exp_hi: int = 123) -> Mxfp8Layer:
    r_codes, r_scales, r_x = _streams(seed, layer)
    z = r_codes.standard_normal(size=(N, K), dtype=np.float32)
    Wq = torch.from_numpy(z).to(torch.float8_e4m3fn).view(torch.uint8).numpy().copy()
    Ws = r_scales.integers(exp_lo, exp_hi + 1, size=(N, K // 32), dtype=np.uint8)
    X = bf16_bits_of_normals(r_x, (M, K))
    return Mxfp8Layer(M, K, N, X, Wq, Ws)


@dataclass
class Int8Layer:
    M: int
    K: int
    N: int
    group_size: int
    X: np.ndarray        # uint16 bf16 bits [M][K]
    codes: np.ndarray    # uint8 [N][K], 0..255
    qweight: np.ndarray  # int32 [K/4][N]
    scales: np.ndarray   # uint16 fp16 bits [K/G][N]


def int8_layer(M: int, K: int, N: int, group_size: int = 128, seed: int = 0,
               layer: int = 0) -> Int8Layer:
    r_codes, r_scales, r_x = _streams(seed, layer)
    codes = r_codes.integers(0, 256, size=(N, K), dtype=np.uint8)
    z = r_scales.standard_normal(size=(K // group_size, N), dtype=np.float32)
    scales = (1e-4 + 0.001 * np.abs(z.astype(np.float64))).astype(np.float16)
    X = bf16_bits_of_normals(r_x, (M, K))
    # codes[N][K] -> words[K/4][N]: byte j of word (i, n) is code (n, 4i + j)
    qweight = np.ascontiguousarray(codes.T).reshape(K // 4, 4, N).transpose(0, 2, 1)
    qweight = np.ascontiguousarray(qweight).view(np.uint32).reshape(K // 4, N).view(np.int32)
    return Int8Layer(M, K, N, group_size, X, codes, np.ascontiguousarray(qweight),
                     scales.view(np.uint16).copy())


@dataclass
class Bf16Layer:
    M: int
    K: int
    N: int
    X: np.ndarray        # uint16 bf16 bits [M][K]
    W: np.ndarray        # uint16 bf16 bits [N][K]


def bf16_layer(M: int, K: int, N: int, seed: int = 0, layer: int = 0) -> Bf16Layer:
    r_w, _, r_x = _streams(seed, layer)
    z = r_w.standard_normal(size=(N, K), dtype=np.float32) * np.float32(0.02)
    W = torch.from_numpy(z).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16).copy()
    X = bf16_bits_of_normals(r_x, (M, K))
    return Bf16Layer(M, K, N, X, W)


# Layer shapes of the measured workloads (hidden 5120, MLP width 17408).
MTP4_VERIFY_LAYERS = [(5120, 5120), (5120, 17408), (17408, 5120)]  # (K, N)
C32_MTP3_LAYERS = [(5120, 17408), (17408, 5120)]
