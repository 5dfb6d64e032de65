"""Pins for the oracle's format decoders and its bf16 rounding.

Each decoder is checked against an independent library routine over its whole
code space, and against hand-derived values (tests/golden).  The rounding is
checked against torch's float32 -> bfloat16 cast (round to nearest even).
"""
import math
import os

import numpy as np
import pytest
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _same(a: float, b: float) -> bool:
    if math.isnan(a) or math.isnan(b):
        return math.isnan(a) and math.isnan(b)
    return a == b and math.copysign(1.0, a) == math.copysign(1.0, b)


def test_fp16_all_codes_match_numpy(orc):
    codes = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = codes.view(np.float16).astype(np.float64)
    for c, r in zip(codes.tolist(), ref.tolist()):
        assert _same(orc.decode_fp16(c), r), hex(c)


def test_bf16_all_codes_match_torch(orc):
    codes = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = torch.from_numpy(codes.view(np.int16)).view(torch.bfloat16).double().numpy()
    for c, r in zip(codes.tolist(), ref.tolist()):
        assert _same(orc.decode_bf16(c), r), hex(c)


def test_e4m3_all_codes_match_torch(orc):
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy()
    for c, r in zip(codes.tolist(), ref.tolist()):
        assert _same(orc.decode_e4m3(c), r), hex(c)


def test_e8m0_all_codes_match_torch(orc):
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e8m0fnu).double().numpy()
    for c, r in zip(codes.tolist(), ref.tolist()):
        assert _same(orc.decode_e8m0(c), r), hex(c)
    # invariant: consecutive exponents double, E = 127 is one
    assert orc.decode_e8m0(127) == 1.0
    for e in range(254):
        assert orc.decode_e8m0(e + 1) == 2.0 * orc.decode_e8m0(e)


def test_e4m3_e8m0_hand_table(orc):
    with open(os.path.join(GOLDEN, "e4m3_e8m0_values.txt")) as f:
        rows = [l.split() for l in f if l.strip() and not l.startswith("#")]
    assert len(rows) >= 20
    for kind, code, value in rows:
        c = int(code, 16)
        got = orc.decode_e4m3(c) if kind == "e4m3" else orc.decode_e8m0(c)
        want = float("nan") if value == "nan" else float(value)
        assert _same(got, want), (kind, code, got, want)


def _torch_bf16_bits(vals: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(vals.astype(np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def test_round_bf16_matches_torch_random(orc):
    rng = np.random.default_rng(1234)
    bits = rng.integers(0, 2**32, size=200_000, dtype=np.uint64).astype(np.uint32)
    vals = bits.view(np.float32)
    vals = vals[np.isfinite(vals)]
    ref = _torch_bf16_bits(vals)
    got = orc.round_bf16_array(vals.astype(np.float64))
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, [(float(vals[i]), hex(got[i]), hex(ref[i])) for i in bad[:5]]


def test_round_bf16_ties_subnormals_overflow(orc):
    vals = []
    # exact ties between consecutive bf16 values (fp32 bit 15 set, bits 0..14 clear)
    for hi in [0x3F80, 0x3F81, 0x0001, 0x0080, 0x7F7E, 0x7F7F, 0xBF80, 0xBF81, 0x8000]:
        vals.append(np.uint32((hi << 16) | 0x8000))
        vals.append(np.uint32((hi << 16) | 0x8001))
        vals.append(np.uint32((hi << 16) | 0x7FFF))
    # fp32 subnormals and the largest finite values
    vals += [np.uint32(x) for x in (0x00000001, 0x00008000, 0x00018000, 0x007FFFFF,
                                     0x7F7FFFFF, 0xFF7FFFFF, 0x7F7F8000, 0x80000001)]
    f = np.array(vals, dtype=np.uint32).view(np.float32)
    ref = _torch_bf16_bits(f)
    got = orc.round_bf16_array(f.astype(np.float64))
    assert np.array_equal(got, ref), [(float(a), hex(b), hex(c)) for a, b, c in zip(f, got, ref) if b != c]
    assert orc.round_bf16(0.0) == 0x0000
    assert orc.round_bf16(-0.0) == 0x8000
    assert orc.round_bf16(float("inf")) == 0x7F80
    assert orc.round_bf16(2.0 ** 200) == 0x7F80      # beyond every finite bf16


def test_round_bf16_double_inputs_exact_rule(orc):
    """Values between fp32 neighbours: RNE of the exact double, not of a float."""
    one = 1.0
    ulp = 2.0 ** -7
    assert orc.round_bf16(one + ulp / 2) == 0x3F80                     # tie -> even (1.0)
    assert orc.round_bf16(one + ulp / 2 + 2.0 ** -40) == 0x3F81        # just above the tie
    assert orc.round_bf16(one + 3 * ulp / 2) == 0x3F82                 # tie -> even (1+2ulp)
    assert orc.round_bf16(one + 3 * ulp / 2 - 2.0 ** -40) == 0x3F81
