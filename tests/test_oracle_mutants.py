"""The oracle's pins catch plausible mistakes.

Each case plants one mistake in a copy of oracle.c (on the CPU), builds it,
and runs the oracle pin suites against that build in a subprocess; the suite
must fail.  The unmodified source must pass the same suites.
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "oracle.c")
PIN_SUITES = ["tests/test_oracle_formats.py", "tests/test_oracle_int4.py",
              "tests/test_oracle_mxfp8.py", "tests/test_oracle_bf16.py",
              "tests/test_oracle_int8.py"]

MUTANTS = {
    "zero_point_7": ("return (double)(q - 8) * s;", "return (double)(q - 7) * s;"),
    "nibble_order_reversed": ("(word >> (4 * (k % 8)))", "(word >> (4 * (7 - k % 8)))"),
    "word_column_shifted": ("qweight[(size_t)(k / 8) * N + n]", "qweight[(size_t)(k / 8) * N + (n + 1) % N]"),
    "ct_words_read_as_gptq": ("weight_packed[(size_t)n * (K / 8) + k / 8]", "weight_packed[(size_t)(k / 8) * N + n]"),
    "ct_nibble_order_reversed": ("(word >> (4 * (k & 7)))", "(word >> (4 * (7 - (k & 7))))"),
    "ct_scales_read_as_gptq": ("weight_scale[(size_t)n * (K / G) + k / G]", "weight_scale[(size_t)(k / G) * N + n]"),
    "group_index_fixed_128": ("scales[(size_t)(k / G) * N + n]", "scales[(size_t)(k / 128) * N + n]"),
    "fp16_bias_off_by_one": ("ldexp((double)(1024 + f), e - 25)", "ldexp((double)(1024 + f), e - 24)"),
    "bf16_drops_implicit_bit": ("ldexp((double)(128 + f), e - 134)", "ldexp((double)(f), e - 134)"),
    "e4m3_subnormal_scale": ("v = ldexp((double)f, -9);", "v = ldexp((double)f, -10);"),
    "e8m0_bias_128": ("return ldexp(1.0, (int)e - 127);", "return ldexp(1.0, (int)e - 128);"),
    "round_ties_away": ("r = (fmod(lo, 2.0) == 0.0) ? lo : lo + 1.0;", "r = lo + 1.0;"),
    "gemm_reversed_k": ("acc += x[k] * w[k];", "acc += x[k] * w[K - 1 - k];"),
    "mxfp8_block_index": ("Ws[(size_t)n * (K / 32) + k / 32]", "Ws[(size_t)n * (K / 32) + (k % 32) / 32]"),
    "bf16_gemm_reversed_w": ("mxo_decode_bf16(W[(size_t)n * K + k])", "mxo_decode_bf16(W[(size_t)n * K + (K - 1 - k)])"),
    "bf16_gemm_drops_last_k": ("            for (int k = 0; k < K; ++k)\n                acc += mxo_decode_bf16(X[(size_t)m * K + k]) * mxo_decode_bf16(W", "            for (int k = 0; k < K - 1; ++k)\n                acc += mxo_decode_bf16(X[(size_t)m * K + k]) * mxo_decode_bf16(W"),
    "int8_byte_order_reversed": ("(word >> (8 * (k % 4)))", "(word >> (8 * (3 - k % 4)))"),
    "int8_gemm_group_fixed_128": ("mxo_decode_fp16(scales[(size_t)N * (k / G) + n]);\n            for (int m", "mxo_decode_fp16(scales[(size_t)N * (k / 128) + n]);\n            for (int m"),
    "int8_zero_point_127": ("(double)(w8a16_code(qweight, N, n, k) - 128)", "(double)(w8a16_code(qweight, N, n, k) - 127)"),
    "mxfp8_gemm_drops_scale": ("w[k] = mxfp8_weight(Wq, Ws, K, n, k);", "w[k] = mxo_decode_e4m3(Wq[(size_t)n * K + k]);"),
}


def _build(src_text: str, out: str) -> None:
    path = out + ".c"
    with open(path, "w") as f:
        f.write(src_text)
    subprocess.run(["gcc", "-O1", "-std=c11", "-fPIC", "-shared", "-fopenmp",
                    "-ffp-contract=off", "-w", path, "-o", out, "-lm"], check=True)


def _run_pins(lib: str) -> int:
    env = dict(os.environ, MXG_ORACLE_LIB=lib)
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        *PIN_SUITES], cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=600)
    return r.returncode


def test_unmodified_source_passes(tmp_path):
    lib = str(tmp_path / "orig.so")
    _build(open(SRC).read(), lib)
    assert _run_pins(lib) == 0


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(tmp_path, name):
    old, new = MUTANTS[name]
    text = open(SRC).read()
    assert text.count(old) == 1, f"mutation site for {name} not found exactly once"
    text = text.replace(old, new)
    lib = str(tmp_path / f"{name}.so")
    _build(text, lib)
    assert _run_pins(lib) != 0, f"the pins did not catch the planted mistake {name}"
