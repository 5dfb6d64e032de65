"""CPU oracle for Y = X * dequant(W)^T (INT4 W4A16 and MXFP8 weights).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  It shares no code with the CUDA library and never imports it; the
two meet only through the seeded inputs of the ``synth`` module.

The arithmetic lives in ``oracle.c`` (plain C, fp64, k ascending).  This
module compiles it with gcc (``build()``) and marshals numpy arrays into it.
The environment variable ``MXG_ORACLE_LIB`` points it at another build of the
same source instead (the mutation tests use it to load deliberately broken
copies and check that the pins reject them).
Every function cites the passage it follows in ``oracle.c``'s header:

* GPTQ INT4 symmetric grouped weights: "Qwen3.8-27B GPTQ-Int4-sym-G128"
  model card, section "Quantization contract"; Eole Qwen3.8 recipe, section
  "Compressed-tensors INT4 layout".
* MXFP8: "Qwen3.8-27B-MXFP8 AutoRound" model card, header, section 2 (kernel
  constraints) and section 8 (OCP MX format, E8M0 scale per 32 elements).
* Dense bf16 projections: Eole Qwen3.8 recipe, section "Pack inference
  projections" (the paired GDN A/B projection).
* INT8 W8A16 head: Eole Qwen3.8 recipe, section "Optional vocabulary-head
  quantization"; W4A16 LowLatency model card (INT8 lm_head, RTN g128).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "libmxg_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.c into libmxg_oracle.so (gcc, OpenMP, no FP contraction)."""
    if force or not os.path.exists(_LIB_PATH) or (
        os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)
    ):
        cmd = [
            "gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
            "-ffp-contract=off", "-fno-fast-math", "-Wall", "-Wextra",
            _SRC, "-o", _LIB_PATH + ".tmp", "-lm",
        ]
        subprocess.run(cmd, check=True)
        os.replace(_LIB_PATH + ".tmp", _LIB_PATH)
    return _LIB_PATH


def _bind(lib):
    p = ctypes.c_void_p
    i = ctypes.c_int
    i64 = ctypes.c_int64
    lib.mxo_decode_fp16.restype = ctypes.c_double
    lib.mxo_decode_fp16.argtypes = [ctypes.c_uint16]
    lib.mxo_decode_bf16.restype = ctypes.c_double
    lib.mxo_decode_bf16.argtypes = [ctypes.c_uint16]
    lib.mxo_decode_e4m3.restype = ctypes.c_double
    lib.mxo_decode_e4m3.argtypes = [ctypes.c_uint8]
    lib.mxo_decode_e8m0.restype = ctypes.c_double
    lib.mxo_decode_e8m0.argtypes = [ctypes.c_uint8]
    lib.mxo_round_bf16.restype = ctypes.c_uint16
    lib.mxo_round_bf16.argtypes = [ctypes.c_double]
    lib.mxo_w4a16_unpack.restype = i
    lib.mxo_w4a16_unpack.argtypes = [p, p, i, i, i, p, p]
    lib.mxo_w8a16_unpack.restype = i
    lib.mxo_w8a16_unpack.argtypes = [p, p, i, i, i, p, p]
    lib.mxo_w8a16_gemm.restype = i
    lib.mxo_w8a16_gemm.argtypes = [p, p, p, i, i, i, i, p, i]
    lib.mxo_bf16_gemm.restype = i
    lib.mxo_bf16_gemm.argtypes = [p, p, i, i, i, p]
    lib.mxo_w4a16_unpack_ct.restype = i
    lib.mxo_w4a16_unpack_ct.argtypes = [p, p, i, i, i, p, p]
    lib.mxo_w4a16_pack.restype = i
    lib.mxo_w4a16_pack.argtypes = [p, i, i, p]
    lib.mxo_w4a16_gemm.restype = i
    lib.mxo_w4a16_gemm.argtypes = [p, p, p, i, i, i, i, p, i]
    lib.mxo_w4a16_gemm_at.restype = i
    lib.mxo_w4a16_gemm_at.argtypes = [p, p, p, i, i, i, i, p, p, i64, p, i]
    lib.mxo_mxfp8_dequant.restype = i
    lib.mxo_mxfp8_dequant.argtypes = [p, p, i, i, p]
    lib.mxo_mxfp8_gemm.restype = i
    lib.mxo_mxfp8_gemm.argtypes = [p, p, p, i, i, i, p, i]
    lib.mxo_mxfp8_gemm_at.restype = i
    lib.mxo_mxfp8_gemm_at.argtypes = [p, p, p, i, i, i, p, p, i64, p, i]
    lib.mxo_threads.restype = i
    lib.mxo_threads.argtypes = [i]
    return lib


def _load():
    global _lib
    if _lib is None:
        lib_path = os.environ.get("MXG_ORACLE_LIB")
        if not lib_path:
            lib_path = build()
        _lib = _bind(ctypes.CDLL(lib_path))
    return _lib


def _c(a: np.ndarray, dtype) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype != np.dtype(dtype):
        raise TypeError(f"expected {np.dtype(dtype)}, got {a.dtype}")
    return a


def _ptr(a: np.ndarray):
    return ctypes.c_void_p(a.ctypes.data)


def _check(status: int, what: str) -> None:
    if status != 0:
        raise ValueError(f"oracle {what}: invalid argument or undefined input")


# ------------------------------------------------------------------ decoders
def decode_fp16(bits: int) -> float:
    return _load().mxo_decode_fp16(int(bits))


def decode_bf16(bits: int) -> float:
    return _load().mxo_decode_bf16(int(bits))


def decode_e4m3(code: int) -> float:
    return _load().mxo_decode_e4m3(int(code))


def decode_e8m0(e: int) -> float:
    return _load().mxo_decode_e8m0(int(e))


def round_bf16(x: float) -> int:
    """Bits of the bfloat16 nearest to x (ties to even)."""
    return int(_load().mxo_round_bf16(float(x)))


def round_bf16_array(values: np.ndarray) -> np.ndarray:
    """Elementwise ``round_bf16`` (uint16 bits); a loop over the C routine."""
    lib = _load()
    flat = np.asarray(values, dtype=np.float64).ravel()
    out = np.empty(flat.shape, dtype=np.uint16)
    for i, v in enumerate(flat):
        out[i] = lib.mxo_round_bf16(float(v))
    return out.reshape(np.shape(values))


# ------------------------------------------------------------------- INT4
def w4a16_unpack(qweight: np.ndarray, scales: np.ndarray | None, K: int, N: int,
                 group_size: int = 128, want_codes: bool = True,
                 want_weights: bool = True):
    """Codes[N][K] (uint8) and exact weights[N][K] (float64) of GPTQ words."""
    qw = _c(qweight, np.int32)
    sc = _c(scales, np.uint16) if scales is not None else None
    codes = np.empty((N, K), dtype=np.uint8) if want_codes else None
    w = np.empty((N, K), dtype=np.float64) if want_weights else None
    st = _load().mxo_w4a16_unpack(
        _ptr(qw), _ptr(sc) if sc is not None else None, K, N, group_size,
        _ptr(codes) if codes is not None else None,
        _ptr(w) if w is not None else None)
    _check(st, "w4a16_unpack")
    return codes, w


def w4a16_unpack_ct(weight_packed: np.ndarray, weight_scale: np.ndarray | None, K: int, N: int,
                    group_size: int = 128, want_codes: bool = True,
                    want_weights: bool = True):
    """Codes[N][K] (uint8) and exact weights[N][K] (float64) of a
    compressed-tensors export: words weight_packed[N][K/8], scales
    weight_scale[N][K/G] (fp16 bits)."""
    wp = _c(weight_packed, np.int32)
    sc = _c(weight_scale, np.uint16) if weight_scale is not None else None
    codes = np.empty((N, K), dtype=np.uint8) if want_codes else None
    w = np.empty((N, K), dtype=np.float64) if want_weights else None
    st = _load().mxo_w4a16_unpack_ct(
        _ptr(wp), _ptr(sc) if sc is not None else None, K, N, group_size,
        _ptr(codes) if codes is not None else None,
        _ptr(w) if w is not None else None)
    _check(st, "w4a16_unpack_ct")
    return codes, w


def w4a16_pack(codes: np.ndarray) -> np.ndarray:
    """GPTQ words qweight[K/8][N] (int32) of codes[N][K]."""
    c = _c(codes, np.uint8)
    N, K = c.shape
    qw = np.empty((K // 8, N), dtype=np.int32)
    _check(_load().mxo_w4a16_pack(_ptr(c), K, N, _ptr(qw)), "w4a16_pack")
    return qw


def w4a16_gemm(X_bits: np.ndarray, qweight: np.ndarray, scales: np.ndarray,
               M: int, N: int, K: int, group_size: int = 128,
               nthreads: int = 1) -> np.ndarray:
    """Y[M][N] in float64 (not rounded).  X_bits: bf16 bit patterns [M][K]."""
    x = _c(X_bits, np.uint16)
    qw = _c(qweight, np.int32)
    sc = _c(scales, np.uint16)
    Y = np.empty((M, N), dtype=np.float64)
    st = _load().mxo_w4a16_gemm(_ptr(x), _ptr(qw), _ptr(sc), M, N, K, group_size,
                                _ptr(Y), int(nthreads))
    _check(st, "w4a16_gemm")
    return Y


def w4a16_gemm_at(X_bits, qweight, scales, M, N, K, group_size, rows, cols,
                  nthreads: int = 1) -> np.ndarray:
    x = _c(X_bits, np.uint16)
    qw = _c(qweight, np.int32)
    sc = _c(scales, np.uint16)
    r = _c(np.asarray(rows, dtype=np.int64), np.int64)
    c = _c(np.asarray(cols, dtype=np.int64), np.int64)
    out = np.empty(r.shape[0], dtype=np.float64)
    st = _load().mxo_w4a16_gemm_at(_ptr(x), _ptr(qw), _ptr(sc), M, N, K, group_size,
                                   _ptr(r), _ptr(c), r.shape[0], _ptr(out),
                                   int(nthreads))
    _check(st, "w4a16_gemm_at")
    return out


# ------------------------------------------------------------------ MXFP8
def mxfp8_dequant(Wq: np.ndarray, Ws: np.ndarray, N: int, K: int) -> np.ndarray:
    wq = _c(Wq, np.uint8)
    ws = _c(Ws, np.uint8)
    w = np.empty((N, K), dtype=np.float64)
    _check(_load().mxo_mxfp8_dequant(_ptr(wq), _ptr(ws), N, K, _ptr(w)), "mxfp8_dequant")
    return w


def mxfp8_gemm(X_bits, Wq, Ws, M: int, N: int, K: int, nthreads: int = 1) -> np.ndarray:
    x = _c(X_bits, np.uint16)
    wq = _c(Wq, np.uint8)
    ws = _c(Ws, np.uint8)
    Y = np.empty((M, N), dtype=np.float64)
    st = _load().mxo_mxfp8_gemm(_ptr(x), _ptr(wq), _ptr(ws), M, N, K, _ptr(Y),
                                int(nthreads))
    _check(st, "mxfp8_gemm")
    return Y


def mxfp8_gemm_at(X_bits, Wq, Ws, M, N, K, rows, cols, nthreads: int = 1) -> np.ndarray:
    x = _c(X_bits, np.uint16)
    wq = _c(Wq, np.uint8)
    ws = _c(Ws, np.uint8)
    r = _c(np.asarray(rows, dtype=np.int64), np.int64)
    c = _c(np.asarray(cols, dtype=np.int64), np.int64)
    out = np.empty(r.shape[0], dtype=np.float64)
    st = _load().mxo_mxfp8_gemm_at(_ptr(x), _ptr(wq), _ptr(ws), M, N, K, _ptr(r),
                                   _ptr(c), r.shape[0], _ptr(out), int(nthreads))
    _check(st, "mxfp8_gemm_at")
    return out


def threads(requested: int) -> int:
    """Threads an oracle call with ``nthreads=requested`` actually uses."""
    return int(_load().mxo_threads(int(requested)))


def bf16_gemm(X_bits: np.ndarray, W_bits: np.ndarray, M: int, N: int, K: int) -> np.ndarray:
    """Y[M][N] in float64 (not rounded) of dense bf16 weights W[N][K]."""
    x = _c(X_bits, np.uint16)
    w = _c(W_bits, np.uint16)
    Y = np.empty((M, N), dtype=np.float64)
    _check(_load().mxo_bf16_gemm(_ptr(x), _ptr(w), M, N, K, _ptr(Y)), "bf16_gemm")
    return Y


def w8a16_unpack(qweight: np.ndarray, scales: np.ndarray | None, K: int, N: int,
                 group_size: int = 128):
    """Codes[N][K] (uint8) and exact weights[N][K] (float64) of INT8 words
    qweight[K/4][N] with fp16 scales[K/G][N]."""
    qw = _c(qweight, np.int32)
    sc = _c(scales, np.uint16) if scales is not None else None
    codes = np.empty((N, K), dtype=np.uint8)
    w = np.empty((N, K), dtype=np.float64) if sc is not None else None
    st = _load().mxo_w8a16_unpack(_ptr(qw), _ptr(sc) if sc is not None else None, K, N,
                                  group_size, _ptr(codes), _ptr(w) if w is not None else None)
    _check(st, "w8a16_unpack")
    return codes, w


def w8a16_gemm(X_bits: np.ndarray, qweight: np.ndarray, scales: np.ndarray,
               M: int, N: int, K: int, group_size: int = 128, nthreads: int = 1) -> np.ndarray:
    """Y[M][N] in float64 (not rounded) of INT8 W8A16 weights."""
    x = _c(X_bits, np.uint16)
    qw = _c(qweight, np.int32)
    sc = _c(scales, np.uint16)
    Y = np.empty((M, N), dtype=np.float64)
    _check(_load().mxo_w8a16_gemm(_ptr(x), _ptr(qw), _ptr(sc), M, N, K, group_size, _ptr(Y),
                                  int(nthreads)), "w8a16_gemm")
    return Y
