"""Python binding of libmxg.so: weight-quantized linear layer on B200.

    Y[M][N] = X[M][K] * dequant(W)^T     bf16 activations, fp32 accumulate, bf16 out

with GPTQ-style symmetric INT4 weights (``w4a16_*``) or MXFP8 weights
(``mxfp8_*``).  Every function here only marshals arguments into the C ABI
declared in ``include/mxg.h`` (same names); all computation runs in the
library's CUDA kernels.  PyTorch provides device memory and the current
stream.  There is no CPU fallback: importing this module raises if the
compiled library is missing.

Workspace: the GEMMs need a caller-owned, zero-initialised workspace that
they leave zeroed.  The functions below keep one per (device, stream) and
grow it on demand; pass ``workspace=`` to manage it yourself.
"""
from __future__ import annotations

import ctypes
import functools
import os
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmxg.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python -c 'import __graft_entry__ as g; g.build()'`"
        " (nvcc, sm_100a). There is no fallback implementation.")

_lib = ctypes.CDLL(LIB_PATH)

_p = ctypes.c_void_p
_i = ctypes.c_int
_sz = ctypes.c_size_t

_SIGS = {
    "mxg_status_string": (ctypes.c_char_p, [_i]),
    "w4a16_packed_bytes": (_sz, [_i, _i, _i]),
    "w4a16_repack": (_i, [_p, _p, _i, _i, _i, _p, _p]),
    "w4a16_repack_ct": (_i, [_p, _p, _i, _i, _i, _p, _p]),
    "w4a16_repack_fused": (_i, [_i, _p, _p, _p, _i, _i, _p, _p]),
    "w4a16_workspace_bytes": (_sz, [_i, _i, _i, _i]),
    "w4a16_gemm": (_i, [_p, _p, _i, _i, _i, _i, _p, _p, _sz, _p]),
    "w4a16_gemm_ex": (_i, [_p, _p, _i, _i, _i, _i, _p, _p, _sz, _p, _p]),
    "w4a16_static_scratch_status": (_i, [ctypes.POINTER(_i), _i, _p]),
    "w4a16_gemm_static_scratch": (_i, [_p, _p, _i, _i, _i, _i, _p, _p]),
    "mxfp8_workspace_bytes": (_sz, [_i, _i, _i]),
    "mxfp8_gemm": (_i, [_p, _p, _p, _i, _i, _i, _p, _p, _sz, _p]),
    "mxfp8_gemm_ex": (_i, [_p, _p, _p, _i, _i, _i, _p, _p, _sz, _p, _p]),
    "mxfp8_packed_bytes": (_sz, [_i, _i]),
    "mxfp8_repack": (_i, [_p, _p, _i, _i, _p, _p]),
    "mxfp8_packed_workspace_bytes": (_sz, [_i, _i, _i]),
    "mxfp8_gemm_packed": (_i, [_p, _p, _i, _i, _i, _p, _p, _sz, _p]),
    "mxfp8_gemm_packed_ex": (_i, [_p, _p, _i, _i, _i, _p, _p, _sz, _p, _p]),
    "w4a16_unpack": (_i, [_p, _i, _i, _i, _p, _p, _p, _p]),
    "mxfp8_dequant": (_i, [_p, _p, _i, _i, _p, _p]),
    "mxg_workspace_status": (_i, [_p, ctypes.POINTER(_i), _p]),
    "mxg_selftest_wait_timeout": (_i, [_p, _i, _p]),
    "w8a16_packed_bytes": (_sz, [_i, _i, _i]),
    "w8a16_repack": (_i, [_p, _p, _i, _i, _i, _p, _p]),
    "w8a16_repack_ct": (_i, [_p, _p, _i, _i, _i, _p, _p]),
    "w8a16_workspace_bytes": (_sz, [_i, _i, _i, _i]),
    "w8a16_gemm": (_i, [_p, _p, _i, _i, _i, _i, _p, _p, _sz, _p]),
    "w8a16_gemm_ex": (_i, [_p, _p, _i, _i, _i, _i, _p, _p, _sz, _p, _p]),
    "bf16_gemm_small_workspace_bytes": (_sz, [_i, _i, _i]),
    "bf16_gemm_small": (_i, [_p, _p, _i, _i, _i, _p, _p, _sz, _p]),
    "bf16_gemm_small_ex": (_i, [_p, _p, _i, _i, _i, _p, _p, _sz, _p, _p]),
}
for _name, (_res, _args) in _SIGS.items():
    _f = getattr(_lib, _name)
    _f.restype = _res
    _f.argtypes = _args

EXPORTED = tuple(_SIGS)

MXG_OK = 0
MXG_ERR_INVALID_ARG = -1
MXG_ERR_UNSUPPORTED_SHAPE = -2
MXG_ERR_WORKSPACE = -3
MXG_ERR_CUDA = -4
MXG_ERR_TIMEOUT = -5
MXG_ERR_CAPTURE = -6

PATH_AUTO, PATH_STREAM, PATH_TENSOR = 0, 1, 2


class GemmOptions(ctypes.Structure):
    """mxg_gemm_options of include/mxg.h: per-call path and weight-load
    timing."""
    _fields_ = [("path", ctypes.c_int), ("late_weights", ctypes.c_int)]


def _options(path: int = PATH_AUTO, late_weights: bool = False):
    """A pointer to the call's options, or None for the defaults.  The
    structure is kept alive by the returned pointer object."""
    if path == PATH_AUTO and not late_weights:
        return None
    return ctypes.pointer(GemmOptions(int(path), 1 if late_weights else 0))


class MxgError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {mxg_status_string(status)} (status {status})")
        self.status = status


def mxg_status_string(status: int) -> str:
    return _lib.mxg_status_string(int(status)).decode()


def _check(status: int, what: str) -> None:
    if status != MXG_OK:
        raise MxgError(status, what)


def _ptr(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None, device=None):
    """The CUDA stream handle a call runs on: ``stream``, which must live on
    ``device``, or that device's current stream."""
    if stream is None:
        s = torch.cuda.current_stream(device)
    else:
        s = stream
        sdev = getattr(s, "device", None)
        if device is not None and sdev is not None and torch.device(sdev) != torch.device(device):
            raise ValueError(f"stream is on {sdev}, the call's tensors on {device}")
    return ctypes.c_void_p(s.cuda_stream)


def _on_device(device):
    """Makes ``device`` current for a C call: the library plans and launches
    on the current device (its SM count, its kernels, its static scratch)."""
    return torch.cuda.device(device)


def _dev_call(device, what: str, fn, *args, stream=None) -> None:
    """fn(*args, stream handle) with ``device`` current; raises on a nonzero
    status."""
    with _on_device(device):
        _check(fn(*args, _stream(stream, device)), what)


def _need(t: torch.Tensor, dtype, name: str) -> None:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


# The C ABI takes plain pointers and cannot see buffer sizes: the binding
# checks every buffer a kernel reads or writes against the call's shape
# (type, then size, then layout and device), so a mismatch raises here
# instead of reaching memory past the end of a tensor.
def _same_device(t: torch.Tensor, device, name: str) -> None:
    if t.device != device:
        raise ValueError(f"{name} must be on {device}, got {t.device}")


def _need_out(out: torch.Tensor, M: int, N: int, device) -> None:
    if out.dtype != torch.bfloat16:
        raise ValueError(f"out must be torch.bfloat16, got {out.dtype}")
    if tuple(out.shape) != (M, N):
        raise ValueError(f"out must be [{M}][{N}], got {list(out.shape)}")
    _need(out, torch.bfloat16, "out")
    _same_device(out, device, "out")


def _need_weights(t: torch.Tensor, dtype, nbytes: int, device, name: str) -> None:
    """t holds at least nbytes bytes of weights (nbytes = 0: a shape the
    library rejects itself, with its own status)."""
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if nbytes and t.numel() * t.element_size() < nbytes:
        raise ValueError(f"{name} holds {t.numel() * t.element_size()} bytes, the shape needs "
                         f"{nbytes}")
    _need(t, dtype, name)
    _same_device(t, device, name)


def _empty(shape, dtype, device, stream) -> torch.Tensor:
    """An uninitialised tensor for a result the library writes on `stream`:
    allocated on that stream, so its memory, once freed, is reused only
    behind the work already queued there."""
    if stream is None:
        return torch.empty(shape, dtype=dtype, device=device)
    with torch.cuda.stream(stream):
        return torch.empty(shape, dtype=dtype, device=device)


def _need_shape(t: torch.Tensor, shape, name: str) -> None:
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must be {list(shape)}, got {list(t.shape)}")


def _need_ws(ws: torch.Tensor, device) -> None:
    if ws.dtype != torch.uint8:
        raise ValueError(f"workspace_buf must be torch.uint8, got {ws.dtype}")
    _need(ws, torch.uint8, "workspace_buf")
    _same_device(ws, device, "workspace_buf")


def _gemm_buffers(x: torch.Tensor, K: int, N: int, out, workspace_buf, need_ws, stream):
    """(M, out, ws) for a GEMM on x [M][K]: `out` and `workspace_buf` checked,
    or made (a [M][N] bf16 output; the cached workspace of `need_ws()`
    bytes)."""
    _need(x, torch.bfloat16, "x")
    if x.dim() != 2 or x.shape[1] != K:
        raise ValueError(f"x must be [M][{K}], got {list(x.shape)}")
    M = x.shape[0]
    if out is None:
        out = _empty((M, N), torch.bfloat16, x.device, stream)
    _need_out(out, M, N, x.device)
    if workspace_buf is None:
        ws = workspace(need_ws(), x.device, stream)
    else:
        ws = workspace_buf
        _need_ws(ws, x.device)
    return M, out, ws


# ------------------------------------------------------------- workspaces
_ws_lock = threading.Lock()
_ws_cache: dict[tuple[int, int], torch.Tensor] = {}


def workspace(nbytes: int, device=None, stream=None) -> torch.Tensor:
    """A zero-filled uint8 workspace of at least ``nbytes`` for (device, stream).
    It is allocated and zeroed on that stream, so the zero fill is ordered
    before the stream's next kernel, and the memory of a workspace it
    replaces goes back to that stream's pool (reused only behind the calls
    already queued there)."""
    dev = torch.device("cuda", torch.cuda.current_device() if device is None else
                       torch.device(device).index)
    s = stream if stream is not None else torch.cuda.current_stream(dev)
    key = (dev.index, s.cuda_stream)
    with _ws_lock:
        ws = _ws_cache.get(key)
        if ws is None or ws.numel() < nbytes:
            with torch.cuda.stream(s):
                ws = torch.zeros(max(int(nbytes), 256), dtype=torch.uint8, device=dev)
            _ws_cache[key] = ws
        return ws


@functools.lru_cache(maxsize=4096)
def _need_bytes(kind: str, device: int, M: int, N: int, K: int, G: int = 0) -> int:
    """Workspace size query, cached per (device, shape); the size depends on
    the device's SM count, so the query runs with that device current."""
    with torch.cuda.device(device):
        if kind == "w4a16":
            return int(_lib.w4a16_workspace_bytes(M, N, K, G))
        return int(_lib.mxfp8_workspace_bytes(M, N, K))


# -------------------------------------------------------------------- INT4
def w4a16_packed_bytes(K: int, N: int, group_size: int = 128) -> int:
    return int(_lib.w4a16_packed_bytes(K, N, group_size))


def _repack_out(words: torch.Tensor, K: int, N: int, group_size: int, out, what: str,
                stream=None):
    nbytes = w4a16_packed_bytes(K, N, group_size)
    if nbytes == 0:
        raise MxgError(MXG_ERR_UNSUPPORTED_SHAPE, what)
    if out is None:
        return _empty(nbytes, torch.uint8, words.device, stream)
    _need(out, torch.uint8, "out")
    if out.numel() != nbytes or out.device != words.device:
        raise ValueError(f"out must hold {nbytes} bytes on {words.device}")
    return out


def _need_scales(scales: torch.Tensor, name: str) -> None:
    if scales.dtype not in (torch.float16, torch.int16):
        raise ValueError(f"{name} must be float16 (or its int16 bit view)")
    _need(scales, scales.dtype, name)


def w4a16_repack(qweight: torch.Tensor, scales: torch.Tensor, group_size: int = 128,
                 stream=None, out: torch.Tensor | None = None) -> torch.Tensor:
    """Re-pack GPTQ words qweight[K/8][N] (int32) and scales[K/G][N] (fp16),
    into `out` (uint8, w4a16_packed_bytes bytes) when given."""
    _need(qweight, torch.int32, "qweight")
    _need_scales(scales, "scales")
    K = qweight.shape[0] * 8
    N = qweight.shape[1]
    packed = _repack_out(qweight, K, N, group_size, out, "w4a16_repack", stream)
    _need_shape(scales, (K // group_size, N), "scales")
    _same_device(scales, qweight.device, "scales")
    _dev_call(qweight.device, "w4a16_repack", _lib.w4a16_repack, _ptr(qweight), _ptr(scales), K, N,
              group_size, _ptr(packed), stream=stream)
    return packed


def w4a16_repack_ct(weight_packed: torch.Tensor, weight_scale: torch.Tensor,
                    group_size: int = 128, stream=None,
                    out: torch.Tensor | None = None) -> torch.Tensor:
    """Re-pack compressed-tensors words weight_packed[N][K/8] (int32) and
    weight_scale[N][K/G] (fp16) into the same buffer w4a16_repack makes."""
    _need(weight_packed, torch.int32, "weight_packed")
    _need_scales(weight_scale, "weight_scale")
    N = weight_packed.shape[0]
    K = weight_packed.shape[1] * 8
    packed = _repack_out(weight_packed, K, N, group_size, out, "w4a16_repack_ct", stream)
    _need_shape(weight_scale, (N, K // group_size), "weight_scale")
    _same_device(weight_scale, weight_packed.device, "weight_scale")
    _dev_call(weight_packed.device, "w4a16_repack_ct", _lib.w4a16_repack_ct, _ptr(weight_packed),
              _ptr(weight_scale), K, N, group_size, _ptr(packed), stream=stream)
    return packed


def w4a16_repack_fused(parts, group_size: int = 128, stream=None,
                       out: torch.Tensor | None = None) -> torch.Tensor:
    """One re-packed buffer for projections that share their input: `parts`
    is a sequence of GPTQ (qweight[K/8][Ni], scales[K/G][Ni]) pairs with the
    same K; the fused layer has N = sum Ni columns, part i's in order."""
    parts = list(parts)
    if not parts:
        raise ValueError("parts must not be empty")
    for qw, sc in parts:
        _need(qw, torch.int32, "qweight")
        _need_scales(sc, "scales")
    K = parts[0][0].shape[0] * 8
    if any(qw.shape[0] * 8 != K for qw, _ in parts):
        raise ValueError("every part must have the same K")
    Ns = [int(qw.shape[1]) for qw, _ in parts]
    packed = _repack_out(parts[0][0], K, sum(Ns), group_size, out, "w4a16_repack_fused", stream)
    for i, (qw, sc) in enumerate(parts):
        _need_shape(sc, (K // group_size, Ns[i]), f"scales of part {i}")
        _same_device(qw, packed.device, f"qweight of part {i}")
        _same_device(sc, packed.device, f"scales of part {i}")
    n = len(parts)
    qptrs = (ctypes.c_void_p * n)(*[qw.data_ptr() for qw, _ in parts])
    sptrs = (ctypes.c_void_p * n)(*[sc.data_ptr() for _, sc in parts])
    narr = (ctypes.c_int * n)(*Ns)
    _dev_call(packed.device, "w4a16_repack_fused", _lib.w4a16_repack_fused, n, qptrs, sptrs, narr,
              K, group_size, _ptr(packed), stream=stream)
    return packed


def w4a16_workspace_bytes(M: int, N: int, K: int, group_size: int = 128) -> int:
    return int(_lib.w4a16_workspace_bytes(M, N, K, group_size))


def w4a16_gemm(x: torch.Tensor, packed: torch.Tensor, N: int, K: int, group_size: int = 128,
               out: torch.Tensor | None = None, workspace_buf: torch.Tensor | None = None,
               stream=None, path: int = PATH_AUTO, late_weights: bool = False) -> torch.Tensor:
    """Y = x * dequant(W)^T for x bf16 [M][K] and a re-packed INT4 weight.
    ``path`` forces the weight-streaming (1) or tensor-core (2) path;
    ``late_weights`` makes the kernel load weights only after the previous
    kernel on the stream (for weights that kernel writes)."""
    M, out, ws = _gemm_buffers(
        x, K, N, out, workspace_buf,
        lambda: _need_bytes("w4a16", x.device.index, x.shape[0], N, K, group_size), stream)
    _need_weights(packed, torch.uint8, w4a16_packed_bytes(K, N, group_size), x.device, "packed")
    _dev_call(x.device, "w4a16_gemm", _lib.w4a16_gemm_ex, _ptr(x), _ptr(packed), M, N, K,
              group_size, _ptr(out), _ptr(ws), ws.numel(), _options(path, late_weights),
              stream=stream)
    return out


class PreparedCall:
    """One library call with its arguments marshalled once, for a loop that
    repeats it on the same buffers (a serving step).  The tensors are held
    here so they stay alive; their contents may change between calls, their
    storage must not move."""

    def __init__(self, fn, args, what: str, keep, device):
        self._fn, self._args, self._what, self._keep = fn, tuple(args), what, keep
        self._device = device

    def __call__(self) -> None:
        with _on_device(self._device):
            status = self._fn(*self._args)
        if status != MXG_OK:
            raise MxgError(status, self._what)


def prepare_w4a16_gemm(x: torch.Tensor, packed: torch.Tensor, N: int, K: int,
                       group_size: int = 128, out: torch.Tensor | None = None,
                       workspace_buf: torch.Tensor | None = None, stream=None,
                       path: int = PATH_AUTO, late_weights: bool = False):
    """(call, out): ``call()`` runs w4a16_gemm(x, packed) into ``out``."""
    M, out, ws = _gemm_buffers(
        x, K, N, out, workspace_buf,
        lambda: _need_bytes("w4a16", x.device.index, x.shape[0], N, K, group_size), stream)
    _need_weights(packed, torch.uint8, w4a16_packed_bytes(K, N, group_size), x.device, "packed")
    args = (_ptr(x), _ptr(packed), M, N, K, group_size, _ptr(out), _ptr(ws), ws.numel(),
            _options(path, late_weights), _stream(stream, x.device))
    return PreparedCall(_lib.w4a16_gemm_ex, args, "w4a16_gemm", (x, packed, out, ws, stream),
                        x.device), out


def prepare_mxfp8_gemm(x: torch.Tensor, wq: torch.Tensor, ws: torch.Tensor,
                       out: torch.Tensor | None = None, workspace_buf: torch.Tensor | None = None,
                       stream=None, path: int = PATH_AUTO, late_weights: bool = False):
    """(call, out): ``call()`` runs mxfp8_gemm(x, wq, ws) into ``out``."""
    M, K, N = _mx_shapes(x, wq, ws)
    M, out, wsb = _gemm_buffers(x, K, N, out, workspace_buf,
                                lambda: _need_bytes("mxfp8", x.device.index, M, N, K), stream)
    args = (_ptr(x), _ptr(wq), _ptr(ws), M, N, K, _ptr(out), _ptr(wsb), wsb.numel(),
            _options(path, late_weights), _stream(stream, x.device))
    return PreparedCall(_lib.mxfp8_gemm_ex, args, "mxfp8_gemm", (x, wq, ws, out, wsb, stream),
                        x.device), out


def prepare_bf16_gemm_small(x: torch.Tensor, w: torch.Tensor, out: torch.Tensor | None = None,
                            workspace_buf: torch.Tensor | None = None, stream=None,
                            late_weights: bool = False):
    """(call, out): ``call()`` runs bf16_gemm_small(x, w) into ``out``."""
    M, K, N, need = _small_shapes(x, w)
    M, out, wsb = _gemm_buffers(x, K, N, out, workspace_buf, lambda: need, stream)
    args = (_ptr(x), _ptr(w), M, N, K, _ptr(out), _ptr(wsb), wsb.numel(),
            _options(PATH_AUTO, late_weights), _stream(stream, x.device))
    return PreparedCall(_lib.bf16_gemm_small_ex, args, "bf16_gemm_small",
                        (x, w, out, wsb, stream), x.device), out


def w4a16_gemm_static_scratch(x: torch.Tensor, packed: torch.Tensor, N: int, K: int,
                              group_size: int = 128, out: torch.Tensor | None = None,
                              stream=None) -> torch.Tensor:
    """w4a16_gemm (M <= 32) with the library's fixed device scratch instead of a workspace."""
    _need(x, torch.bfloat16, "x")
    if x.dim() != 2 or x.shape[1] != K:
        raise ValueError(f"x must be [M][{K}], got {list(x.shape)}")
    M = x.shape[0]
    if out is None:
        out = _empty((M, N), torch.bfloat16, x.device, stream)
    _need_out(out, M, N, x.device)
    _need_weights(packed, torch.uint8, w4a16_packed_bytes(K, N, group_size), x.device, "packed")
    _dev_call(x.device, "w4a16_gemm_static_scratch", _lib.w4a16_gemm_static_scratch, _ptr(x),
              _ptr(packed), M, N, K, group_size, _ptr(out), stream=stream)
    return out


def w4a16_unpack(packed: torch.Tensor, K: int, N: int, group_size: int = 128, stream=None):
    """(codes uint8 [N][K], w_fp32 float32 [N][K], w_bf16 bfloat16 [N][K])."""
    dev = packed.device
    _need_weights(packed, torch.uint8, w4a16_packed_bytes(K, N, group_size), dev, "packed")
    codes = _empty((N, K), torch.uint8, dev, stream)
    w32 = _empty((N, K), torch.float32, dev, stream)
    w16 = _empty((N, K), torch.bfloat16, dev, stream)
    _dev_call(packed.device, "w4a16_unpack", _lib.w4a16_unpack, _ptr(packed), K, N, group_size,
              _ptr(codes), _ptr(w32), _ptr(w16), stream=stream)
    return codes, w32, w16


# ------------------------------------------------------------------- MXFP8
def _mx_shapes(x: torch.Tensor, wq: torch.Tensor, ws: torch.Tensor):
    """(M, K, N) of x [M][K] against E4M3 wq [N][K] and E8M0 ws [N][K/32]."""
    _need(x, torch.bfloat16, "x")
    if wq.dtype not in (torch.uint8, torch.float8_e4m3fn):
        raise ValueError("wq must be uint8 or float8_e4m3fn")
    if ws.dtype not in (torch.uint8, torch.float8_e8m0fnu):
        raise ValueError("ws must be uint8 or float8_e8m0fnu")
    if x.dim() != 2 or wq.dim() != 2 or ws.dim() != 2:
        raise ValueError("x, wq and ws must be 2-D")
    M, K = x.shape
    N = wq.shape[0]
    if wq.shape[1] != K or ws.shape[0] != N or ws.shape[1] * 32 != K:
        raise ValueError("shape mismatch between x, wq and ws")
    _need(wq, wq.dtype, "wq")
    _need(ws, ws.dtype, "ws")
    _same_device(wq, x.device, "wq")
    _same_device(ws, x.device, "ws")
    return M, K, N


def mxfp8_workspace_bytes(M: int, N: int, K: int) -> int:
    return int(_lib.mxfp8_workspace_bytes(M, N, K))


def mxfp8_gemm(x: torch.Tensor, wq: torch.Tensor, ws: torch.Tensor,
               out: torch.Tensor | None = None, workspace_buf: torch.Tensor | None = None,
               stream=None, path: int = PATH_AUTO, late_weights: bool = False) -> torch.Tensor:
    """Y = x * dequant(W)^T for x bf16 [M][K], E4M3 codes wq[N][K], E8M0 ws[N][K/32]."""
    M, K, N = _mx_shapes(x, wq, ws)
    M, out, wsb = _gemm_buffers(x, K, N, out, workspace_buf,
                                lambda: _need_bytes("mxfp8", x.device.index, M, N, K), stream)
    _dev_call(x.device, "mxfp8_gemm", _lib.mxfp8_gemm_ex, _ptr(x), _ptr(wq), _ptr(ws), M, N, K,
              _ptr(out), _ptr(wsb), wsb.numel(), _options(path, late_weights), stream=stream)
    return out


def mxfp8_repack(wq: torch.Tensor, ws: torch.Tensor, stream=None) -> torch.Tensor:
    """Re-pack E4M3 wq[N][K] and E8M0 ws[N][K/32] for mxfp8_gemm_packed."""
    if wq.dtype not in (torch.uint8, torch.float8_e4m3fn):
        raise ValueError("wq must be uint8 or float8_e4m3fn")
    if ws.dtype not in (torch.uint8, torch.float8_e8m0fnu):
        raise ValueError("ws must be uint8 or float8_e8m0fnu")
    if wq.dim() != 2:
        raise ValueError("wq must be [N][K]")
    N, K = wq.shape
    nbytes = int(_lib.mxfp8_packed_bytes(N, K))
    if nbytes == 0:
        raise MxgError(MXG_ERR_UNSUPPORTED_SHAPE, "mxfp8_repack")
    _need_shape(ws, (N, K // 32), "ws")
    _need(wq, wq.dtype, "wq")
    _need(ws, ws.dtype, "ws")
    _same_device(ws, wq.device, "ws")
    packed = _empty(nbytes, torch.uint8, wq.device, stream)
    _dev_call(wq.device, "mxfp8_repack", _lib.mxfp8_repack, _ptr(wq), _ptr(ws), N, K,
              _ptr(packed), stream=stream)
    return packed


def _mxp_ws_bytes(M: int, N: int, K: int) -> int:
    need = int(_lib.mxfp8_packed_workspace_bytes(M, N, K))
    if need == 0:
        raise MxgError(MXG_ERR_UNSUPPORTED_SHAPE, "mxfp8_gemm_packed")
    return need


def mxfp8_packed_workspace_bytes(M: int, N: int, K: int) -> int:
    return int(_lib.mxfp8_packed_workspace_bytes(M, N, K))


def mxfp8_gemm_packed(x: torch.Tensor, packed: torch.Tensor, N: int, K: int,
                      out: torch.Tensor | None = None, workspace_buf: torch.Tensor | None = None,
                      stream=None, late_weights: bool = False) -> torch.Tensor:
    """Y = x * dequant(W)^T for x bf16 [M][K] (M <= 16) and mxfp8_repack's buffer."""
    M, out, ws = _gemm_buffers(x, K, N, out, workspace_buf,
                               lambda: _mxp_ws_bytes(x.shape[0], N, K), stream)
    _need_weights(packed, torch.uint8, int(_lib.mxfp8_packed_bytes(N, K)), x.device, "packed")
    _dev_call(x.device, "mxfp8_gemm_packed", _lib.mxfp8_gemm_packed_ex, _ptr(x), _ptr(packed), M,
              N, K, _ptr(out), _ptr(ws), ws.numel(), _options(PATH_AUTO, late_weights),
              stream=stream)
    return out


def prepare_mxfp8_gemm_packed(x: torch.Tensor, packed: torch.Tensor, N: int, K: int,
                              out: torch.Tensor | None = None,
                              workspace_buf: torch.Tensor | None = None, stream=None,
                              late_weights: bool = False):
    """(call, out): ``call()`` runs mxfp8_gemm_packed(x, packed) into ``out``."""
    M, out, ws = _gemm_buffers(x, K, N, out, workspace_buf,
                               lambda: _mxp_ws_bytes(x.shape[0], N, K), stream)
    _need_weights(packed, torch.uint8, int(_lib.mxfp8_packed_bytes(N, K)), x.device, "packed")
    args = (_ptr(x), _ptr(packed), M, N, K, _ptr(out), _ptr(ws), ws.numel(),
            _options(PATH_AUTO, late_weights), _stream(stream, x.device))
    return PreparedCall(_lib.mxfp8_gemm_packed_ex, args, "mxfp8_gemm_packed",
                        (x, packed, out, ws, stream), x.device), out


def mxfp8_dequant(wq: torch.Tensor, ws: torch.Tensor, stream=None) -> torch.Tensor:
    """bf16 [N][K] weights of E4M3 wq[N][K] and E8M0 ws[N][K/32]."""
    if wq.dtype not in (torch.uint8, torch.float8_e4m3fn):
        raise ValueError("wq must be uint8 or float8_e4m3fn")
    if ws.dtype not in (torch.uint8, torch.float8_e8m0fnu):
        raise ValueError("ws must be uint8 or float8_e8m0fnu")
    if wq.dim() != 2:
        raise ValueError("wq must be [N][K]")
    N, K = wq.shape
    _need_shape(ws, (N, K // 32), "ws")
    _need(wq, wq.dtype, "wq")
    _need(ws, ws.dtype, "ws")
    _same_device(ws, wq.device, "ws")
    out = _empty((N, K), torch.bfloat16, wq.device, stream)
    _dev_call(wq.device, "mxfp8_dequant", _lib.mxfp8_dequant, _ptr(wq), _ptr(ws), N, K, _ptr(out),
              stream=stream)
    return out


# ------------------------------------------------------------- diagnostics
def _need_header(workspace_buf: torch.Tensor) -> None:
    """A workspace holding at least its 256-byte status header."""
    if workspace_buf.dtype != torch.uint8:
        raise ValueError(f"workspace_buf must be torch.uint8, got {workspace_buf.dtype}")
    if workspace_buf.numel() < 256:
        raise ValueError("workspace_buf must hold at least its 256-byte header")
    _need(workspace_buf, torch.uint8, "workspace_buf")


def mxg_workspace_status(workspace_buf: torch.Tensor, stream=None) -> int:
    _need_header(workspace_buf)
    v = ctypes.c_int(0)
    _dev_call(workspace_buf.device, "mxg_workspace_status", _lib.mxg_workspace_status,
              _ptr(workspace_buf), ctypes.byref(v), stream=stream)
    return v.value


def w8a16_repack(qweight: torch.Tensor, scales: torch.Tensor, group_size: int = 128,
                 stream=None) -> torch.Tensor:
    """Re-pack INT8 words qweight[K/4][N] (int32, 4 codes per word along K,
    zero point 128) and scales[K/G][N] (fp16)."""
    _need(qweight, torch.int32, "qweight")
    _need_scales(scales, "scales")
    K = qweight.shape[0] * 4
    N = qweight.shape[1]
    nbytes = int(_lib.w8a16_packed_bytes(K, N, group_size))
    if nbytes == 0:
        raise MxgError(MXG_ERR_UNSUPPORTED_SHAPE, "w8a16_repack")
    _need_shape(scales, (K // group_size, N), "scales")
    _same_device(scales, qweight.device, "scales")
    packed = _empty(nbytes, torch.uint8, qweight.device, stream)
    _dev_call(qweight.device, "w8a16_repack", _lib.w8a16_repack, _ptr(qweight), _ptr(scales), K, N,
              group_size, _ptr(packed), stream=stream)
    return packed


def w8a16_repack_ct(weight_packed: torch.Tensor, weight_scale: torch.Tensor,
                    group_size: int = 128, stream=None) -> torch.Tensor:
    """Re-pack the compressed-tensors INT8 export weight_packed[N][K/4]
    (int32) and weight_scale[N][K/G] (fp16) into the w8a16_repack buffer."""
    _need(weight_packed, torch.int32, "weight_packed")
    _need_scales(weight_scale, "weight_scale")
    N = weight_packed.shape[0]
    K = weight_packed.shape[1] * 4
    nbytes = int(_lib.w8a16_packed_bytes(K, N, group_size))
    if nbytes == 0:
        raise MxgError(MXG_ERR_UNSUPPORTED_SHAPE, "w8a16_repack_ct")
    _need_shape(weight_scale, (N, K // group_size), "weight_scale")
    _same_device(weight_scale, weight_packed.device, "weight_scale")
    packed = _empty(nbytes, torch.uint8, weight_packed.device, stream)
    _dev_call(weight_packed.device, "w8a16_repack_ct", _lib.w8a16_repack_ct, _ptr(weight_packed),
              _ptr(weight_scale), K, N, group_size, _ptr(packed), stream=stream)
    return packed


def _w8_ws_bytes(M: int, N: int, K: int, group_size: int) -> int:
    need = int(_lib.w8a16_workspace_bytes(M, N, K, group_size))
    if need == 0:
        raise MxgError(MXG_ERR_UNSUPPORTED_SHAPE, "w8a16_gemm")
    return need


def w8a16_gemm(x: torch.Tensor, packed: torch.Tensor, N: int, K: int, group_size: int = 128,
               out: torch.Tensor | None = None, workspace_buf: torch.Tensor | None = None,
               stream=None, late_weights: bool = False) -> torch.Tensor:
    """Y = x * dequant(W)^T for x bf16 [M][K] (M <= 32) and a re-packed INT8 weight."""
    M, out, ws = _gemm_buffers(x, K, N, out, workspace_buf,
                               lambda: _w8_ws_bytes(x.shape[0], N, K, group_size), stream)
    _need_weights(packed, torch.uint8, int(_lib.w8a16_packed_bytes(K, N, group_size)), x.device,
                  "packed")
    _dev_call(x.device, "w8a16_gemm", _lib.w8a16_gemm_ex, _ptr(x), _ptr(packed), M, N, K,
              group_size, _ptr(out), _ptr(ws), ws.numel(), _options(PATH_AUTO, late_weights),
              stream=stream)
    return out


def prepare_w8a16_gemm(x: torch.Tensor, packed: torch.Tensor, N: int, K: int,
                       group_size: int = 128, out: torch.Tensor | None = None,
                       workspace_buf: torch.Tensor | None = None, stream=None,
                       late_weights: bool = False):
    """(call, out): ``call()`` runs w8a16_gemm(x, packed) into ``out``."""
    M, out, ws = _gemm_buffers(x, K, N, out, workspace_buf,
                               lambda: _w8_ws_bytes(x.shape[0], N, K, group_size), stream)
    _need_weights(packed, torch.uint8, int(_lib.w8a16_packed_bytes(K, N, group_size)), x.device,
                  "packed")
    args = (_ptr(x), _ptr(packed), M, N, K, group_size, _ptr(out), _ptr(ws), ws.numel(),
            _options(PATH_AUTO, late_weights), _stream(stream, x.device))
    return PreparedCall(_lib.w8a16_gemm_ex, args, "w8a16_gemm", (x, packed, out, ws, stream),
                        x.device), out


def _small_shapes(x: torch.Tensor, w: torch.Tensor):
    """(M, K, N, workspace bytes) of x [M][K] against dense bf16 w [N][K]."""
    _need(x, torch.bfloat16, "x")
    _need(w, torch.bfloat16, "w")
    if x.dim() != 2 or w.dim() != 2 or x.shape[1] != w.shape[1]:
        raise ValueError("x must be [M][K] and w [N][K]")
    _same_device(w, x.device, "w")
    M, K = x.shape
    N = w.shape[0]
    need = int(_lib.bf16_gemm_small_workspace_bytes(M, N, K))
    if need == 0:
        raise MxgError(MXG_ERR_UNSUPPORTED_SHAPE, "bf16_gemm_small")
    return M, K, N, need


def bf16_gemm_small(x: torch.Tensor, w: torch.Tensor, out: torch.Tensor | None = None,
                    workspace_buf: torch.Tensor | None = None, stream=None,
                    late_weights: bool = False) -> torch.Tensor:
    """Y = x * w^T with dense bf16 w [N][K] (few columns, e.g. the paired
    48 + 48 GDN A/B projection) and x bf16 [M][K], M <= 8."""
    M, K, N, need = _small_shapes(x, w)
    M, out, ws = _gemm_buffers(x, K, N, out, workspace_buf, lambda: need, stream)
    _dev_call(x.device, "bf16_gemm_small", _lib.bf16_gemm_small_ex, _ptr(x), _ptr(w), M, N, K,
              _ptr(out), _ptr(ws), ws.numel(), _options(PATH_AUTO, late_weights),
              stream=stream)
    return out


def mxg_selftest_wait_timeout(workspace_buf: torch.Tensor | None, limit_us: int,
                              stream=None, device=None) -> None:
    """Runs the library's bounded-wait self-test, which records
    MXG_ERR_TIMEOUT in ``workspace_buf``'s status word, or (None) in the
    static scratch array of ``device`` (default: the current device)."""
    if workspace_buf is None:
        dev = torch.device("cuda", torch.cuda.current_device() if device is None else
                           torch.device(device).index)
        _dev_call(dev, "mxg_selftest_wait_timeout", _lib.mxg_selftest_wait_timeout, None,
                  int(limit_us), stream=stream)
        return
    _need_header(workspace_buf)
    _dev_call(workspace_buf.device, "mxg_selftest_wait_timeout", _lib.mxg_selftest_wait_timeout,
              _ptr(workspace_buf), int(limit_us), stream=stream)


def w4a16_static_scratch_status(reset: bool = False, stream=None, device=None) -> int:
    """The status word of the static scratch array of ``device`` (default:
    the current device): 0, or the first error a kernel recorded there.
    ``reset`` also zeroes the status word and the arrival counters.
    Synchronizes the stream."""
    dev = torch.device("cuda", torch.cuda.current_device() if device is None else
                       torch.device(device).index)
    v = ctypes.c_int(0)
    _dev_call(dev, "w4a16_static_scratch_status", _lib.w4a16_static_scratch_status,
              ctypes.byref(v), 1 if reset else 0, stream=stream)
    return v.value


def raw_lib() -> ctypes.CDLL:
    """The loaded C library (for callers that pass raw pointers)."""
    return _lib
