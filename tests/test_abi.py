"""The C ABI library: loads, exports every declared symbol, validates
arguments before touching the GPU (no kernel runs here)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mxg.h")


@pytest.fixture(scope="module")
def mxg():
    import __graft_entry__
    __graft_entry__.build()
    import mxfp8_gemm_speculative_b200 as m
    return m


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*MXG_API\s+(?:const\s+)?[a-z_0-9]+\s*\**\s*([a-z_0-9]+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_boundary():
    names = declared_functions()
    for want in ["w4a16_packed_bytes", "w4a16_repack", "w4a16_workspace_bytes", "w4a16_gemm",
                 "mxfp8_workspace_bytes", "mxfp8_gemm", "w4a16_unpack", "mxfp8_dequant",
                 "mxg_status_string"]:
        assert want in names


def test_library_exports_every_declared_symbol(mxg):
    lib = ctypes.CDLL(mxg.LIB_PATH)
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert set(declared_functions()) == set(mxg.EXPORTED)


def test_status_strings(mxg):
    for s in range(-6, 1):
        assert mxg.mxg_status_string(s) not in ("", "unknown status")
    assert mxg.mxg_status_string(-99) == "unknown status"


def test_packed_bytes(mxg):
    assert mxg.w4a16_packed_bytes(5120, 17408, 128) == 44564480 + 1392640
    assert mxg.w4a16_packed_bytes(5120, 5120, 128) == 13107200 + 409600
    assert mxg.w4a16_packed_bytes(512, 512, 32) == 512 * 512 // 2 + 512 * 16 * 2
    assert mxg.w4a16_packed_bytes(512, 512, 48) == 0       # group size
    assert mxg.w4a16_packed_bytes(500, 512, 128) == 0      # K % G
    assert mxg.w4a16_packed_bytes(512, 96, 128) == 0       # N % 64


def test_arguments_rejected_before_launch(mxg):
    lib = mxg.raw_lib()
    a = ctypes.c_void_p(4096)          # aligned, never dereferenced on these paths
    mis = ctypes.c_void_p(4096 + 8)
    null = None
    # NULL / misaligned pointers
    assert lib.w4a16_gemm(null, a, 5, 512, 512, 128, a, a, 1 << 20, null) == mxg.MXG_ERR_INVALID_ARG
    assert lib.w4a16_gemm(a, mis, 5, 512, 512, 128, a, a, 1 << 20, null) == mxg.MXG_ERR_INVALID_ARG
    assert lib.mxfp8_gemm(a, a, mis, 4, 256, 512, a, a, 1 << 20, null) == mxg.MXG_ERR_INVALID_ARG
    assert lib.w4a16_repack(a, null, 512, 512, 128, a, null) == mxg.MXG_ERR_INVALID_ARG
    assert lib.w4a16_repack_ct(null, a, 512, 512, 128, a, null) == mxg.MXG_ERR_INVALID_ARG
    ptrs = (ctypes.c_void_p * 2)(4096, 8192)
    ns = (ctypes.c_int * 2)(512, 256)
    assert lib.w4a16_repack_fused(0, ptrs, ptrs, ns, 512, 128, a, null) == mxg.MXG_ERR_INVALID_ARG
    assert lib.w4a16_repack_fused(2, null, ptrs, ns, 512, 128, a, null) == mxg.MXG_ERR_INVALID_ARG
    assert lib.w4a16_repack_fused(2, ptrs, ptrs, ns, 512, 128, mis, null) == mxg.MXG_ERR_INVALID_ARG
    bad = (ctypes.c_int * 2)(512, 96)
    assert lib.w4a16_repack_fused(2, ptrs, ptrs, bad, 512, 128, a, null) == mxg.MXG_ERR_UNSUPPORTED_SHAPE
    assert lib.w4a16_repack_ct(a, mis, 512, 512, 128, a, null) == mxg.MXG_ERR_INVALID_ARG
    # M < 1
    assert lib.w4a16_gemm(a, a, 0, 512, 512, 128, a, a, 1 << 20, null) == mxg.MXG_ERR_INVALID_ARG
    # shapes the format or the kernels reject
    assert lib.w4a16_gemm(a, a, 5, 512, 512, 96, a, a, 1 << 20, null) == mxg.MXG_ERR_UNSUPPORTED_SHAPE
    assert lib.w4a16_gemm(a, a, 5, 96, 512, 128, a, a, 1 << 20, null) == mxg.MXG_ERR_UNSUPPORTED_SHAPE
    assert lib.w4a16_repack(a, a, 480, 512, 32, a, null) == mxg.MXG_ERR_UNSUPPORTED_SHAPE
    assert lib.w4a16_repack_ct(a, a, 480, 512, 32, a, null) == mxg.MXG_ERR_UNSUPPORTED_SHAPE
    assert lib.w4a16_repack_ct(a, a, 512, 96, 128, a, null) == mxg.MXG_ERR_UNSUPPORTED_SHAPE
    assert lib.mxfp8_gemm(a, a, a, 4, 96, 512, a, a, 1 << 20, null) == mxg.MXG_ERR_UNSUPPORTED_SHAPE
    assert lib.mxfp8_gemm(a, a, a, 4, 256, 500, a, a, 1 << 20, null) == mxg.MXG_ERR_UNSUPPORTED_SHAPE
    assert lib.mxfp8_dequant(a, a, 96, 512, a, null) == mxg.MXG_ERR_UNSUPPORTED_SHAPE
    assert lib.w4a16_unpack(a, 512, 512, 128, mis, null, null, null) == mxg.MXG_ERR_INVALID_ARG
    assert lib.mxg_selftest_wait_timeout(a, 0, null) == mxg.MXG_ERR_INVALID_ARG
    # dense bf16 few-column projection: M <= 8, 16 <= N <= 2048, N % 16, K % 64
    for M, N, K in [(9, 96, 5120), (4, 100, 5120), (4, 2064, 5120), (4, 96, 5000), (4, 96, 0)]:
        assert lib.bf16_gemm_small(a, a, M, N, K, a, a, 1 << 20, null) == mxg.MXG_ERR_UNSUPPORTED_SHAPE
        assert lib.bf16_gemm_small_workspace_bytes(M, N, K) == 0
    assert lib.bf16_gemm_small(a, mis, 4, 96, 5120, a, a, 1 << 20, null) == mxg.MXG_ERR_INVALID_ARG
    assert lib.bf16_gemm_small(a, a, 4, 96, 5120, a, a, 256, null) == mxg.MXG_ERR_WORKSPACE
    assert lib.bf16_gemm_small_workspace_bytes(4, 96, 5120) > 256
    # INT8: the streaming path only (M <= 32), shape rules of the INT4 re-pack
    assert lib.w8a16_gemm(a, a, 33, 512, 512, 128, a, a, 1 << 20, null) == mxg.MXG_ERR_UNSUPPORTED_SHAPE
    assert lib.w8a16_gemm(a, a, 5, 512, 512, 96, a, a, 1 << 20, null) == mxg.MXG_ERR_UNSUPPORTED_SHAPE
    assert lib.w8a16_gemm(a, mis, 5, 512, 512, 128, a, a, 1 << 20, null) == mxg.MXG_ERR_INVALID_ARG
    assert lib.w8a16_repack(a, a, 480, 512, 32, a, null) == mxg.MXG_ERR_UNSUPPORTED_SHAPE
    assert lib.w8a16_repack_ct(a, a, 480, 512, 32, a, null) == mxg.MXG_ERR_UNSUPPORTED_SHAPE
    assert lib.w8a16_repack_ct(a, mis, 512, 512, 32, a, null) == mxg.MXG_ERR_INVALID_ARG
    assert lib.w8a16_packed_bytes(5120, 248320, 128) == 5120 * 248320 + 248320 * 40 * 2
    assert lib.w8a16_workspace_bytes(33, 512, 512, 128) == 0


def test_per_call_options_rejected_before_launch(mxg):
    """The *_ex entry points check their options before anything else: a
    path or late_weights value outside its range, or a path the format does
    not have, is MXG_ERR_INVALID_ARG (no kernel runs here)."""
    lib = mxg.raw_lib()
    a = ctypes.c_void_p(4096)
    null = None

    def opts(path, late):
        return ctypes.byref(mxg.GemmOptions(path, late))
    for bad in [opts(3, 0), opts(-1, 0), opts(0, 2)]:
        assert lib.w4a16_gemm_ex(a, a, 5, 512, 512, 128, a, a, 1 << 20, bad, null) == \
            mxg.MXG_ERR_INVALID_ARG
        assert lib.mxfp8_gemm_ex(a, a, a, 4, 256, 512, a, a, 1 << 20, bad, null) == \
            mxg.MXG_ERR_INVALID_ARG
        assert lib.w8a16_gemm_ex(a, a, 5, 512, 512, 128, a, a, 1 << 20, bad, null) == \
            mxg.MXG_ERR_INVALID_ARG
        assert lib.bf16_gemm_small_ex(a, a, 4, 96, 5120, a, a, 1 << 20, bad, null) == \
            mxg.MXG_ERR_INVALID_ARG
    # INT8 has no tensor-core path; the bf16 projection has no path choice
    assert lib.w8a16_gemm_ex(a, a, 5, 512, 512, 128, a, a, 1 << 20, opts(2, 0), null) == \
        mxg.MXG_ERR_INVALID_ARG
    assert lib.bf16_gemm_small_ex(a, a, 4, 96, 5120, a, a, 1 << 20, opts(1, 0), null) == \
        mxg.MXG_ERR_INVALID_ARG
    # valid options reach the usual argument checks
    assert lib.w4a16_gemm_ex(a, a, 0, 512, 512, 128, a, a, 1 << 20, opts(1, 1), null) == \
        mxg.MXG_ERR_INVALID_ARG          # M < 1
    assert lib.w4a16_gemm_ex(a, a, 5, 512, 512, 96, a, a, 1 << 20, null, null) == \
        mxg.MXG_ERR_UNSUPPORTED_SHAPE
    assert lib.bf16_gemm_small_ex(a, a, 4, 96, 5120, a, a, 256, opts(0, 1), null) == \
        mxg.MXG_ERR_WORKSPACE


def test_no_process_wide_settings(mxg):
    """Every choice a caller makes is an argument of its call: the library
    exports no setter that would change another caller's behaviour."""
    names = declared_functions()
    assert not [n for n in names if "set_" in n]
    lib = ctypes.CDLL(mxg.LIB_PATH)
    assert not hasattr(lib, "mxg_set_path") and not hasattr(lib, "mxg_set_early_weight_loads")


def test_static_scratch_status_rejects_bad_arguments(mxg):
    lib = mxg.raw_lib()
    v = ctypes.c_int(0)
    assert lib.w4a16_static_scratch_status(None, 0, None) == mxg.MXG_ERR_INVALID_ARG
    assert lib.w4a16_static_scratch_status(ctypes.byref(v), 2, None) == mxg.MXG_ERR_INVALID_ARG


def test_binding_refuses_to_load_without_the_library(tmp_path):
    """No CPU fallback: a copy of the binding without libmxg.so next to it
    raises at import."""
    import shutil
    import subprocess
    import sys
    pkg = tmp_path / "mxfp8_gemm_speculative_b200"
    pkg.mkdir()
    src = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                       "mxfp8_gemm_speculative_b200", "__init__.py")
    shutil.copy(src, pkg / "__init__.py")
    r = subprocess.run([sys.executable, "-c", "import mxfp8_gemm_speculative_b200"],
                       cwd=tmp_path, capture_output=True, text=True, timeout=300)
    assert r.returncode != 0
    assert "is missing" in r.stderr and "no fallback" in r.stderr


def test_binding_checks_buffers_before_the_call(mxg):
    """The C ABI cannot see buffer sizes, so the binding checks every buffer
    against the call's shape before any launch: type, then size, then
    layout and device (CPU tensors here: the size checks fire first)."""
    import torch
    cuda0 = torch.device("cuda", 0)
    # output: dtype, then exact [M][N]
    with pytest.raises(ValueError, match="bfloat16"):
        mxg._need_out(torch.empty((5, 512), dtype=torch.float32), 5, 512, cuda0)
    with pytest.raises(ValueError, match=r"\[5\]\[512\]"):
        mxg._need_out(torch.empty((5, 256), dtype=torch.bfloat16), 5, 512, cuda0)
    with pytest.raises(ValueError, match=r"\[5\]\[512\]"):
        mxg._need_out(torch.empty((512, 5), dtype=torch.bfloat16), 5, 512, cuda0)
    with pytest.raises(ValueError, match="CUDA"):
        mxg._need_out(torch.empty((5, 512), dtype=torch.bfloat16), 5, 512, cuda0)
    # packed weights: dtype, then at least the bytes the shape needs
    need = mxg.w4a16_packed_bytes(512, 512, 128)
    with pytest.raises(ValueError, match="uint8"):
        mxg._need_weights(torch.empty(need, dtype=torch.int8), torch.uint8, need, cuda0, "packed")
    with pytest.raises(ValueError, match="needs"):
        mxg._need_weights(torch.empty(need - 16, dtype=torch.uint8), torch.uint8, need, cuda0,
                          "packed")
    with pytest.raises(ValueError, match="CUDA"):
        mxg._need_weights(torch.empty(need, dtype=torch.uint8), torch.uint8, need, cuda0, "packed")
    # a shape the library rejects itself (0 bytes) is left to its status
    with pytest.raises(ValueError, match="CUDA"):
        mxg._need_weights(torch.empty(16, dtype=torch.uint8), torch.uint8, 0, cuda0, "packed")
    # caller workspaces are bytes
    with pytest.raises(ValueError, match="uint8"):
        mxg._need_ws(torch.empty(1024, dtype=torch.int32), cuda0)
    # x must be [M][K] for the K of the call
    with pytest.raises(ValueError, match="CUDA"):
        mxg._gemm_buffers(torch.empty((5, 512), dtype=torch.bfloat16), 512, 512, None, None,
                          lambda: 0, None)
