"""The Python binding's argument marshalling, on CPU: every GEMM entry is
called with CPU tensors against a recording stand-in for libmxg.so (the
device checks and the stream lookup are stubbed), and the test checks the
pointers, sizes and shape arguments each C function receives, in the order
include/mxg.h declares them.  No kernel runs."""
import ctypes

import pytest
import torch


class FakeLib:
    """Records every C call and returns MXG_OK; the size queries and the
    status strings go to the real library (they need no GPU)."""

    def __init__(self, real):
        self.calls = []
        self.devices = []     # the device current during each recorded call
        self.current = []
        self._real = real

    def __getattr__(self, name):
        if name == "w8a16_workspace_bytes":
            # the real query looks at the current device (none here): the
            # streaming path's rule, M <= 32, with a stand-in size
            return lambda M, N, K, G: 4096 if 1 <= M <= 32 else 0
        if name == "mxfp8_packed_workspace_bytes":
            return lambda M, N, K: 4096 if 1 <= M <= 16 else 0
        if name.endswith("_bytes") or name == "mxg_status_string":
            return getattr(self._real, name)

        def fn(*args):
            self.calls.append((name, args))
            self.devices.append(self.current[-1] if self.current else None)
            return 0
        return fn


def _val(a):
    return a.value if isinstance(a, ctypes.c_void_p) else a


@pytest.fixture()
def fake(monkeypatch):
    import __graft_entry__
    __graft_entry__.build()
    import mxfp8_gemm_speculative_b200 as m
    lib = FakeLib(m._lib)
    monkeypatch.setattr(m, "_lib", lib)

    def need_cpu(t, dtype, name):
        if t.dtype != dtype:
            raise ValueError(f"{name} must be {dtype}")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    monkeypatch.setattr(m, "_need", need_cpu)

    class OnDevice:
        """Records the device made current around each C call."""

        def __init__(self, device):
            self.device = device

        def __enter__(self):
            lib.current.append(self.device)

        def __exit__(self, *exc):
            lib.current.pop()
    monkeypatch.setattr(m, "_on_device", OnDevice)
    monkeypatch.setattr(m, "_stream",
                        lambda stream=None, device=None: ("stream", stream, device))
    monkeypatch.setattr(m, "workspace",
                        lambda nbytes, device=None, stream=None: torch.zeros(max(nbytes, 256),
                                                                             dtype=torch.uint8))
    monkeypatch.setattr(m, "_need_bytes", lambda *a: 4096)
    return m, lib


def bf16(*shape):
    return torch.zeros(shape, dtype=torch.bfloat16)


def test_w4a16_calls(fake):
    m, lib = fake
    M, K, N, G = 5, 512, 256, 128
    x = bf16(M, K)
    packed = torch.zeros(m.w4a16_packed_bytes(K, N, G), dtype=torch.uint8)
    y = m.w4a16_gemm(x, packed, N, K, G)
    name, a = lib.calls[-1]
    assert name == "w4a16_gemm_ex"
    assert [_val(v) for v in a[:6]] == [x.data_ptr(), packed.data_ptr(), M, N, K, G]
    assert _val(a[6]) == y.data_ptr() and tuple(y.shape) == (M, N)
    assert a[8] == 4096          # the workspace's bytes
    assert a[9] is None          # default options: NULL
    m.w4a16_gemm(x, packed, N, K, G, path=m.PATH_STREAM, late_weights=True)
    opts = lib.calls[-1][1][9].contents
    assert (opts.path, opts.late_weights) == (1, 1)
    call, y2 = m.prepare_w4a16_gemm(x, packed, N, K, G)
    call()
    name, a = lib.calls[-1]
    assert name == "w4a16_gemm_ex" and _val(a[6]) == y2.data_ptr() and a[2:6] == (M, N, K, G)
    m.w4a16_gemm_static_scratch(x, packed, N, K, G)
    name, a = lib.calls[-1]
    assert name == "w4a16_gemm_static_scratch" and a[2:6] == (M, N, K, G)
    codes, w32, w16 = m.w4a16_unpack(packed, K, N, G)
    name, a = lib.calls[-1]
    assert name == "w4a16_unpack" and a[1:4] == (K, N, G)
    assert [_val(v) for v in a[4:7]] == [codes.data_ptr(), w32.data_ptr(), w16.data_ptr()]
    # a caller output and workspace are used as given
    out = bf16(M, N)
    ws = torch.zeros(8192, dtype=torch.uint8)
    m.w4a16_gemm(x, packed, N, K, G, out=out, workspace_buf=ws)
    name, a = lib.calls[-1]
    assert _val(a[6]) == out.data_ptr() and _val(a[7]) == ws.data_ptr() and a[8] == 8192


def test_w4a16_rejects_mismatched_buffers(fake):
    m, lib = fake
    M, K, N, G = 5, 512, 256, 128
    x = bf16(M, K)
    packed = torch.zeros(m.w4a16_packed_bytes(K, N, G), dtype=torch.uint8)
    n0 = len(lib.calls)
    with pytest.raises(ValueError):
        m.w4a16_gemm(x, packed[:-16], N, K, G)            # too few weight bytes
    with pytest.raises(ValueError):
        m.w4a16_gemm(x, packed, N, K, G, out=bf16(M, N - 64))
    with pytest.raises(ValueError):
        m.w4a16_gemm(bf16(M, K - 64), packed, N, K, G)    # x of another K
    with pytest.raises(ValueError):
        m.w4a16_gemm(x, packed, N, K, G, workspace_buf=torch.zeros(64, dtype=torch.int32))
    with pytest.raises(ValueError):
        m.prepare_w4a16_gemm(x, packed[:100], N, K, G)
    with pytest.raises(ValueError):
        m.w4a16_gemm_static_scratch(x, packed[:100], N, K, G)
    assert len(lib.calls) == n0                            # nothing reached the library


def test_w8a16_calls(fake):
    m, lib = fake
    M, K, N, G = 4, 512, 256, 128
    x = bf16(M, K)
    packed = torch.zeros(int(m.raw_lib().w8a16_packed_bytes(K, N, G)), dtype=torch.uint8)
    y = m.w8a16_gemm(x, packed, N, K, G)
    name, a = lib.calls[-1]
    assert name == "w8a16_gemm_ex" and a[2:6] == (M, N, K, G) and _val(a[6]) == y.data_ptr()
    call, _ = m.prepare_w8a16_gemm(x, packed, N, K, G)
    call()
    assert lib.calls[-1][0] == "w8a16_gemm_ex"
    with pytest.raises(ValueError):
        m.w8a16_gemm(x, packed[: packed.numel() // 2], N, K, G)
    with pytest.raises(ValueError):
        m.prepare_w8a16_gemm(bf16(M, K + 64), packed, N, K, G)
    with pytest.raises(m.MxgError):
        m.w8a16_gemm(bf16(33, K), packed, N, K, G)        # streaming path only


def test_mxfp8_calls(fake):
    m, lib = fake
    M, K, N = 4, 512, 256
    x = bf16(M, K)
    wq = torch.zeros((N, K), dtype=torch.uint8)
    ws = torch.zeros((N, K // 32), dtype=torch.uint8)
    y = m.mxfp8_gemm(x, wq, ws)
    name, a = lib.calls[-1]
    assert name == "mxfp8_gemm_ex"
    assert [_val(v) for v in a[:3]] == [x.data_ptr(), wq.data_ptr(), ws.data_ptr()]
    assert a[3:6] == (M, N, K) and _val(a[6]) == y.data_ptr()
    call, _ = m.prepare_mxfp8_gemm(x, wq, ws)
    call()
    assert lib.calls[-1][0] == "mxfp8_gemm_ex"
    with pytest.raises(ValueError):
        m.mxfp8_gemm(x, wq, ws[:, :-1])
    with pytest.raises(ValueError):
        m.mxfp8_gemm(x, wq, ws, out=bf16(M + 1, N))


def test_mxfp8_packed_calls(fake):
    m, lib = fake
    M, K, N = 4, 512, 256
    x = bf16(M, K)
    wq = torch.zeros((N, K), dtype=torch.uint8)
    ws = torch.zeros((N, K // 32), dtype=torch.uint8)
    packed = m.mxfp8_repack(wq, ws)
    name, a = lib.calls[-1]
    assert name == "mxfp8_repack"
    assert [_val(v) for v in a[:2]] == [wq.data_ptr(), ws.data_ptr()]
    assert a[2:4] == (N, K) and _val(a[4]) == packed.data_ptr()
    assert packed.numel() == N * K + N * K // 32
    y = m.mxfp8_gemm_packed(x, packed, N, K)
    name, a = lib.calls[-1]
    assert name == "mxfp8_gemm_packed_ex"
    assert [_val(v) for v in a[:2]] == [x.data_ptr(), packed.data_ptr()]
    assert a[2:5] == (M, N, K) and _val(a[5]) == y.data_ptr() and a[7] == 4096 and a[8] is None
    call, y2 = m.prepare_mxfp8_gemm_packed(x, packed, N, K)
    call()
    name, a = lib.calls[-1]
    assert name == "mxfp8_gemm_packed_ex" and _val(a[5]) == y2.data_ptr()
    n0 = len(lib.calls)
    with pytest.raises(ValueError):
        m.mxfp8_gemm_packed(x, packed[:-16], N, K)         # too few weight bytes
    with pytest.raises(m.MxgError):
        m.mxfp8_gemm_packed(bf16(17, K), packed, N, K)    # M <= 16 only
    with pytest.raises(m.MxgError):
        m.mxfp8_repack(torch.zeros((96, K), dtype=torch.uint8),
                       torch.zeros((96, K // 32), dtype=torch.uint8))   # N % 64
    assert len(lib.calls) == n0


def test_bf16_small_calls(fake):
    m, lib = fake
    M, K, N = 4, 5120, 96
    x, w = bf16(M, K), bf16(N, K)
    y = m.bf16_gemm_small(x, w)
    name, a = lib.calls[-1]
    assert name == "bf16_gemm_small_ex" and a[2:5] == (M, N, K) and _val(a[5]) == y.data_ptr()
    call, _ = m.prepare_bf16_gemm_small(x, w)
    call()
    assert lib.calls[-1][0] == "bf16_gemm_small_ex"
    with pytest.raises(ValueError):
        m.bf16_gemm_small(x, w, out=bf16(M, N + 16))
    with pytest.raises(m.MxgError):
        m.bf16_gemm_small(bf16(9, K), w)                  # M <= 8


def test_repack_and_decoder_shapes(fake):
    m, lib = fake
    K, N, G = 512, 256, 128
    qw = torch.zeros((K // 8, N), dtype=torch.int32)
    sc = torch.zeros((K // G, N), dtype=torch.float16)
    packed = m.w4a16_repack(qw, sc, G)
    name, a = lib.calls[-1]
    assert name == "w4a16_repack" and a[2:5] == (K, N, G) and _val(a[5]) == packed.data_ptr()
    assert packed.numel() == m.w4a16_packed_bytes(K, N, G)
    m.w4a16_repack_ct(qw.T.contiguous(), sc.T.contiguous(), G)
    assert lib.calls[-1][0] == "w4a16_repack_ct" and lib.calls[-1][1][2:5] == (K, N, G)
    m.w4a16_repack_fused([(qw, sc), (qw, sc)], G)
    name, a = lib.calls[-1]
    assert name == "w4a16_repack_fused" and a[0] == 2 and a[4:6] == (K, G)
    q8 = torch.zeros((K // 4, N), dtype=torch.int32)
    m.w8a16_repack(q8, sc, G)
    assert lib.calls[-1][0] == "w8a16_repack" and lib.calls[-1][1][2:5] == (K, N, G)
    n0 = len(lib.calls)
    with pytest.raises(ValueError):
        m.w4a16_repack(qw, sc[:, :-64], G)                 # scales of another N
    with pytest.raises(ValueError):
        m.w4a16_repack(qw, torch.zeros((K // 64, N), dtype=torch.float16), G)
    with pytest.raises(ValueError):
        m.w4a16_repack_ct(qw.T.contiguous(), sc, G)        # GPTQ-oriented scales
    with pytest.raises(ValueError):
        m.w4a16_repack_fused([(qw, sc), (qw, sc[:, :64])], G)
    with pytest.raises(ValueError):
        m.w8a16_repack(q8, sc[:1], G)
    with pytest.raises(ValueError):
        m.w8a16_repack_ct(q8.T.contiguous(), sc, G)
    with pytest.raises(ValueError):
        m.mxfp8_dequant(torch.zeros((N, K), dtype=torch.uint8),
                        torch.zeros((N, K // 64), dtype=torch.uint8))
    with pytest.raises(ValueError):
        m.mxg_workspace_status(torch.zeros(128, dtype=torch.uint8))
    with pytest.raises(ValueError):
        m.mxg_selftest_wait_timeout(torch.zeros(64, dtype=torch.int32), 1000)
    assert len(lib.calls) == n0
    w16 = m.mxfp8_dequant(torch.zeros((N, K), dtype=torch.uint8),
                          torch.zeros((N, K // 32), dtype=torch.uint8))
    name, a = lib.calls[-1]
    assert name == "mxfp8_dequant" and a[2:4] == (N, K) and _val(a[4]) == w16.data_ptr()


def test_calls_run_on_the_tensors_device_and_stream(fake):
    """Every C call runs with its tensors' device current (the library plans
    for, and launches on, the current device) and gets a stream of that
    device: the caller's, or the device's current one."""
    m, lib = fake
    M, K, N, G = 5, 512, 256, 128
    x = bf16(M, K)
    packed = torch.zeros(m.w4a16_packed_bytes(K, N, G), dtype=torch.uint8)
    sentinel = object()
    m.w4a16_gemm(x, packed, N, K, G, stream=sentinel)
    assert lib.devices[-1] == x.device
    assert lib.calls[-1][1][-1] == ("stream", sentinel, x.device)
    m.w4a16_gemm(x, packed, N, K, G)
    assert lib.calls[-1][1][-1] == ("stream", None, x.device)
    call, _ = m.prepare_w4a16_gemm(x, packed, N, K, G, stream=sentinel)
    call()
    assert lib.devices[-1] == x.device and lib.calls[-1][1][-1] == ("stream", sentinel, x.device)
    wq = torch.zeros((N, K), dtype=torch.uint8)
    ws = torch.zeros((N, K // 32), dtype=torch.uint8)
    m.mxfp8_gemm(x, wq, ws)
    assert lib.devices[-1] == x.device
    m.w4a16_repack(torch.zeros((K // 8, N), dtype=torch.int32),
                   torch.zeros((K // G, N), dtype=torch.float16), G)
    assert lib.devices[-1] == x.device
    assert not lib.current                      # every device context was left


def test_stream_of_another_device_is_refused():
    """A stream that lives on another device than the call's tensors is
    refused before any C call."""
    import __graft_entry__
    __graft_entry__.build()
    import mxfp8_gemm_speculative_b200 as m

    class FakeStream:
        device = torch.device("cuda", 1)
        cuda_stream = 0
    with pytest.raises(ValueError):
        m._stream(FakeStream(), torch.device("cuda", 0))
    assert m._stream(FakeStream(), torch.device("cuda", 1)).value is None
