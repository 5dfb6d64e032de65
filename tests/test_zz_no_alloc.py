"""w4a16_gemm_static_scratch: the weight-streaming GEMM with the library's
fixed device scratch instead of a caller workspace, through the C ABI.

Some callers cannot allocate device memory for a workspace: a plain C host
that links only this library, or a serving process whose device memory was
reserved up front by its own pools.  Their entry point must give the same
result as w4a16_gemm: it runs the same kernel in the same fixed reduction
order, so the two are compared bit for bit, and the first of them against
the CPU oracle.  Two calls in a row on different activations each agree (the
second starts from whatever the first left in the shared array).  The status
word of the array is read back and can be cleared.  The file is named to be
collected last, so the suite also runs it after every other test; it must
pass alone in a fresh process as well, and two of its cases start a fresh
process of their own (the array's one-time set-up happens on the first call
in a process).
"""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import assert_parity, bf16_tensor, to_f64

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda", 0)
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def mxg():
    import __graft_entry__
    __graft_entry__.build()
    import mxfp8_gemm_speculative_b200 as m
    return m


# (M, K, N, G): the 27B verify-chunk layers at M = 5 and M = 32 (largest
# scratch: four token tiles), a ragged M, and the small group sizes.
CASES = [
    (5, 5120, 17408, 128),
    (32, 17408, 5120, 128),
    (13, 5120, 5120, 128),
    (3, 1024, 512, 64),
    (8, 512, 1024, 32),
]


def bits(y):
    return y.view(torch.int16)


@pytest.mark.parametrize("M,K,N,G", CASES)
def test_two_calls_match_workspace_entry(mxg, M, K, N, G):
    lay = synth.int4_layer(M, K, N, G, seed=7)
    qw = torch.from_numpy(lay.qweight).to(DEV)
    sc = torch.from_numpy(lay.scales.view(np.int16)).to(DEV)
    packed = mxg.w4a16_repack(qw, sc, G)
    rng = np.random.default_rng(np.random.SeedSequence([7, M, K, N, G]))
    x2 = synth.bf16_bits_of_normals(rng, (M, K))
    xs = [bf16_tensor(lay.X, DEV), bf16_tensor(x2, DEV)]

    ys = [mxg.w4a16_gemm_static_scratch(x, packed, N, K, G) for x in xs]   # back to back
    refs = [mxg.w4a16_gemm(x, packed, N, K, G) for x in xs]
    torch.cuda.synchronize()
    for i, (y, ref) in enumerate(zip(ys, refs)):
        assert torch.equal(bits(y), bits(ref)), f"call {i + 1} M={M} K={K} N={N} G={G}"
    want = oracle.w4a16_gemm(lay.X, lay.qweight, lay.scales, M, N, K, G)
    assert_parity(to_f64(ys[0]), want, f"static scratch vs oracle M={M} K={K} N={N} G={G}")
    assert mxg.w4a16_static_scratch_status() == 0


def test_timeout_status_is_read_and_cleared(mxg):
    """A bounded wait that runs out records MXG_ERR_TIMEOUT in the array's
    status word (the library's self-test kernel, pointed at the array, waits
    on a barrier nothing completes and gives up after 1 ms); the status call
    reads it and, with reset, clears it, and calls work again afterwards."""
    mxg.mxg_selftest_wait_timeout(None, 1000)
    assert mxg.w4a16_static_scratch_status() == mxg.MXG_ERR_TIMEOUT
    assert mxg.w4a16_static_scratch_status(reset=True) == mxg.MXG_ERR_TIMEOUT
    assert mxg.w4a16_static_scratch_status() == 0
    M, K, N, G = 5, 2048, 1024, 128
    lay = synth.int4_layer(M, K, N, G, seed=9)
    packed = mxg.w4a16_repack(torch.from_numpy(lay.qweight).to(DEV),
                              torch.from_numpy(lay.scales.view(np.int16)).to(DEV), G)
    x = bf16_tensor(lay.X, DEV)
    y = mxg.w4a16_gemm_static_scratch(x, packed, N, K, G)
    ref = mxg.w4a16_gemm(x, packed, N, K, G)
    torch.cuda.synchronize()
    assert torch.equal(bits(y), bits(ref))
    assert mxg.w4a16_static_scratch_status() == 0


def test_rejects_before_launch(mxg):
    lay = synth.int4_layer(33, 512, 128, 128, seed=1)
    x = bf16_tensor(lay.X, DEV)
    packed = torch.zeros(mxg.w4a16_packed_bytes(512, 128, 128), dtype=torch.uint8, device=DEV)
    y = torch.empty((33, 128), dtype=torch.bfloat16, device=DEV)
    lib = mxg.raw_lib()
    stream = torch.cuda.current_stream().cuda_stream

    def call(M, N, K, G, yp=y.data_ptr()):
        return lib.w4a16_gemm_static_scratch(x.data_ptr(), packed.data_ptr(), M, N, K, G, yp,
                                             stream)

    assert call(33, 128, 512, 128) == mxg.MXG_ERR_UNSUPPORTED_SHAPE   # M > 32
    assert call(4, 96, 512, 128) == mxg.MXG_ERR_UNSUPPORTED_SHAPE     # N % 64
    assert call(4, 128, 512, 100) == mxg.MXG_ERR_UNSUPPORTED_SHAPE    # group size
    assert call(0, 128, 512, 128) == mxg.MXG_ERR_INVALID_ARG
    assert call(4, 128, 512, 128, y.data_ptr() + 2) == mxg.MXG_ERR_INVALID_ARG


# the array's documented size (include/mxg.h): the weight-streaming path of
# every M <= 32 shape must fit
STATIC_SCRATCH_BYTES = 16 << 20


@pytest.mark.parametrize("K,N", [(5120, 5120), (5120, 17408), (17408, 5120), (5120, 34816),
                                 (5120, 248320)])
def test_largest_shapes_fit_the_array(mxg, K, N):
    # w4a16_workspace_bytes also covers the tensor-core plan, which the
    # static entry never runs; the INT8 query is the same streaming planner
    # (same grid, token tiles, counters and partial sums) and nothing else
    for M in (1, 8, 16, 24, 32):
        need = mxg.raw_lib().w8a16_workspace_bytes(M, N, K, 128)
        assert 0 < need <= STATIC_SCRATCH_BYTES, (M, K, N, need)


def run_fresh(script: str) -> str:
    """Runs `script` in a new Python process (repository root on the path)
    and returns its output; the test fails with that output on a nonzero
    exit."""
    env = dict(os.environ)
    env["PYTHONPATH"] = ROOT + os.pathsep + os.path.join(ROOT, "tests") + os.pathsep + \
        env.get("PYTHONPATH", "")
    r = subprocess.run([sys.executable, "-c", script], capture_output=True, text=True,
                       timeout=300, cwd=ROOT, env=env)
    assert r.returncode == 0, r.stdout + r.stderr
    return r.stdout


FRESH_PRELUDE = """
import numpy as np, torch, synth
import mxfp8_gemm_speculative_b200 as mxg
from helpers import bf16_tensor
DEV = torch.device("cuda", 0)
M, K, N, G = 5, 5120, 17408, 128
lay = synth.int4_layer(M, K, N, G, seed=21)
packed = mxg.w4a16_repack(torch.from_numpy(lay.qweight).to(DEV),
                          torch.from_numpy(lay.scales.view(np.int16)).to(DEV), G)
x = bf16_tensor(lay.X, DEV)
torch.cuda.synchronize()
"""


def test_first_call_on_a_side_stream(mxg):
    """In a fresh process, the first call (which zeroes the array's header
    and counters on its stream) runs on a side stream, then a second call on
    the same stream; both equal w4a16_gemm bit for bit."""
    out = run_fresh(FRESH_PRELUDE + """
side = torch.cuda.Stream()
with torch.cuda.stream(side):
    y1 = mxg.w4a16_gemm_static_scratch(x, packed, N, K, G, stream=side)
    y2 = mxg.w4a16_gemm_static_scratch(x, packed, N, K, G, stream=side)
side.synchronize()
ref = mxg.w4a16_gemm(x, packed, N, K, G)
torch.cuda.synchronize()
assert torch.equal(y1.view(torch.int16), ref.view(torch.int16))
assert torch.equal(y2.view(torch.int16), ref.view(torch.int16))
assert mxg.w4a16_static_scratch_status(stream=side) == 0
print("side-stream ok")
""")
    assert "side-stream ok" in out


def test_first_call_inside_a_capture_is_refused_then_works(mxg):
    """In a fresh process, a first call made while its stream is captured is
    refused with MXG_ERR_CAPTURE (its one-time set-up cannot be captured);
    the refusal is not remembered: the next call, outside the capture, sets
    up and matches w4a16_gemm."""
    out = run_fresh(FRESH_PRELUDE + """
s = torch.cuda.Stream()
y = torch.empty((M, N), dtype=torch.bfloat16, device=DEV)
refused = None
g = torch.cuda.CUDAGraph()
with torch.cuda.graph(g, stream=s):
    try:
        mxg.w4a16_gemm_static_scratch(x, packed, N, K, G, out=y, stream=s)
    except mxg.MxgError as e:
        refused = e.status
assert refused == mxg.MXG_ERR_CAPTURE, refused
y2 = mxg.w4a16_gemm_static_scratch(x, packed, N, K, G)
ref = mxg.w4a16_gemm(x, packed, N, K, G)
torch.cuda.synchronize()
assert torch.equal(y2.view(torch.int16), ref.view(torch.int16))
print("capture refusal ok")
""")
    assert "capture refusal ok" in out
