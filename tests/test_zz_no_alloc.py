"""w4a16_gemm_static_scratch: the weight-streaming GEMM with the library's
fixed device scratch instead of a caller workspace, through the C ABI.

Two calls in a row on different activations must each agree with
w4a16_gemm (caller workspace) within the layer's tolerance: the second call
starts from whatever the first left in the shared array.  The file is named
to be collected last, so the suite also runs it after every other test; it
must pass alone in a fresh process as well.
"""
import numpy as np
import pytest
import torch

import synth
from helpers import assert_parity, bf16_tensor, to_f64

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda", 0)


@pytest.fixture(scope="module")
def mxg():
    import __graft_entry__
    __graft_entry__.build()
    import mxfp8_gemm_speculative_b200 as m
    m.mxg_set_path(0)
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


@pytest.mark.parametrize("M,K,N,G", CASES)
def test_two_calls_match_workspace_entry(mxg, M, K, N, G):
    lay = synth.int4_layer(M, K, N, G, seed=7)
    qw = torch.from_numpy(lay.qweight).to(DEV)
    sc = torch.from_numpy(lay.scales.view(np.int16)).to(DEV)
    packed = mxg.w4a16_repack(qw, sc, G)
    rng = np.random.default_rng(np.random.SeedSequence([7, M, K, N, G]))
    xs = [bf16_tensor(lay.X, DEV), bf16_tensor(synth.bf16_bits_of_normals(rng, (M, K)), DEV)]

    ys = [mxg.w4a16_gemm_static_scratch(x, packed, N, K, G) for x in xs]   # back to back
    refs = [mxg.w4a16_gemm(x, packed, N, K, G) for x in xs]
    torch.cuda.synchronize()
    for i, (y, ref) in enumerate(zip(ys, refs)):
        assert_parity(to_f64(y), to_f64(ref), f"call {i + 1} M={M} K={K} N={N} G={G}")


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
