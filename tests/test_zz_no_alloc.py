"""The allocation-free packing entry point, checked against the ordinary one.

bitlinear_pack_weights_noalloc serves callers that cannot allocate device
memory when they pack weights (for example while capturing a CUDA graph,
where cudaMalloc is not allowed, or inside a runtime whose memory pool owns
all device memory).  It keeps its partial sums in a fixed array inside the
library instead of a caller-supplied workspace.  This file is named so that
pytest collects it last; it must pass alone in a fresh process and after the
other tests.
"""
import ctypes

import numpy as np
import pytest
import torch

import ternary_weight_linear_bitlinear_b200 as bl
from ternary_weight_linear_bitlinear_b200 import build as blbuild
from workloads import Problem, draw

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    blbuild.build()
    return bl.lib()


def _noalloc(lib, W):
    d_out, d_in = W.shape
    packed = torch.empty(bl.packed_words(d_out, d_in), dtype=torch.int32, device=W.device)
    gamma = torch.empty(1, dtype=torch.float32, device=W.device)
    st = lib.bitlinear_pack_weights_noalloc(
        ctypes.c_void_p(W.data_ptr()), d_out, d_in, 1e-5, ctypes.c_void_p(packed.data_ptr()),
        ctypes.c_void_p(gamma.data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == bl.OK, bl.status_string(st)
    return packed, gamma


def test_noalloc_pack_matches_workspace_pack(lib):
    dev = torch.device("cuda:0")
    # Two calls in a row with different shapes and values: the second must
    # not see anything left in the shared array by the first.
    for (d_out, d_in, seed) in ((6912, 2560, 21), (272, 768, 22)):
        W = draw(Problem("n", d_in, d_out, 1, 0.02, 0.0, 1.0, seed))[0].to(dev)
        ref = bl.pack_weights(W, 1e-5)
        packed, gamma = _noalloc(lib, W)
        torch.cuda.synchronize()
        # Same grid and reduction order as the workspace path: the same bits.
        assert int(gamma.view(torch.int32).item()) == int(ref.gamma.view(torch.int32).item())
        np.testing.assert_array_equal(packed.cpu().numpy(), ref.packed.cpu().numpy())
    assert bl.device_error(clear=True) == bl.OK


def test_noalloc_rejects_bad_arguments(lib):
    S0 = ctypes.c_void_p(0)
    P = ctypes.c_void_p
    f = lib.bitlinear_pack_weights_noalloc
    assert f(None, 64, 256, 1e-5, P(0x1000), P(0x2000), S0) == bl.ERR_INVALID_ARG
    assert f(P(0x1000), 64, 100, 1e-5, P(0x1000), P(0x2000), S0) == bl.ERR_UNSUPPORTED_SHAPE
    assert f(P(0x1000), 64, 65536 * 2, 1e-5, P(0x1000), P(0x2000), S0) == bl.ERR_UNSUPPORTED_SHAPE
    assert f(P(0x1004), 64, 256, 1e-5, P(0x1000), P(0x2000), S0) == bl.ERR_MISALIGNED
