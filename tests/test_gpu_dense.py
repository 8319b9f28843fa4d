"""Parity of the dense bf16 context layer (bitlinear_dense_bf16_forward)
with the oracle's double-precision product of the same bf16 operands.

Bound, from the arithmetic: the kernels form each product and sum in fp32
(fused multiply-add, any order), so |y32 - y| <= K u32 sum_k |w_k x_k| with
u32 = 2^-24 (first-order bound of a K-term fp32 dot product); the bf16
output adds one rounding, |bf16(y32) - y32| <= 2^-8 |y32|.  The tests allow
twice the accumulation term.
"""
import numpy as np
import pytest
import torch

import oracle
import ternary_weight_linear_bitlinear_b200 as bl
from ternary_weight_linear_bitlinear_b200 import build as blbuild
from workloads import ALL, bf16_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    blbuild.build()
    bl.lib()
    yield
    assert bl.device_error(clear=True) == bl.OK


def _abs_bits(b):
    return np.asarray(b, dtype=np.uint16) & np.uint16(0x7FFF)


def _operands(d_out, d_in, T, seed):
    g = torch.Generator().manual_seed(seed)
    W = (torch.randn(d_out, d_in, generator=g) * 0.02).to(torch.bfloat16)
    X = torch.randn(T, d_in, generator=g).to(torch.bfloat16)
    return W, X


def _check(y_gpu, y_ref, mag, K, bf16_out):
    err = np.abs(y_gpu.astype(np.float64) - y_ref)
    bound = 2.0 * K * 2.0 ** -24 * mag
    if bf16_out:
        bound = bound + 2.0 ** -8 * np.abs(y_ref) * (1 + 2.0 * K * 2.0 ** -24)
    bad = err > bound
    assert not bad.any(), "max excess %g at %s" % ((err - bound).max(), np.argwhere(bad)[:3])


CASES = [
    # (d_out, d_in, T): GEMV for T <= 16, tcgen05 GEMM above
    (16, 256, 1), (272, 1024, 3), (6912, 2560, 1), (400, 4096, 16), (144, 65536, 2),
    (144, 256, 17), (400, 1024, 100), (1040, 512, 300), (272, 768, 513),
]


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("d_out,d_in,T", CASES)
def test_dense_matches_oracle(d_out, d_in, T, out_dtype):
    W, X = _operands(d_out, d_in, T, 5)
    wb, xb = bf16_bits(W), bf16_bits(X)
    y_ref = oracle.dense_bf16(wb, xb)
    mag = oracle.dense_bf16(_abs_bits(wb), _abs_bits(xb))
    y = bl.dense_bf16_forward(W.cuda(), X.cuda(), out_dtype=out_dtype)
    torch.cuda.synchronize()
    _check(y.float().cpu().numpy(), y_ref, mag, d_in, out_dtype == torch.bfloat16)


def test_dense_prefill_full_size_sampled():
    """The prefill shape (2048 x 4096 -> 11008) on 512 sampled outputs."""
    p = ALL["prefill_2048x4096x11008"].problems[0]
    W, X = _operands(p.d_out, p.d_in, p.tokens, 11)
    y = bl.dense_bf16_forward(W.cuda(), X.cuda(), out_dtype=torch.bfloat16).float().cpu().numpy()
    wb, xb = bf16_bits(W), bf16_bits(X)
    rng = np.random.default_rng(3)
    ts = rng.integers(0, p.tokens, 512)
    os_ = rng.integers(0, p.d_out, 512)
    ref = np.array([oracle.dense_bf16_dot(wb[o], xb[t]) for t, o in zip(ts, os_)])
    mag = np.array([oracle.dense_bf16_dot(_abs_bits(wb[o]), _abs_bits(xb[t]))
                    for t, o in zip(ts, os_)])
    _check(y[ts, os_], ref, mag, p.d_in, True)


def test_dense_rejects_bad_shapes():
    W = torch.zeros(16, 200, dtype=torch.bfloat16, device="cuda")
    X = torch.zeros(1, 200, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(bl.BitLinearError):
        bl.dense_bf16_forward(W, X)
    W = torch.zeros(16, 256, dtype=torch.bfloat16, device="cuda")
    X = torch.zeros(0, 256, dtype=torch.bfloat16, device="cuda")
    assert bl.dense_bf16_forward(W, X).shape == (0, 16)
