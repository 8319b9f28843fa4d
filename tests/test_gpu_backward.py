"""Parity of bitlinear_backward (straight-through-estimator gradients) with
the oracle's double-precision statement of the same.

Bound, from the arithmetic: every product is exact in fp32 (bf16 dY times
W~ in {-1, 0, 1}; bf16 dY times bf16 X^), the kernels sum R of them in fp32
(R = d_out for dX, T for dW) and multiply by gamma once, so
|g - ref| <= (R + 1) 2^-24 gamma sum |terms|; a bf16 output adds 2^-8 |ref|.
The tests allow twice the fp32 term.
"""
import numpy as np
import pytest
import torch

import oracle
import ternary_weight_linear_bitlinear_b200 as bl
from ternary_weight_linear_bitlinear_b200 import build as blbuild
from workloads import ALL, Problem, bf16_bits, draw

pytestmark = pytest.mark.gpu
EPS = 1e-5


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    blbuild.build()
    bl.lib()
    yield
    assert bl.device_error(clear=True) == bl.OK


def _setup(d_out, d_in, T, seed):
    W, X = draw(Problem("bw", d_in, d_out, max(T, 1), 0.02, 0.01, 50.0, seed))
    Wn = W.numpy()
    g = oracle.absmean_gamma(Wn)
    wq = oracle.ternarize(Wn, g, EPS)
    xq, beta, _, _ = oracle.quant_act(bf16_bits(X[:T]) if T else np.zeros((0, d_in), np.uint16))
    gen = torch.Generator().manual_seed(seed + 7)
    dY = torch.randn(T, d_out, generator=gen).to(torch.bfloat16)
    w = bl.PackedTernary(torch.from_numpy(oracle.pack(wq).view(np.int32)).cuda(),
                         torch.tensor([g], device="cuda"), d_out, d_in)
    return w, wq, g, xq, beta, dY


def _check(got, ref, mag, R, bf16_out):
    bound = 2.0 * (R + 1) * 2.0 ** -24 * mag
    if bf16_out:
        bound = bound + 2.0 ** -8 * np.abs(ref) * (1 + 1e-3)
    err = np.abs(got.astype(np.float64) - ref)
    bad = err > bound
    assert not bad.any(), "max excess %g at %s" % ((err - bound).max(), np.argwhere(bad)[:3])


CASES = [(256, 256, 1), (256, 512, 17), (512, 1024, 300), (1024, 256, 600), (768, 768, 256)]


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("d_out,d_in,T", CASES)
def test_backward_matches_oracle(d_out, d_in, T, out_dtype):
    w, wq, g, xq, beta, dY = _setup(d_out, d_in, T, 31)
    dX, dW = bl.backward(w, torch.from_numpy(xq).cuda(), torch.from_numpy(beta).cuda(),
                         dY.cuda(), out_dtype=out_dtype)
    torch.cuda.synchronize()
    dy_bits = bf16_bits(dY)
    rX, rW = oracle.backward(wq, g, xq, beta, dy_bits)
    # Magnitudes: the same sums over |terms|.
    aW = np.abs(wq).astype(np.int8)
    xh_bits = np.vectorize(oracle.dequant_act_bf16)(xq, beta[:, None]).astype(np.uint16)
    mX, _ = oracle.backward(aW, g, xq, beta, dy_bits & np.uint16(0x7FFF), want_dw=False)
    aX = np.abs(oracle.bf16_bits_to_f32(xh_bits))
    mW = g * (np.abs(oracle.bf16_bits_to_f32(dy_bits)).T.astype(np.float64) @ aX.astype(np.float64))
    bf = out_dtype == torch.bfloat16
    _check(dX.float().cpu().numpy(), rX, mX, d_out, bf)
    _check(dW.float().cpu().numpy(), rW, mW, T, bf)


def test_backward_one_gradient_only_and_no_tokens():
    w, wq, g, xq, beta, dY = _setup(256, 512, 40, 5)
    dX, dW = bl.backward(w, None, None, dY.cuda(), want_dw=False)
    assert dW is None
    rX, _ = oracle.backward(wq, g, xq, beta, bf16_bits(dY), want_dw=False)
    np.testing.assert_allclose(dX.cpu().numpy(), rX, rtol=1e-4, atol=1e-6)
    w0, _, _, xq0, beta0, dY0 = _setup(256, 512, 0, 5)
    dX0, dW0 = bl.backward(w0, torch.from_numpy(xq0).cuda(), torch.from_numpy(beta0).cuda(),
                           dY0.cuda())
    assert dX0.shape == (0, 512) and not dW0.any()


def test_backward_prefill_full_size_sampled():
    """2048 tokens, 4096 -> 11008: 128 sampled entries of each gradient, each
    against the oracle on the one column (or row) pair it depends on."""
    p = ALL["prefill_2048x4096x11008"].problems[0]
    w, wq, g, xq, beta, dY = _setup(p.d_out, p.d_in, p.tokens, 2)
    dX, dW = bl.backward(w, torch.from_numpy(xq).cuda(), torch.from_numpy(beta).cuda(),
                         dY.cuda())
    dX, dW = dX.cpu().numpy(), dW.cpu().numpy()
    dy = bf16_bits(dY)
    rng = np.random.default_rng(8)
    for _ in range(128):
        t, k, o = (int(rng.integers(0, p.tokens)), int(rng.integers(0, p.d_in)),
                   int(rng.integers(0, p.d_out)))
        rx, _ = oracle.backward(wq[:, k:k + 1], g, None, None, dy[t:t + 1], want_dw=False)
        mx, _ = oracle.backward(np.abs(wq[:, k:k + 1]), g, None, None,
                                dy[t:t + 1] & np.uint16(0x7FFF), want_dw=False)
        _check(dX[t:t + 1, k:k + 1], rx, mx, p.d_out, False)
        _, rw = oracle.backward(wq[o:o + 1, k:k + 1], g, xq[:, k:k + 1], beta, dy[:, o:o + 1],
                                want_dx=False)
        _, mw = oracle.backward(wq[o:o + 1, k:k + 1], g, np.abs(xq[:, k:k + 1]), beta,
                                dy[:, o:o + 1] & np.uint16(0x7FFF), want_dx=False)
        _check(dW[o:o + 1, k:k + 1], rw, mw, p.tokens, False)


def test_backward_rejects_bad_shapes():
    w = bl.PackedTernary(torch.zeros(16 * 256 // 16, dtype=torch.int32, device="cuda"),
                         torch.ones(1, device="cuda"), 16, 256)
    with pytest.raises(bl.BitLinearError):       # d_out must be a multiple of 256
        bl.backward(w, None, None, torch.zeros(4, 16, dtype=torch.bfloat16, device="cuda"),
                    want_dw=False)
