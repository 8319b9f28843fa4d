"""Parity of the W1A4 path (sign-binarised weights, 4-bit activation codes)
on the GPU with the oracle: packed bits and codes bit for bit, int32
accumulators bit for bit, rescaled outputs within the output bar.

The regime is the W1A4 of "The End of Matrix Multiplications: Welcome to
Addition" (Technical Details); binary weights {-1, +1} are those of "BitNet
b1.58: Mathematical Foundations ...", section 1, and the k-bit activation
quantiser with Q_b = 2^(k-1) that of its section 2.
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
NORM_EPS = 1e-5


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    blbuild.build()
    bl.lib()
    yield
    assert bl.device_error(clear=True) == bl.OK


def dev():
    return torch.device("cuda:0")


def to_dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(dev())


def check_y(y_gpu, acc_ref, gamma, beta, out_bf16, act_bits):
    qmax = 2 ** (act_bits - 1) - 1
    y_ref = oracle.rescale(acc_ref, gamma, beta, act_bits=act_bits)
    scale = beta.astype(np.float64)[:, None] * gamma / qmax
    yg = y_gpu.float().cpu().numpy().astype(np.float64)
    tol = (1e-2 if out_bf16 else 1e-5) * np.maximum(np.abs(y_ref), scale)
    bad = np.abs(yg - y_ref) > tol
    assert not bad.any(), "y mismatch at %s" % (np.argwhere(bad)[:5],)


def binary_weights(W):
    Wn = W.numpy()
    g = oracle.absmean_gamma(Wn)
    wq = oracle.binarize(Wn)
    w = bl.PackedBinary(to_dev(oracle.pack_w1(wq).view(np.int32)),
                        torch.tensor([g], device=dev()), W.shape[0], W.shape[1])
    return wq, g, w


# ------------------------------------------------------------- packing ---

@pytest.mark.parametrize("d_out,d_in", [(16, 256), (48, 768), (272, 1024), (6912, 2560),
                                        (32, 11008), (16, 65536)])
def test_pack_w1_matches_oracle(d_out, d_in):
    W = draw(Problem("p1", d_in, d_out, 1, 0.02, 0.0, 1.0, 3))[0]
    W[0, :7] = torch.tensor([0.0, -0.0, 1e-30, -1e-30, 0.5, -0.5, 0.0])
    Wd = W.to(dev())
    own = bl.pack_weights_w1(Wd)
    torch.cuda.synchronize()
    g = oracle.absmean_gamma(W.numpy())
    assert abs(own.gamma.item() - g) <= 1e-6 * g
    np.testing.assert_array_equal(own.packed.cpu().numpy().view(np.uint32),
                                  oracle.pack_w1(oracle.binarize(W.numpy())))
    given = bl.pack_weights_w1(Wd, gamma=torch.tensor([g], device=dev()))
    assert given.gamma.item() == np.float32(g)


# ----------------------------------------------------------- quantiser ---

@pytest.mark.parametrize("T,K,per_tensor", [(1, 2560, False), (5, 1024, False), (16, 4096, False),
                                            (300, 4096, False), (40, 1024, True)])
def test_quant_act_4bit_matches_oracle(T, K, per_tensor):
    X = draw(Problem("q4", K, 16, T, 0.02, 0.01, 50.0, 8))[1]
    xq_r, b_r, s_r, r_r = oracle.quant_act(bf16_bits(X), eps=EPS, norm_eps=NORM_EPS,
                                           per_tensor=per_tensor, act_bits=4)
    Xd = X.to(dev())
    xq, beta, rowsum, _ = bl.quant_act(Xd, inv_rms=to_dev(r_r), per_tensor=per_tensor,
                                       act_bits=4)
    torch.cuda.synchronize()
    if per_tensor:
        np.testing.assert_allclose(beta.cpu().numpy(), b_r, rtol=2e-6)
        if not np.array_equal(beta.cpu().numpy(), b_r):
            return
    np.testing.assert_array_equal(xq.cpu().numpy(), xq_r)
    np.testing.assert_array_equal(beta.cpu().numpy(), b_r)
    np.testing.assert_array_equal(rowsum.cpu().numpy(), s_r)
    assert xq.abs().max().item() <= 7


# ------------------------------------------------------------- product ---

W1_SHAPES = [(16, 256), (48, 512), (272, 768), (512, 2560), (6912, 2560), (32, 11008),
             (144, 32768)]


@pytest.mark.parametrize("act_bits", [4, 8])
@pytest.mark.parametrize("d_out,d_in", W1_SHAPES)
@pytest.mark.parametrize("T", [1, 3, 8, 9, 16])
def test_forward_w1_matches_oracle(d_out, d_in, T, act_bits):
    W, X = draw(Problem("f1", d_in, d_out, T, 0.02, 0.01, 50.0, 5))
    wq, g, w = binary_weights(W)
    xq, beta, rowsum, _ = oracle.quant_act(bf16_bits(X), eps=EPS, norm_eps=NORM_EPS,
                                           act_bits=act_bits)
    y, acc = bl.forward(w, to_dev(xq), to_dev(beta), to_dev(rowsum), want_acc=True,
                        act_bits=act_bits)
    acc_ref = oracle.int_matmul(wq, xq)
    np.testing.assert_array_equal(acc.cpu().numpy(), acc_ref)
    check_y(y, acc_ref, g, beta, False, act_bits)


def test_forward_w1_two_row_tiles_and_bf16():
    for d_out, d_in, T in ((18960, 256, 1), (18960, 512, 12)):
        W, X = draw(Problem("f1w", d_in, d_out, T, 0.02, 0.01, 50.0, 6))
        wq, g, w = binary_weights(W)
        xq, beta, rowsum, _ = oracle.quant_act(bf16_bits(X), act_bits=4)
        y, acc = bl.forward(w, to_dev(xq), to_dev(beta), to_dev(rowsum), want_acc=True,
                            act_bits=4, out_dtype=torch.bfloat16)
        acc_ref = oracle.int_matmul(wq, xq)
        np.testing.assert_array_equal(acc.cpu().numpy(), acc_ref)
        check_y(y, acc_ref, g, beta, True, 4)


@pytest.mark.parametrize("T", [1, 8])
def test_forward_w1_large_gemv_sampled(T):
    """8192 -> 28672 (the large decode GEMV workload) with 4-bit codes: every
    output of 256 sampled rows against the oracle."""
    p = ALL["large_gemv_8192x28672_t1"].problems[0]
    W, X = draw(Problem(p.name, p.d_in, p.d_out, T, p.sigma, p.outlier_frac, p.outlier_factor,
                        p.seed))
    wq, g, w = binary_weights(W)
    xq, beta, rowsum, _ = oracle.quant_act(bf16_bits(X), act_bits=4)
    _, acc = bl.forward(w, to_dev(xq), to_dev(beta), to_dev(rowsum), want_acc=True, act_bits=4)
    rows = np.random.default_rng(4).choice(p.d_out, 256, replace=False)
    np.testing.assert_array_equal(acc.cpu().numpy()[:, rows], oracle.int_matmul(wq[rows], xq))


def test_forward_w1_extreme_codes():
    d_out, d_in = 32, 2560
    for wv in (1, -1):
        wq = np.full((d_out, d_in), wv, np.int8)
        w = bl.PackedBinary(to_dev(oracle.pack_w1(wq).view(np.int32)),
                            torch.tensor([1.0], device=dev()), d_out, d_in)
        for xv in (7, -7, 127, -127):
            xq = np.full((2, d_in), xv, np.int8)
            rowsum = xq.astype(np.int64).sum(axis=1).astype(np.int32)
            _, acc = bl.forward(w, to_dev(xq), to_dev(np.ones(2, np.float32)), to_dev(rowsum),
                                want_acc=True, act_bits=8)
            assert (acc.cpu().numpy() == wv * xv * d_in).all()


def test_w1_rejects_prefill_sizes():
    W = draw(Problem("r", 512, 64, 1, 0.02, 0.0, 1.0, 1))[0]
    _, _, w = binary_weights(W)
    with pytest.raises(bl.BitLinearError):
        bl.linear(w, torch.zeros(17, 512, dtype=torch.bfloat16, device=dev()), act_bits=4)


# -------------------------------------------------------------- linear ---

LINEAR_CASES = [
    # (d_out, d_in, T, rmsnorm, gain, static, per_tensor, act_bits, out_dtype)
    (6912, 2560, 1, True, False, True, False, 4, torch.bfloat16),    # fused W1A4 decode
    (272, 1024, 8, True, False, False, False, 4, torch.float32),
    (512, 4096, 4, True, True, True, False, 4, torch.float32),      # gain
    (512, 4096, 3, False, False, False, False, 8, torch.float32),   # W1A8, no RMSNorm
    (4096, 11008, 1, True, False, True, False, 4, torch.bfloat16),  # half-padded last tile
    (512, 4096, 9, True, False, False, False, 4, torch.float32),    # quantiser + product
    (4096, 4096, 16, True, True, True, False, 4, torch.bfloat16),
    (512, 2560, 5, True, False, False, True, 4, torch.float32),     # per-tensor absmax
]


@pytest.mark.parametrize("d_out,d_in,T,rmsnorm,use_gain,static,per_tensor,act_bits,out_dtype",
                         LINEAR_CASES)
def test_linear_w1_matches_quantiser_forward_and_oracle(d_out, d_in, T, rmsnorm, use_gain,
                                                        static, per_tensor, act_bits, out_dtype):
    W, X = draw(Problem("l1", d_in, d_out, T, 0.02, 0.01, 50.0, 17))
    gain = None
    if use_gain:
        gen = torch.Generator().manual_seed(2)
        gain = (torch.rand(d_in, generator=gen) * 2).numpy().astype(np.float32)
    wq, g, w = binary_weights(W)
    Xd = X.to(dev())
    gd = None if gain is None else to_dev(gain)
    scratch = (torch.empty((T, d_in), dtype=torch.int8, device=dev()),
               torch.empty(T, dtype=torch.float32, device=dev()),
               torch.empty(T, dtype=torch.int32, device=dev()))
    y = bl.linear(w, Xd, gain=gd, rmsnorm=rmsnorm, out_dtype=out_dtype, scratch=scratch,
                  static_weights=static, per_tensor=per_tensor, act_bits=act_bits)
    xq2, b2, s2, _ = bl.quant_act(Xd, gain=gd, rmsnorm=rmsnorm, per_tensor=per_tensor,
                                  act_bits=act_bits)
    torch.cuda.synchronize()
    assert torch.equal(scratch[0], xq2) and torch.equal(scratch[1], b2)
    assert torch.equal(scratch[2], s2)
    y2 = bl.forward(w, xq2, b2, s2, out_dtype=out_dtype, act_bits=act_bits)
    assert torch.equal(y, y2)
    xq_r, beta_r, _, _ = oracle.quant_act(bf16_bits(X), gain=gain, rmsnorm=rmsnorm, eps=EPS,
                                          norm_eps=NORM_EPS, per_tensor=per_tensor,
                                          act_bits=act_bits)
    if np.array_equal(xq2.cpu().numpy(), xq_r):
        check_y(y, oracle.int_matmul(wq, xq_r), g, beta_r, out_dtype == torch.bfloat16,
                act_bits)


def test_linear_plan_w1a4():
    W, X = draw(Problem("lp1", 2560, 6912, 1, 0.02, 0.01, 50.0, 12))
    w = bl.pack_weights_w1(W.to(dev()))
    Xd = X.to(dev())
    ref = bl.linear(w, Xd, out_dtype=torch.bfloat16, act_bits=4)
    plan = bl.LinearPlan(w, 1, out_dtype=torch.bfloat16, static_weights=True, act_bits=4)
    got = plan(Xd)
    torch.cuda.synchronize()
    assert torch.equal(got, ref)
