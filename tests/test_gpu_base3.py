"""Parity of the base-3 weight format (five ternary codes per byte) on the GPU
with the oracle: the repacker byte for byte, the decode product's int32
accumulators bit for bit, the rescaled outputs within the output bar.

The format follows "BitNet b1.58: Mathematical Foundations ...", section 4
(Memory Bandwidth and Latency Bounds: five ternary values per 8-bit byte).
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


def check_y(y_gpu, acc_ref, gamma, beta, out_bf16):
    y_ref = oracle.rescale(acc_ref, gamma, beta)
    scale = beta.astype(np.float64)[:, None] * gamma / 127.0
    yg = y_gpu.float().cpu().numpy().astype(np.float64)
    tol = (1e-2 if out_bf16 else 1e-5) * np.maximum(np.abs(y_ref), scale)
    bad = np.abs(yg - y_ref) > tol
    assert not bad.any(), "y mismatch at %s" % (np.argwhere(bad)[:5],)


def weights(d_out, d_in, seed):
    W, _ = draw(Problem("b3", d_in, d_out, 1, 0.02, 0.0, 1.0, seed))
    Wn = W.numpy()
    g = oracle.absmean_gamma(Wn)
    wq = oracle.ternarize(Wn, g, EPS)
    w2 = bl.PackedTernary(to_dev(oracle.pack(wq).view(np.int32)), torch.tensor([g], device=dev()),
                          d_out, d_in)
    w3 = bl.PackedTernaryBase3(to_dev(oracle.pack_base3(wq)), w2.gamma, d_out, d_in)
    return W, wq, g, w2, w3


# --------------------------------------------------------------- repack ---

REPACK_SHAPES = [(16, 256), (48, 512), (272, 768), (6912, 2560), (4096, 4096), (32, 11008),
                 (16, 65536)]


@pytest.mark.parametrize("d_out,d_in", REPACK_SHAPES)
def test_repack_matches_oracle(d_out, d_in):
    _, wq, _, w2, _ = weights(d_out, d_in, 3)
    w3 = bl.repack_base3(w2)
    torch.cuda.synchronize()
    assert w3.packed.numel() == bl.base3_bytes(d_out, d_in) == d_out * oracle.base3_cols(d_in) // 5
    np.testing.assert_array_equal(w3.packed.cpu().numpy(), oracle.pack_base3(wq))


def test_repack_of_gpu_packed_weights():
    """pack_weights then repack_base3 on the device: the bytes of the oracle's
    base-3 pack of the oracle's ternarisation (the oracle's gamma supplied)."""
    W, wq, g, _, _ = weights(272, 1024, 9)
    w2 = bl.pack_weights(W.to(dev()), EPS, gamma=torch.tensor([g], device=dev()))
    w3 = bl.repack_base3(w2)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(w3.packed.cpu().numpy(), oracle.pack_base3(wq))


# -------------------------------------------------------------- product ---

# d_in values cover whole 160-column tiles (2560), a ragged last tile
# (256, 512, 768, 4096, 11008) and several slabs per row (11008, 32768).
B3_SHAPES = [(16, 256), (48, 512), (272, 768), (512, 512), (6912, 2560), (32, 11008),
             (4096, 4096), (144, 32768)]


def product_case(d_out, d_in, T, out_dtype, seed=5):
    W, X = draw(Problem("b3f", d_in, d_out, T, 0.02, 0.01, 50.0, seed))
    Wn = W.numpy()
    g = oracle.absmean_gamma(Wn)
    wq = oracle.ternarize(Wn, g, EPS)
    xq, beta, rowsum, _ = oracle.quant_act(bf16_bits(X), eps=EPS, norm_eps=NORM_EPS)
    w3 = bl.PackedTernaryBase3(to_dev(oracle.pack_base3(wq)), torch.tensor([g], device=dev()),
                               d_out, d_in)
    y, acc = bl.forward(w3, to_dev(xq), to_dev(beta), to_dev(rowsum), out_dtype=out_dtype,
                        want_acc=True)
    acc_ref = oracle.int_matmul(wq, xq)
    np.testing.assert_array_equal(acc.cpu().numpy(), acc_ref)
    check_y(y, acc_ref, g, beta, out_dtype == torch.bfloat16)


@pytest.mark.parametrize("d_out,d_in", B3_SHAPES)
@pytest.mark.parametrize("T", [1, 2, 5, 8, 9, 16])
def test_forward_base3_matches_oracle(d_out, d_in, T):
    product_case(d_out, d_in, T, torch.float32)


@pytest.mark.parametrize("T", [1, 16])
def test_forward_base3_bf16_out(T):
    product_case(512, 4096, T, torch.bfloat16)


def test_forward_base3_two_row_tiles_per_group():
    """1185 row tiles: the kernel takes two per group (and a ragged last)."""
    product_case(18960, 256, 1, torch.float32)
    product_case(18960, 512, 12, torch.float32)


@pytest.mark.parametrize("T", [1, 8])
def test_forward_base3_large_gemv_sampled(T):
    """8192 -> 28672 (the large decode GEMV workload): every output of 256
    sampled rows against the oracle's product on those rows."""
    p = ALL["large_gemv_8192x28672_t1"].problems[0]
    W, X = draw(Problem(p.name, p.d_in, p.d_out, T, p.sigma, p.outlier_frac,
                        p.outlier_factor, p.seed))
    Wn = W.numpy()
    g = oracle.absmean_gamma(Wn)
    wq = oracle.ternarize(Wn, g, EPS)
    xq, beta, rowsum, _ = oracle.quant_act(bf16_bits(X), eps=EPS, norm_eps=NORM_EPS)
    w3 = bl.PackedTernaryBase3(to_dev(oracle.pack_base3(wq)), torch.tensor([g], device=dev()),
                               p.d_out, p.d_in)
    y, acc = bl.forward(w3, to_dev(xq), to_dev(beta), to_dev(rowsum), want_acc=True)
    rows = np.random.default_rng(4).choice(p.d_out, 256, replace=False)
    acc_ref = oracle.int_matmul(wq[rows], xq)
    np.testing.assert_array_equal(acc.cpu().numpy()[:, rows], acc_ref)


def test_forward_base3_equals_two_bit():
    """The two formats give the same outputs bit for bit."""
    _, wq, g, w2, w3 = weights(6912, 2560, 21)
    X = draw(Problem("eq", 2560, 16, 16, 0.02, 0.01, 50.0, 6))[1].to(dev())
    for T in (1, 4, 16):
        Xq, beta, rowsum, _ = bl.quant_act(X[:T])
        y2, a2 = bl.forward(w2, Xq, beta, rowsum, want_acc=True)
        y3, a3 = bl.forward(w3, Xq, beta, rowsum, want_acc=True)
        torch.cuda.synchronize()
        assert torch.equal(a2, a3) and torch.equal(y2, y3)


def test_forward_base3_extreme_codes():
    """All weights +1 against all activations -127 and +127 (the largest
    accumulators), and all weights -1."""
    d_out, d_in = 32, 2560
    for wv in (1, -1):
        wq = np.full((d_out, d_in), wv, np.int8)
        w3 = bl.PackedTernaryBase3(to_dev(oracle.pack_base3(wq)),
                                   torch.tensor([1.0], device=dev()), d_out, d_in)
        for xv in (127, -127):
            xq = np.full((3, d_in), xv, np.int8)
            beta = np.ones(3, np.float32)
            rowsum = xq.astype(np.int64).sum(axis=1).astype(np.int32)
            _, acc = bl.forward(w3, to_dev(xq), to_dev(beta), to_dev(rowsum), want_acc=True)
            assert (acc.cpu().numpy() == wv * xv * d_in).all()


def test_base3_rejects_prefill_sizes():
    _, _, _, _, w3 = weights(64, 512, 1)
    X = torch.zeros(17, 512, dtype=torch.bfloat16, device=dev())
    with pytest.raises(bl.BitLinearError):
        bl.linear(w3, X)


# --------------------------------------------------------------- linear ---

LINEAR_CASES = [
    # (d_out, d_in, T, rmsnorm, gain, static, per_tensor, out_dtype)
    (6912, 2560, 1, True, False, True, False, torch.bfloat16),   # fused decode forward
    (272, 1024, 8, True, False, False, False, torch.float32),
    (512, 4096, 4, True, True, True, False, torch.float32),      # gain
    (512, 4096, 3, False, False, False, False, torch.float32),   # no RMSNorm
    (4096, 11008, 1, True, False, True, False, torch.bfloat16),  # ragged last tile
    (512, 4096, 9, True, False, False, False, torch.float32),    # quantiser + product
    (4096, 4096, 16, True, True, True, False, torch.bfloat16),
    (512, 2560, 5, True, False, False, True, torch.float32),     # per-tensor absmax
]


@pytest.mark.parametrize("d_out,d_in,T,rmsnorm,use_gain,static,per_tensor,out_dtype",
                         LINEAR_CASES)
def test_linear_base3_matches_two_bit_and_oracle(d_out, d_in, T, rmsnorm, use_gain, static,
                                                 per_tensor, out_dtype):
    W, X = draw(Problem("b3l", d_in, d_out, T, 0.02, 0.01, 50.0, 17))
    gain = None
    if use_gain:
        gen = torch.Generator().manual_seed(2)
        gain = (torch.rand(d_in, generator=gen) * 2).numpy().astype(np.float32)
    Wn = W.numpy()
    g = oracle.absmean_gamma(Wn)
    wq = oracle.ternarize(Wn, g, EPS)
    w2 = bl.PackedTernary(to_dev(oracle.pack(wq).view(np.int32)), torch.tensor([g], device=dev()),
                          d_out, d_in)
    w3 = bl.PackedTernaryBase3(to_dev(oracle.pack_base3(wq)), w2.gamma, d_out, d_in)
    Xd = X.to(dev())
    gd = None if gain is None else to_dev(gain)

    def run(w):
        scratch = (torch.empty((T, d_in), dtype=torch.int8, device=dev()),
                   torch.empty(T, dtype=torch.float32, device=dev()),
                   torch.empty(T, dtype=torch.int32, device=dev()))
        y = bl.linear(w, Xd, gain=gd, rmsnorm=rmsnorm, out_dtype=out_dtype, scratch=scratch,
                      static_weights=static, per_tensor=per_tensor)
        return y, scratch

    y3, s3 = run(w3)
    y2, s2 = run(w2)
    torch.cuda.synchronize()
    for a, b in zip(s3, s2):
        assert torch.equal(a, b)
    assert torch.equal(y3, y2)
    # With the oracle's codes (bit-exact when the reciprocal RMS agrees).
    xq_ref, beta_ref, _, _ = oracle.quant_act(bf16_bits(X), gain=gain, rmsnorm=rmsnorm, eps=EPS,
                                               norm_eps=NORM_EPS, per_tensor=per_tensor)
    if np.array_equal(s3[0].cpu().numpy(), xq_ref):
        check_y(y3, oracle.int_matmul(wq, xq_ref), g, beta_ref, out_dtype == torch.bfloat16)


def test_linear_plan_base3():
    W, X = draw(Problem("lp3", 2560, 6912, 1, 0.02, 0.01, 50.0, 12))
    w2 = bl.pack_weights(W.to(dev()), EPS)
    w3 = bl.repack_base3(w2)
    Xd = X.to(dev())
    ref = bl.linear(w2, Xd, out_dtype=torch.bfloat16)
    plan = bl.LinearPlan(w3, 1, out_dtype=torch.bfloat16, static_weights=True)
    got = plan(Xd)
    torch.cuda.synchronize()
    assert torch.equal(got, ref)
