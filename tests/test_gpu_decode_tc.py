"""Parity of the tensor-core decode product (tcgen05, codes in tensor memory)
with the CPU oracle.

The same bars as the other parity tests ("BitNet b1.58: Mathematical
Foundations ...", section 2: exact int32 accumulation, then the rescale):
int32 accumulators bit-exact, fp32 outputs within 1e-5 and bf16 within 1e-2
of max(|y|, gamma beta_t / 127), every output between guard zones, the split
workspace zero after every call.  BITLINEAR_DECODE_TCGEN05 forces the kernel;
the shapes cover ragged 128-row blocks, k-tile counts that leave a short last
stage, token counts 1..16 and both split modes.
"""
import numpy as np
import pytest
import torch

import oracle
import ternary_weight_linear_bitlinear_b200 as bl
from guard import Guarded, check_all
from ternary_weight_linear_bitlinear_b200 import build as blbuild
from workloads import Problem, bf16_bits, draw

pytestmark = pytest.mark.gpu
EPS = 1e-5
NORM_EPS = 1e-5


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    blbuild.build()
    bl.lib()
    bl.set_decode_kernel(bl.DECODE_TCGEN05)
    yield
    bl.set_decode_kernel(bl.DECODE_AUTO)
    bl.set_decode_split(bl.SPLIT_AUTO)
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


def case(d_out, d_in, T, seed):
    W, X = draw(Problem("tc", d_in, d_out, T, 0.02, 0.01, 50.0, seed))
    Wn = W.numpy()
    g = oracle.absmean_gamma(Wn)
    wq = oracle.ternarize(Wn, g, EPS)
    xq, beta, rowsum, rms = oracle.quant_act(bf16_bits(X), eps=EPS, norm_eps=NORM_EPS)
    w = bl.PackedTernary(to_dev(oracle.pack(wq).view(np.int32)), torch.tensor([g], device=dev()),
                         d_out, d_in)
    return dict(X=X, wq=wq, g=g, xq=xq, beta=beta, rowsum=rowsum, rms=rms, w=w,
                acc=oracle.int_matmul(wq, xq))


class Workspace:
    def __init__(self, d_out, T):
        self.g = Guarded((bl.decode_workspace_bytes(d_out, T),), torch.uint8)
        self.g.t.zero_()
        self.t = self.g.t

    def check_clean(self):
        check_all(self.g)
        assert int(torch.count_nonzero(self.t).item()) == 0, "workspace not left zero"


TC_SHAPES = [
    # (d_out, d_in, T)
    (16, 256, 1),          # one row tile: a block of 128 rows with 112 empty
    (128, 256, 1),
    (272, 768, 5),         # 2.1 blocks, 3 k-tiles (one stage)
    (512, 4096, 16),
    (512, 4096, 9),
    (6912, 2560, 1),       # 54 blocks, 10 k-tiles: stages of 4, 4 and 2
    (6928, 2560, 3),       # a last block of 16 rows
    (4096, 11008, 8),      # 43 k-tiles
    (18960, 512, 12),
]


@pytest.mark.parametrize("d_out,d_in,T", TC_SHAPES)
@pytest.mark.parametrize("split", ["none", "always"])
def test_tc_forward_matches_oracle(d_out, d_in, T, split):
    c = case(d_out, d_in, T, 61)
    xq, beta, rs = to_dev(c["xq"]), to_dev(c["beta"]), to_dev(c["rowsum"])
    ws = None
    if split == "always":
        bl.set_decode_split(bl.SPLIT_ALWAYS)
        ws = Workspace(d_out, T)
    try:
        for out_dtype in (torch.float32, torch.bfloat16):
            gy, ga = Guarded((T, d_out), out_dtype), Guarded((T, d_out), torch.int32)
            y, acc = bl.forward(c["w"], xq, beta, rs, out=gy.t, acc=ga.t,
                                workspace=None if ws is None else ws.t)
            check_all(gy, ga)
            if ws is not None:
                ws.check_clean()
            np.testing.assert_array_equal(acc.cpu().numpy(), c["acc"])
            check_y(y, c["acc"], c["g"], c["beta"], out_dtype == torch.bfloat16)
    finally:
        bl.set_decode_split(bl.SPLIT_AUTO)


@pytest.mark.parametrize("d_out,d_in,T", [(272, 1024, 1), (6912, 2560, 1), (4096, 4096, 8),
                                          (512, 4096, 16)])
def test_tc_linear_matches_oracle(d_out, d_in, T):
    """bitlinear_linear with the tensor-core product: the quantiser, then the
    product; the oracle's reciprocal RMS supplied."""
    c = case(d_out, d_in, T, 67)
    ws = Workspace(d_out, T)
    sc = (Guarded((T, d_in), torch.int8), Guarded((T,), torch.float32),
          Guarded((T,), torch.int32))
    gy = Guarded((T, d_out), torch.float32)
    y = bl.linear(c["w"], c["X"].to(dev()), out=gy.t, scratch=tuple(s.t for s in sc),
                  static_weights=True, inv_rms=to_dev(c["rms"]), workspace=ws.t)
    check_all(gy, *sc)
    ws.check_clean()
    np.testing.assert_array_equal(sc[0].t.cpu().numpy(), c["xq"])
    check_y(y, c["acc"], c["g"], c["beta"], False)


def test_tc_plan_equals_linear():
    d_out, d_in, T = 2064, 2560, 4
    c = case(d_out, d_in, T, 71)
    plan = bl.LinearPlan(c["w"], T, out_dtype=torch.bfloat16, static_weights=True)
    gen = torch.Generator().manual_seed(5)
    for _ in range(3):
        X = (torch.randn(T, d_in, generator=gen) * 2).to(torch.bfloat16).to(dev())
        got = plan(X).clone()
        ref = bl.linear(c["w"], X, out_dtype=torch.bfloat16, static_weights=True)
        torch.cuda.synchronize()
        assert torch.equal(got, ref)
    del plan


@pytest.mark.parametrize("T", [1, 16])
def test_tc_large_equals_warp_mma(T):
    """8192 -> 28672 (224 blocks on the resident CTAs: split automatically):
    the same accumulators as the warp-MMA kernel, and the oracle's on a sample
    of rows."""
    d_out, d_in = 28672, 8192
    W, X = draw(Problem("tl", d_in, d_out, T, 0.015, 0.001, 1000.0, 3))
    Wn = W.numpy()
    g = oracle.absmean_gamma(Wn)
    Wd = W.to(dev())
    w = bl.pack_weights(Wd, EPS, gamma=torch.tensor([g], device=dev()))
    del Wd
    xq, beta, rs, _ = oracle.quant_act(bf16_bits(X), eps=EPS, norm_eps=NORM_EPS)
    xqd, bd, rsd = to_dev(xq), to_dev(beta), to_dev(rs)
    ws = Workspace(d_out, T)
    ga = Guarded((T, d_out), torch.int32)
    for _ in range(2):
        _, acc = bl.forward(w, xqd, bd, rsd, acc=ga.t, workspace=ws.t)
        check_all(ga)
        ws.check_clean()
    bl.set_decode_kernel(bl.DECODE_WARP_MMA)
    try:
        _, acc0 = bl.forward(w, xqd, bd, rsd, want_acc=True)
    finally:
        bl.set_decode_kernel(bl.DECODE_TCGEN05)
    assert torch.equal(acc, acc0)
    rows = np.sort(np.random.default_rng(9).choice(d_out, 64, replace=False))
    wq_rows = oracle.ternarize(Wn[rows], g, EPS)
    np.testing.assert_array_equal(acc.cpu().numpy()[:, rows], oracle.int_matmul(wq_rows, xq))
