"""Parity of the decode product's balanced split with the oracle.

With a split workspace the decode kernel cuts the (16-row tiles, k-tile)
units into equal shares, one per resident CTA, and CTAs that share a row tile
add exact int32 partial sums in the workspace ("BitNet b1.58: Mathematical
Foundations ...", section 2: the accumulation X~ W~^T is exact in int32, so
the result cannot depend on how the sum is cut).  Bars: int32 accumulators,
codes, absmax and row sums bit-exact against the oracle; outputs within the
output bar of the other parity tests, and bit-equal to the same call without
a workspace; the workspace zero again after every call; every output and the
workspace itself between guard zones.

BITLINEAR_SPLIT_ALWAYS makes every call with a workspace split, so small
shapes cut row tiles across many CTAs (shares shorter than one row tile);
the automatic rule is exercised at the 8192 -> 28672 decode, the shape it is
for.
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
    yield
    bl.set_decode_split(bl.SPLIT_AUTO)
    assert bl.device_error(clear=True) == bl.OK


@pytest.fixture()
def always():
    bl.set_decode_split(bl.SPLIT_ALWAYS)
    yield
    bl.set_decode_split(bl.SPLIT_AUTO)


def dev():
    return torch.device("cuda:0")


def to_dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(dev())


class Workspace:
    """A zero-filled split workspace between guard zones."""

    def __init__(self, d_out, T):
        n = bl.decode_workspace_bytes(d_out, T)
        assert n > 0
        self.g = Guarded((n,), torch.uint8)
        self.g.t.zero_()
        self.t = self.g.t

    def check_clean(self):
        check_all(self.g)
        assert int(torch.count_nonzero(self.t).item()) == 0, "workspace not left zero"


def check_y(y_gpu, acc_ref, gamma, beta, out_bf16):
    y_ref = oracle.rescale(acc_ref, gamma, beta)
    scale = beta.astype(np.float64)[:, None] * gamma / 127.0
    yg = y_gpu.float().cpu().numpy().astype(np.float64)
    tol = (1e-2 if out_bf16 else 1e-5) * np.maximum(np.abs(y_ref), scale)
    bad = np.abs(yg - y_ref) > tol
    assert not bad.any(), "y mismatch at %s" % (np.argwhere(bad)[:5],)


def case(d_out, d_in, T, seed):
    W, X = draw(Problem("sp", d_in, d_out, T, 0.02, 0.01, 50.0, seed))
    Wn = W.numpy()
    g = oracle.absmean_gamma(Wn)
    wq = oracle.ternarize(Wn, g, EPS)
    xq, beta, rowsum, rms = oracle.quant_act(bf16_bits(X), eps=EPS, norm_eps=NORM_EPS)
    w = bl.PackedTernary(to_dev(oracle.pack(wq).view(np.int32)), torch.tensor([g], device=dev()),
                         d_out, d_in)
    return dict(W=W, X=X, wq=wq, g=g, xq=xq, beta=beta, rowsum=rowsum, rms=rms, w=w,
                acc=oracle.int_matmul(wq, xq))


SPLIT_SHAPES = [
    # (d_out, d_in, T)
    (16, 256, 1),          # one unit: nothing to share
    (272, 768, 1),
    (272, 768, 5),
    (272, 768, 9),         # two token groups
    (272, 768, 16),
    (512, 4096, 1),
    (512, 4096, 8),
    (6912, 2560, 1),
    (6912, 2560, 16),
    (4096, 11008, 1),      # 43 k-tiles per row
    (18960, 512, 1),       # 1185 row tiles: two per unit, the last one alone
    (18960, 512, 12),
]


@pytest.mark.parametrize("d_out,d_in,T", SPLIT_SHAPES)
def test_split_forward_matches_oracle(d_out, d_in, T, always):
    """The product with every unit share split: bit-exact accumulators, run
    after run on one workspace, which stays zero."""
    c = case(d_out, d_in, T, 41)
    ws = Workspace(d_out, T)
    xq, beta, rs = to_dev(c["xq"]), to_dev(c["beta"]), to_dev(c["rowsum"])
    for out_dtype in (torch.float32, torch.bfloat16, torch.float32):
        gy, ga = Guarded((T, d_out), out_dtype), Guarded((T, d_out), torch.int32)
        y, acc = bl.forward(c["w"], xq, beta, rs, out=gy.t, acc=ga.t, workspace=ws.t)
        check_all(gy, ga)
        ws.check_clean()
        np.testing.assert_array_equal(acc.cpu().numpy(), c["acc"])
        check_y(y, c["acc"], c["g"], c["beta"], out_dtype == torch.bfloat16)
        y0 = bl.forward(c["w"], xq, beta, rs, out_dtype=out_dtype)
        assert torch.equal(y, y0)


FUSED_SPLIT = [
    # (d_out, d_in, T, static)
    (272, 1024, 1, False),
    (272, 1024, 8, True),
    (6912, 2560, 1, True),
    (4096, 4096, 3, False),
    (18960, 256, 1, True),
    (512, 4096, 12, False),   # T > 8: quantiser, then the split product
]


@pytest.mark.parametrize("d_out,d_in,T,static", FUSED_SPLIT)
def test_split_linear_matches_oracle(d_out, d_in, T, static, always):
    """bitlinear_linear (fused quantiser + product for T <= 8) with the split:
    intermediates and accumulators through the rescale as the oracle, given
    its reciprocal RMS; the workspace stays zero."""
    c = case(d_out, d_in, T, 43)
    ws = Workspace(d_out, T)
    Xd = c["X"].to(dev())
    for _ in range(2):
        sc = (Guarded((T, d_in), torch.int8), Guarded((T,), torch.float32),
              Guarded((T,), torch.int32))
        gy = Guarded((T, d_out), torch.float32)
        y = bl.linear(c["w"], Xd, out=gy.t, scratch=tuple(s.t for s in sc),
                      static_weights=static, inv_rms=to_dev(c["rms"]), workspace=ws.t)
        check_all(gy, *sc)
        ws.check_clean()
        np.testing.assert_array_equal(sc[0].t.cpu().numpy(), c["xq"])
        np.testing.assert_array_equal(sc[1].t.cpu().numpy(), c["beta"])
        np.testing.assert_array_equal(sc[2].t.cpu().numpy(), c["rowsum"])
        check_y(y, c["acc"], c["g"], c["beta"], False)
        y0 = bl.linear(c["w"], Xd, static_weights=static, inv_rms=to_dev(c["rms"]))
        assert torch.equal(y, y0)


@pytest.mark.parametrize("fmt", ["base3", "w1"])
@pytest.mark.parametrize("T", [1, 8, 16])
def test_split_other_formats_equal_unsplit(fmt, T, always):
    """Base-3 and 1-bit weights through the same split: accumulators equal
    to the unsplit product's (which the format tests pin to the oracle) and,
    for base 3, to the oracle's."""
    d_out, d_in = 400, 1280
    c = case(d_out, d_in, T, 47)
    if fmt == "base3":
        w = bl.PackedTernaryBase3(to_dev(oracle.pack_base3(c["wq"])), c["w"].gamma, d_out, d_in)
        xq, beta, rs = to_dev(c["xq"]), to_dev(c["beta"]), to_dev(c["rowsum"])
        bits = 8
    else:
        w = bl.pack_weights_w1(c["W"].to(dev()))
        bits = 4
        xq, beta, rs, _ = bl.quant_act(c["X"].to(dev()), act_bits=4)
    ws = Workspace(d_out, T)
    ga = Guarded((T, d_out), torch.int32)
    _, acc = bl.forward(w, xq, beta, rs, acc=ga.t, workspace=ws.t, act_bits=bits)
    check_all(ga)
    ws.check_clean()
    _, acc0 = bl.forward(w, xq, beta, rs, want_acc=True, act_bits=bits)
    assert torch.equal(acc, acc0)
    if fmt == "base3":
        np.testing.assert_array_equal(acc.cpu().numpy(), c["acc"])


def test_split_plan_equals_linear(always):
    """A plan owns its workspace: its runs give the bits of bitlinear_linear."""
    d_out, d_in, T = 2064, 2560, 1
    c = case(d_out, d_in, T, 53)
    plan = bl.LinearPlan(c["w"], T, out_dtype=torch.bfloat16, static_weights=True)
    gen = torch.Generator().manual_seed(3)
    for _ in range(3):
        X = (torch.randn(T, d_in, generator=gen) * 2).to(torch.bfloat16).to(dev())
        got = plan(X).clone()
        ref = bl.linear(c["w"], X, out_dtype=torch.bfloat16, static_weights=True)
        torch.cuda.synchronize()
        assert torch.equal(got, ref)
    del plan


@pytest.mark.parametrize("T", [1, 8])
def test_split_auto_large_decode(T):
    """The automatic rule at 8192 -> 28672 (896 groups of two row tiles on the
    resident CTAs, which do not divide them): the split product's accumulators
    equal the unsplit product's, and on a sample of rows the oracle's."""
    d_out, d_in = 28672, 8192
    p = Problem("sa", d_in, d_out, T, 0.015, 0.001, 1000.0, 7)
    W, X = draw(p)
    gen = np.random.default_rng(5)
    rows = np.sort(gen.choice(d_out, 96, replace=False))
    Wn = W.numpy()
    g = oracle.absmean_gamma(Wn)
    Wd = W.to(dev())
    w = bl.pack_weights(Wd, EPS, gamma=torch.tensor([g], device=dev()))
    del Wd
    xq, beta, rs, rms = oracle.quant_act(bf16_bits(X), eps=EPS, norm_eps=NORM_EPS)
    xqd, bd, rsd = to_dev(xq), to_dev(beta), to_dev(rs)
    ws = Workspace(d_out, T)
    ga = Guarded((T, d_out), torch.int32)
    for _ in range(2):
        _, acc = bl.forward(w, xqd, bd, rsd, acc=ga.t, workspace=ws.t)
        check_all(ga)
        ws.check_clean()
    _, acc0 = bl.forward(w, xqd, bd, rsd, want_acc=True)
    assert torch.equal(acc, acc0)
    wq_rows = oracle.ternarize(Wn[rows], g, EPS)
    np.testing.assert_array_equal(acc.cpu().numpy()[:, rows], oracle.int_matmul(wq_rows, xq))
    # The fused serving call (T = 1) or quantiser + product (T = 8), split.
    gy = Guarded((T, d_out), torch.bfloat16)
    y = bl.linear(w, X.to(dev()), out=gy.t, static_weights=True, inv_rms=to_dev(rms),
                  workspace=ws.t)
    check_all(gy)
    ws.check_clean()
    y0 = bl.linear(w, X.to(dev()), out_dtype=torch.bfloat16, static_weights=True,
                   inv_rms=to_dev(rms))
    assert torch.equal(y, y0)
