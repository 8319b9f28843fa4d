"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Bars: packed codes, activation codes, row sums and int32 accumulators
bit-exact; gamma and the reciprocal RMS within 1e-6 relative; fp32 outputs within
1e-5 * max(|y|, scale_t) and bf16 outputs within 1e-2 * max(|y|, scale_t),
where scale_t = gamma beta_t / 127 is one integer step of the output (the
floor keeps a relative bound meaningful at acc = 0).

Inputs only flow oracle -> GPU: where integer codes are compared, the GPU is
handed the oracle's gamma / reciprocal RMS (the GPU's own values are checked separately
against the oracle's to 1e-6), so a last-bit difference in a reduction can
not flip a code and nothing computed on the GPU enters the oracle.  Where the
GPU's own gamma or r is used as well, its results are compared with the
supplied-value results: equal when the values agree bit for bit, otherwise
every differing code must be one step away (a rounding-boundary flip) and the
number of such codes is recorded.

Every output buffer sits between guard zones (tests/guard.py) that are
checked after the call: the bounds evidence in place of a memory checker.
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
    torch.cuda.init()
    yield
    assert bl.device_error(clear=True) == bl.OK


def dev():
    return torch.device("cuda:0")


def u32(t):
    return t.cpu().numpy().view(np.uint32)


def to_dev(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a))
    return t.to(dev()) if dtype is None else t.to(dev(), dtype)


def oracle_side(W, X, rmsnorm=True, gain=None):
    """Everything the oracle computes for (W, X), from W and X alone."""
    Wn = W.numpy()
    g = oracle.absmean_gamma(Wn)
    wq = oracle.ternarize(Wn, g, EPS)
    xb = bf16_bits(X)
    xq, beta, rowsum, rms = oracle.quant_act(xb, gain=gain, rmsnorm=rmsnorm, eps=EPS,
                                             norm_eps=NORM_EPS)
    return dict(gamma=g, wq=wq, xq=xq, beta=beta, rowsum=rowsum, inv_rms=rms, xb=xb)


def code_fields(words):
    """The sixteen 2-bit fields of each packed word (layout-independent)."""
    w = np.asarray(words, dtype=np.uint32)
    return (w[..., None] >> (2 * np.arange(16, dtype=np.uint32))) & 3


def assert_boundary_flips(got, expect, what, record=None, max_frac=1e-3):
    """got and expect are integer codes computed from scales that differ only
    in the last bit: every difference must be a single step (a value on a
    rounding boundary) and such values must be rare.  Records the count."""
    d = np.abs(np.asarray(got, dtype=np.int64) - np.asarray(expect, dtype=np.int64))
    n = int((d != 0).sum())
    if record is not None:
        record("%s_boundary_flips" % what, n)
    assert d.max(initial=0) <= 1, "%s: a code differs by more than one step" % what
    assert n <= max(1, max_frac * d.size), "%s: %d codes differ" % (what, n)
    return n


def guarded_scratch(T, d_in):
    return (Guarded((T, d_in), torch.int8), Guarded((T,), torch.float32),
            Guarded((T,), torch.int32))


def check_y(y_gpu, acc_ref, gamma, beta, out_bf16, rows=None):
    """Compare GPU outputs with the oracle's float64 rescale."""
    y_ref = oracle.rescale(acc_ref, gamma, beta)
    scale = beta.astype(np.float64)[:, None] * gamma / 127.0
    yg = y_gpu.float().cpu().numpy().astype(np.float64)
    if rows is not None:
        yg = yg[:, rows]
    tol = (1e-2 if out_bf16 else 1e-5) * np.maximum(np.abs(y_ref), scale)
    bad = np.abs(yg - y_ref) > tol
    assert not bad.any(), "y mismatch at %s" % (np.argwhere(bad)[:5],)


# ----------------------------------------------------------------- pack ---

PACK_SHAPES = [(16, 256), (48, 512), (272, 768), (512, 512), (6912, 2560)]


@pytest.mark.parametrize("d_out,d_in", PACK_SHAPES)
def test_pack_matches_oracle(d_out, d_in):
    W = draw(Problem("p", d_in, d_out, 1, 0.02, 0.0, 1.0, 3))[0]
    Wd = W.to(dev())
    own = bl.pack_weights(Wd, EPS)
    g_oracle = oracle.absmean_gamma(W.numpy())
    g_gpu = float(own.gamma.item())
    assert abs(g_gpu - g_oracle) <= 1e-6 * g_oracle
    given = bl.pack_weights(Wd, EPS, gamma=torch.tensor([g_oracle], device=dev()))
    assert float(given.gamma.item()) == g_oracle
    expect = oracle.pack(oracle.ternarize(W.numpy(), g_oracle, EPS))
    np.testing.assert_array_equal(u32(given.packed), expect)
    # The GPU's own gamma: the same words when it equals the oracle's, else
    # only rounding-boundary flips.
    if g_gpu == g_oracle:
        np.testing.assert_array_equal(u32(own.packed), expect)
    else:
        assert_boundary_flips(code_fields(u32(own.packed)), code_fields(expect), "pack")


def test_pack_special_weights():
    # All zero: gamma = 0, every code 0 -> word 0x55555555.
    z = bl.pack_weights(torch.zeros(32, 512, device=dev()), EPS)
    assert z.gamma.item() == 0.0
    assert (u32(z.packed) == 0x55555555).all()
    # Ties of RoundClip: gamma = 1, eps = 0 -> z = W exactly.
    vals = torch.tensor([0.5, -0.5, 1.5, -1.5, 0.49999997, -0.50000006, 7.0, -7.0, 0.0, -0.0,
                         1.0, -1.0, 0.25, -0.75, 0.75, -0.25], dtype=torch.float32)
    W = vals.repeat(16, 16)
    p = bl.pack_weights(W.to(dev()), 0.0, gamma=torch.tensor([1.0], device=dev()))
    expect = oracle.pack(oracle.ternarize(W.numpy(), 1.0, 0.0))
    np.testing.assert_array_equal(u32(p.packed), expect)
    codes = oracle.unpack(u32(p.packed), 16, 256)[0, :16].tolist()
    assert codes == [1, 0, 1, -1, 0, -1, 1, -1, 0, 0, 1, -1, 0, -1, 1, 0]


# ------------------------------------------------------------ quant_act ---

QA_CASES = [
    (4, 512, 0.01, 50.0, True, False),
    (1, 2560, 0.005, 100.0, True, False),
    (16, 11008, 0.005, 100.0, True, False),
    (8, 8192, 0.001, 1000.0, True, False),
    (3, 768, 0.01, 50.0, False, False),
    (5, 1024, 0.01, 50.0, True, True),
    (2048, 4096, 0.0, 1.0, True, False),
    (1, 65536, 0.001, 100.0, True, False),
    # More tokens than the GPU holds quantiser CTAs at once (several waves).
    (2400, 768, 0.01, 50.0, True, True),
    (2411, 256, 0.01, 50.0, False, False),
    (2400, 8448, 0.005, 100.0, True, False),   # 1056 vectors: a short last batch
]


@pytest.mark.parametrize("T,K,frac,factor,rmsnorm,use_gain", QA_CASES)
def test_quant_act_matches_oracle(T, K, frac, factor, rmsnorm, use_gain):
    X = draw(Problem("q", K, 16, T, 0.02, frac, factor, 8))[1]
    gain = None
    if use_gain:
        gen = torch.Generator().manual_seed(1)
        gain = (torch.rand(K, generator=gen) * 2).numpy().astype(np.float32)
    xb = bf16_bits(X)
    q_ref, b_ref, s_ref, r_ref = oracle.quant_act(xb, gain=gain, rmsnorm=rmsnorm, eps=EPS,
                                                  norm_eps=NORM_EPS)
    Xd = X.to(dev())
    gd = None if gain is None else to_dev(gain)
    # The GPU's own reciprocal RMS agrees with the oracle's.
    own = [Guarded((T, K), torch.int8), Guarded((T,), torch.float32),
           Guarded((T,), torch.int32), Guarded((T,), torch.float32)]
    _, _, _, r_gpu = bl.quant_act(Xd, gain=gd, rmsnorm=rmsnorm, eps=EPS, norm_eps=NORM_EPS,
                                  outs=tuple(g.t for g in own))
    np.testing.assert_allclose(r_gpu.cpu().numpy(), r_ref, rtol=1e-6)
    # With the oracle's reciprocal RMS the codes, beta and row sums are bit-exact.
    sup = [Guarded((T, K), torch.int8), Guarded((T,), torch.float32),
           Guarded((T,), torch.int32), Guarded((T,), torch.float32)]
    xq, beta, rowsum, r_used = bl.quant_act(Xd, gain=gd, rmsnorm=rmsnorm, eps=EPS,
                                            norm_eps=NORM_EPS, inv_rms=to_dev(r_ref),
                                            outs=tuple(g.t for g in sup))
    check_all(*own, *sup)
    np.testing.assert_array_equal(xq.cpu().numpy(), q_ref)
    np.testing.assert_array_equal(beta.cpu().numpy(), b_ref)
    np.testing.assert_array_equal(rowsum.cpu().numpy(), s_ref)
    assert xq.cpu().numpy().min() >= -127
    # The codes made with the GPU's own r: equal, or rounding-boundary flips.
    assert_boundary_flips(own[0].t.cpu().numpy(), q_ref, "quant_act")


def test_quant_act_special_tokens():
    K = 512
    x = torch.zeros(4, K)
    x[1] = -3.0
    x[2, 77] = 2.5
    x[3] = torch.linspace(-1, 1, K)
    X = x.to(torch.bfloat16)
    xb = bf16_bits(X)
    q_ref, b_ref, s_ref, r_ref = oracle.quant_act(xb, eps=EPS, norm_eps=NORM_EPS)
    xq, beta, rowsum, _ = bl.quant_act(X.to(dev()), inv_rms=to_dev(r_ref))
    np.testing.assert_array_equal(xq.cpu().numpy(), q_ref)
    np.testing.assert_array_equal(rowsum.cpu().numpy(), s_ref)
    assert beta[0].item() == 0 and not xq[0].any()
    assert (xq[1] == -127).all()


PER_TENSOR_CASES = [
    # (T, K, rmsnorm, gain)
    (1, 512, True, False), (5, 512, True, True), (40, 1024, False, False),
    (300, 4096, True, False), (1100, 256, True, False), (2400, 512, True, True),
]


@pytest.mark.parametrize("T,K,rmsnorm,use_gain", PER_TENSOR_CASES)
def test_quant_act_per_tensor_matches_oracle(T, K, rmsnorm, use_gain):
    """One beta for all tokens: statistics, the max over tokens and the codes."""
    X = draw(Problem("pt", K, 16, T, 0.02, 0.01, 50.0, 21))[1]
    gain = None
    if use_gain:
        gen = torch.Generator().manual_seed(4)
        gain = (torch.rand(K, generator=gen) * 2).numpy().astype(np.float32)
    xb = bf16_bits(X)
    q_ref, b_ref, s_ref, r_ref = oracle.quant_act(xb, gain=gain, rmsnorm=rmsnorm, eps=EPS,
                                                  norm_eps=NORM_EPS, per_tensor=True)
    assert np.all(b_ref == b_ref[0])
    Xd = X.to(dev())
    gd = None if gain is None else to_dev(gain)
    _, _, _, r_gpu = bl.quant_act(Xd, gain=gd, rmsnorm=rmsnorm, per_tensor=True)
    np.testing.assert_allclose(r_gpu.cpu().numpy(), r_ref, rtol=1e-6)
    xq, beta, rowsum, _ = bl.quant_act(Xd, gain=gd, rmsnorm=rmsnorm, eps=EPS, norm_eps=NORM_EPS,
                                       inv_rms=to_dev(r_ref), per_tensor=True)
    np.testing.assert_array_equal(beta.cpu().numpy(), b_ref)
    np.testing.assert_array_equal(xq.cpu().numpy(), q_ref)
    np.testing.assert_array_equal(rowsum.cpu().numpy(), s_ref)


@pytest.mark.parametrize("T", [1, 3, 40])
def test_linear_per_tensor_matches_oracle(T):
    """bitlinear_linear with the per-tensor scope (decode and prefill paths)."""
    d_out, d_in = 272, 1024
    W, X = draw(Problem("lpt", d_in, d_out, T, 0.02, 0.01, 50.0, 23))
    Wn = W.numpy()
    g = oracle.absmean_gamma(Wn)
    wq = oracle.ternarize(Wn, g, EPS)
    xq_ref, b_ref, s_ref, r_ref = oracle.quant_act(bf16_bits(X), eps=EPS, norm_eps=NORM_EPS,
                                                   per_tensor=True)
    w = bl.PackedTernary(to_dev(oracle.pack(wq).view(np.int32)), torch.tensor([g], device=dev()),
                         d_out, d_in)
    # Own reciprocal RMS: one beta for all tokens, within 2e-6 of the oracle's.
    sc = guarded_scratch(T, d_in)
    gy = Guarded((T, d_out), torch.float32)
    bl.linear(w, X.to(dev()), scratch=tuple(g_.t for g_ in sc), per_tensor=True, out=gy.t)
    check_all(gy, *sc)
    b_gpu = sc[1].t.cpu().numpy()
    assert np.all(b_gpu == b_gpu[0])
    np.testing.assert_allclose(b_gpu, b_ref, rtol=2e-6)
    # The oracle's reciprocal RMS supplied: beta, codes and Y against the oracle.
    sc2 = guarded_scratch(T, d_in)
    gy2 = Guarded((T, d_out), torch.float32)
    y2 = bl.linear(w, X.to(dev()), scratch=tuple(g_.t for g_ in sc2), per_tensor=True,
                   out=gy2.t, inv_rms=to_dev(r_ref))
    check_all(gy2, *sc2)
    np.testing.assert_array_equal(sc2[1].t.cpu().numpy(), b_ref)
    np.testing.assert_array_equal(sc2[0].t.cpu().numpy(), xq_ref)
    np.testing.assert_array_equal(sc2[2].t.cpu().numpy(), s_ref)
    check_y(y2, oracle.int_matmul(wq, xq_ref), g, b_ref, False)


# ---------------------------------------------------------------- forward ---

def forward_case(d_out, d_in, T, out_dtype, seed=5, frac=0.01, factor=50.0):
    W, X = draw(Problem("f", d_in, d_out, T, 0.02, frac, factor, seed))
    o = oracle_side(W, X)
    packed = oracle.pack(o["wq"])
    w = bl.PackedTernary(to_dev(packed.view(np.int32)),
                         torch.tensor([o["gamma"]], device=dev()), d_out, d_in)
    gy, ga = Guarded((T, d_out), out_dtype), Guarded((T, d_out), torch.int32)
    y, acc = bl.forward(w, to_dev(o["xq"]), to_dev(o["beta"]), to_dev(o["rowsum"]),
                        out=gy.t, acc=ga.t)
    check_all(gy, ga)
    acc_ref = oracle.int_matmul(o["wq"], o["xq"])
    np.testing.assert_array_equal(acc.cpu().numpy(), acc_ref)
    check_y(y, acc_ref, o["gamma"], o["beta"], out_dtype == torch.bfloat16)
    return o, w, y


GEMV_SHAPES = [(16, 256), (48, 512), (272, 768), (512, 512), (6912, 2560), (32, 11008)]


@pytest.mark.parametrize("d_out,d_in", GEMV_SHAPES)
@pytest.mark.parametrize("T", [1, 2, 3, 7, 8, 9, 15, 16])
def test_gemv_matches_oracle(d_out, d_in, T):
    forward_case(d_out, d_in, T, torch.float32)


@pytest.mark.parametrize("T", [1, 4, 16])
def test_gemv_bf16_out(T):
    forward_case(512, 512, T, torch.bfloat16)


# 16 and 48 rows: the pair tile's first CTA is itself mostly past the last
# row; 144 and 272: the second CTA's rows are partly or wholly past it.
GEMM_SHAPES = [(16, 256), (48, 768), (128, 256), (144, 512), (272, 768), (512, 512), (384, 2560)]


@pytest.mark.parametrize("d_out,d_in", GEMM_SHAPES)
@pytest.mark.parametrize("T", [17, 100, 256, 300, 600])
def test_gemm_matches_oracle(d_out, d_in, T):
    forward_case(d_out, d_in, T, torch.float32)


@pytest.mark.parametrize("T", [33, 513])
def test_gemm_bf16_out(T):
    forward_case(256, 1024, T, torch.bfloat16)


# Many tiles per CTA pair (the persistent tile loop and both accumulators in
# turn), ragged rows and tokens in the last pair tile.
LARGE_GEMM_CASES = [
    (4096, 512, 1201, torch.float32),    # ragged tokens in the last tile
    (4112, 256, 1100, torch.bfloat16),   # 4112 rows: the last row tile holds 16
    (9472, 256, 512, torch.float32),
    (8192, 256, 1800, torch.float32),    # 256 pair tiles: up to four per CTA pair
]


@pytest.mark.parametrize("d_out,d_in,T,out_dtype", LARGE_GEMM_CASES)
def test_gemm_many_tiles_matches_oracle(d_out, d_in, T, out_dtype):
    forward_case(d_out, d_in, T, out_dtype)


# Without acc_out the prefill GEMM's epilogue stages each 32 x 32 chunk in
# shared memory and writes it with a tensor-map store (clipped at T and
# d_out); with acc_out it writes both outputs directly.
STAGED_CASES = [
    (16, 256, 17, torch.float32),        # one 16-row tile; 17 tokens
    (48, 768, 100, torch.bfloat16),
    (144, 512, 300, torch.float32),      # a chunk straddling d_out (144 = 4.5 x 32)
    (272, 768, 600, torch.bfloat16),
    (4112, 256, 1100, torch.bfloat16),   # last row tile of 16 rows
    (4096, 512, 1201, torch.float32),
    (8192, 256, 1800, torch.float32),    # up to four pair tiles per pair
]


@pytest.mark.parametrize("d_out,d_in,T,out_dtype", STAGED_CASES)
def test_gemm_staged_store_matches_oracle(d_out, d_in, T, out_dtype):
    W, X = draw(Problem("gs", d_in, d_out, T, 0.02, 0.01, 50.0, 7))
    o = oracle_side(W, X)
    w = bl.PackedTernary(to_dev(oracle.pack(o["wq"]).view(np.int32)),
                         torch.tensor([o["gamma"]], device=dev()), d_out, d_in)
    xq, beta, rs = to_dev(o["xq"]), to_dev(o["beta"]), to_dev(o["rowsum"])
    gy = Guarded((T, d_out), out_dtype)
    y = bl.forward(w, xq, beta, rs, out=gy.t)
    check_all(gy)
    acc_ref = oracle.int_matmul(o["wq"], o["xq"])
    check_y(y, acc_ref, o["gamma"], o["beta"], out_dtype == torch.bfloat16)
    y2, acc = bl.forward(w, xq, beta, rs, out_dtype=out_dtype, want_acc=True)
    assert torch.equal(y, y2)
    np.testing.assert_array_equal(acc.cpu().numpy(), acc_ref)


def test_forward_zero_inputs():
    for T in (1, 40):
        d_out, d_in = 64, 512
        w = bl.pack_weights(torch.zeros(d_out, d_in, device=dev()), EPS)
        X = torch.randn(T, d_in).to(torch.bfloat16).to(dev())
        y = bl.linear(w, X)
        assert not y.any()
        W = torch.randn(d_out, d_in, device=dev()) * 0.02
        w = bl.pack_weights(W, EPS)
        y = bl.linear(w, torch.zeros(T, d_in, dtype=torch.bfloat16, device=dev()))
        assert not y.any()


def test_forward_empty_batch():
    w = bl.pack_weights(torch.randn(64, 512, device=dev()), EPS)
    Xq = torch.empty(0, 512, dtype=torch.int8, device=dev())
    e = torch.empty(0, device=dev())
    y = bl.forward(w, Xq, e, e.to(torch.int32))
    assert y.shape == (0, 64)


def test_forward_max_d_in():
    forward_case(16, 65536, 1, torch.float32, frac=0.001, factor=100.0)
    forward_case(16, 65536, 20, torch.float32, frac=0.001, factor=100.0)


def test_linear_equals_separate_calls_and_oracle():
    d_out, d_in = 272, 1024
    for T in (1, 5, 16, 17, 300):
        W, X = draw(Problem("l", d_in, d_out, T, 0.02, 0.01, 50.0, 11))
        Wd, Xd = W.to(dev()), X.to(dev())
        w = bl.pack_weights(Wd, EPS)
        y1 = bl.linear(w, Xd)
        xq, beta, rowsum, _ = bl.quant_act(Xd)
        y2 = bl.forward(w, xq, beta, rowsum)
        torch.cuda.synchronize()
        assert torch.equal(y1, y2)
        # End to end against the oracle computed from W and X alone: the
        # oracle's gamma and reciprocal RMS supplied.
        o = oracle_side(W, X)
        wo = bl.pack_weights(Wd, EPS, gamma=torch.tensor([o["gamma"]], device=dev()))
        y3 = bl.linear(wo, Xd, inv_rms=to_dev(o["inv_rms"]))
        acc_ref = oracle.int_matmul(o["wq"], o["xq"])
        check_y(y3, acc_ref, o["gamma"], o["beta"], False)


FUSED_CASES = [
    # (d_out, d_in, T, rmsnorm, gain, static, out_dtype)
    (272, 1024, 1, True, False, False, torch.float32),
    (272, 1024, 8, True, False, True, torch.float32),
    (6912, 2560, 1, True, False, True, torch.bfloat16),
    (144, 32768, 1, True, False, False, torch.float32),     # largest fused T * d_in
    (512, 4096, 8, True, True, False, torch.float32),       # gain
    (512, 4096, 3, False, False, True, torch.float32),      # no RMSNorm
    (512, 4096, 9, True, False, False, torch.float32),      # T > 8: two kernels
    (18960, 256, 1, True, False, True, torch.float32),      # 1185 row tiles: 2 per CTA, ragged
    (18960, 256, 12, True, False, False, torch.float32),
    (18960, 512, 5, True, True, True, torch.bfloat16),
    (4096, 4096, 1, True, False, True, torch.bfloat16),     # attention projection, one token
    (6928, 2560, 2, True, False, False, torch.float32),     # 433 row tiles
    (8000, 4096, 4, True, True, True, torch.bfloat16),      # gain, bf16 out
    (4752, 8192, 1, False, False, False, torch.float32),    # no RMSNorm, several slabs
    (4096, 11008, 1, True, False, True, torch.bfloat16),    # down projection, 43 k-blocks
]


@pytest.mark.parametrize("d_out,d_in,T,rmsnorm,use_gain,static,out_dtype", FUSED_CASES)
def test_linear_paths_match_oracle(d_out, d_in, T, rmsnorm, use_gain, static, out_dtype,
                                   record_property):
    """bitlinear_linear (fused one-kernel path for small T*d_in, otherwise
    quantiser + product) against the oracle (its reciprocal RMS supplied, so
    unconditionally); with its own reciprocal RMS, its intermediates against
    the stand-alone quantiser and its output bit-equal to the two separate
    calls."""
    W, X = draw(Problem("fz", d_in, d_out, T, 0.02, 0.01, 50.0, 17))
    gain = None
    if use_gain:
        gen = torch.Generator().manual_seed(2)
        gain = (torch.rand(d_in, generator=gen) * 2).numpy().astype(np.float32)
    Wn = W.numpy()
    g = oracle.absmean_gamma(Wn)
    wq = oracle.ternarize(Wn, g, EPS)
    xq_ref, beta_ref, rs_ref, rms_ref = oracle.quant_act(bf16_bits(X), gain=gain, rmsnorm=rmsnorm,
                                                         eps=EPS, norm_eps=NORM_EPS)
    w = bl.PackedTernary(to_dev(oracle.pack(wq).view(np.int32)), torch.tensor([g], device=dev()),
                         d_out, d_in)
    Xd = X.to(dev())
    gd = None if gain is None else to_dev(gain)
    acc_ref = oracle.int_matmul(wq, xq_ref)
    # The oracle's reciprocal RMS supplied: intermediates bit-exact, Y within
    # the bar, every time.
    sc = guarded_scratch(T, d_in)
    gy = Guarded((T, d_out), out_dtype)
    ys = bl.linear(w, Xd, gain=gd, rmsnorm=rmsnorm, out_dtype=out_dtype, out=gy.t,
                   scratch=tuple(g_.t for g_ in sc), static_weights=static,
                   inv_rms=to_dev(rms_ref))
    check_all(gy, *sc)
    np.testing.assert_array_equal(sc[0].t.cpu().numpy(), xq_ref)
    np.testing.assert_array_equal(sc[1].t.cpu().numpy(), beta_ref)
    np.testing.assert_array_equal(sc[2].t.cpu().numpy(), rs_ref)
    check_y(ys, acc_ref, g, beta_ref, out_dtype == torch.bfloat16)
    # Its own reciprocal RMS (the serving configuration): the same bits as
    # the stand-alone quantiser followed by the product.
    sc = guarded_scratch(T, d_in)
    gy = Guarded((T, d_out), out_dtype)
    y = bl.linear(w, Xd, gain=gd, rmsnorm=rmsnorm, out_dtype=out_dtype, out=gy.t,
                  scratch=tuple(g_.t for g_ in sc), static_weights=static)
    check_all(gy, *sc)
    xq2, b2, s2, r2 = bl.quant_act(Xd, gain=gd, rmsnorm=rmsnorm)
    torch.cuda.synchronize()
    assert torch.equal(sc[0].t, xq2) and torch.equal(sc[1].t, b2)
    assert torch.equal(sc[2].t, s2)
    y2 = bl.forward(w, xq2, b2, s2, out_dtype=out_dtype)
    assert torch.equal(y, y2)
    np.testing.assert_allclose(r2.cpu().numpy(), rms_ref, rtol=1e-6)
    if np.array_equal(r2.cpu().numpy(), rms_ref):
        assert torch.equal(y, ys)
    else:
        assert_boundary_flips(xq2.cpu().numpy(), xq_ref, "linear", record_property)


# ------------------------------------------- failure detection (bounded) ---

def test_bounded_wait_reports_timeout():
    assert bl.device_error(clear=True) == bl.OK
    bl.wait_probe(2_000_000)           # 2 ms on a barrier nothing arrives on
    assert bl.device_error(clear=True) == bl.ERR_TIMEOUT
    assert bl.device_error(clear=True) == bl.OK
    # The same report through the scope table's name, which also clears.
    bl.wait_probe(2_000_000)
    assert bl.get_last_device_error() == bl.ERR_TIMEOUT
    assert bl.get_last_device_error() == bl.OK
    # The context is still usable afterwards.
    forward_case(48, 512, 3, torch.float32)
    forward_case(144, 512, 40, torch.float32)


def test_linear_plan_matches_linear():
    """The bound-argument call path gives the same bits as bl.linear."""
    W, X = draw(Problem("lp", 2560, 272, 1, 0.02, 0.01, 50.0, 12))
    w = bl.pack_weights(W.to(dev()), EPS)
    Xd = X.to(dev())
    ref = bl.linear(w, Xd, out_dtype=torch.bfloat16)
    plan = bl.LinearPlan(w, 1, out_dtype=torch.bfloat16)
    X2 = torch.empty_like(Xd)
    X2.copy_(Xd)
    got = plan(X2)
    torch.cuda.synchronize()
    assert torch.equal(got, ref)
    with pytest.raises(TypeError):
        plan(Xd.float())


PLAN_CASES = [
    # (d_out, d_in, T, flags)   the path each bound call takes
    (6912, 2560, 1, bl.RMSNORM | bl.STATIC_WEIGHTS),     # fused quantiser + GEMV
    (272, 4096, 12, bl.RMSNORM),                           # quantiser, then GEMV
    (512, 1024, 300, bl.RMSNORM | bl.STATIC_WEIGHTS),     # quantiser, then prefill GEMM
    (272, 512, 2400, bl.RMSNORM),                          # several quantiser waves, then GEMM
    (272, 1024, 5, bl.RMSNORM | bl.PER_TENSOR_ABSMAX),     # run as bitlinear_linear
    (144, 512, 3, 0),                                      # no RMSNorm
]


@pytest.mark.parametrize("d_out,d_in,T,flags", PLAN_CASES)
def test_plan_runs_equal_linear(d_out, d_in, T, flags):
    """bitlinear_linear_plan_run gives the bits of bitlinear_linear with the
    same arguments, on every path, run after run with new activations."""
    import ctypes as C
    W = draw(Problem("pl", d_in, d_out, T, 0.02, 0.01, 50.0, 31))[0]
    w = bl.pack_weights(W.to(dev()), EPS)
    sc = guarded_scratch(T, d_in)
    gy = Guarded((T, d_out), torch.bfloat16)
    h = C.c_void_p()
    L = bl.lib()
    assert L.bitlinear_linear_plan_create(
        w.packed.data_ptr(), w.gamma.data_ptr(), d_out, d_in, T, None, flags, EPS, NORM_EPS,
        sc[0].t.data_ptr(), sc[1].t.data_ptr(), sc[2].t.data_ptr(), gy.t.data_ptr(),
        bl.OUT_BF16, C.byref(h)) == bl.OK
    try:
        gen = torch.Generator().manual_seed(9)
        for _ in range(3):
            X = (torch.randn(T, d_in, generator=gen) * 2).to(torch.bfloat16).to(dev())
            assert L.bitlinear_linear_plan_run(h, X.data_ptr(),
                                               torch.cuda.current_stream().cuda_stream) == bl.OK
            ref = bl.linear(w, X, rmsnorm=bool(flags & bl.RMSNORM), out_dtype=torch.bfloat16,
                            static_weights=bool(flags & bl.STATIC_WEIGHTS),
                            per_tensor=bool(flags & bl.PER_TENSOR_ABSMAX))
            check_all(gy, *sc)
            assert torch.equal(gy.t, ref)
    finally:
        L.bitlinear_plan_destroy(h)
    # T = 0: a plan that enqueues nothing.
    assert L.bitlinear_linear_plan_create(
        w.packed.data_ptr(), w.gamma.data_ptr(), d_out, d_in, 0, None, flags, EPS, NORM_EPS,
        None, None, None, None, bl.OUT_BF16, C.byref(h)) == bl.OK
    assert L.bitlinear_linear_plan_run(h, None, None) == bl.OK
    L.bitlinear_plan_destroy(h)


def test_step_graph_replays_copies_and_calls():
    """A StepGraph of (pinned host X -> device, LinearPlan, device Y -> pinned
    host) gives, for new host contents on every replay, the same bits as an
    eager bl.linear of those contents."""
    d_out, d_in = 2560, 1024
    W, X = draw(Problem("sg", d_in, d_out, 2, 0.02, 0.01, 50.0, 14))
    w = bl.pack_weights(W.to(dev()), EPS)
    cs = torch.cuda.Stream()
    host_x = torch.empty((2, d_in), dtype=torch.bfloat16).pin_memory()
    host_y = torch.empty((2, d_out), dtype=torch.bfloat16).pin_memory()
    dev_x = torch.empty((2, d_in), dtype=torch.bfloat16, device=dev())
    plan = bl.LinearPlan(w, 2, out_dtype=torch.bfloat16, static_weights=True, stream=cs)

    def step():
        dev_x.copy_(host_x, non_blocking=True)
        plan(dev_x)
        host_y.copy_(plan.out, non_blocking=True)

    host_x.copy_(X)
    g = bl.StepGraph(step, stream=cs)
    gen = torch.Generator().manual_seed(5)
    for _ in range(3):
        xnew = (torch.randn(2, d_in, generator=gen) * 3).to(torch.bfloat16)
        host_x.copy_(xnew)
        with torch.cuda.stream(cs):
            g()
        cs.synchronize()
        ref = bl.linear(w, xnew.to(dev()), out_dtype=torch.bfloat16)
        torch.cuda.synchronize()
        assert torch.equal(host_y, ref.cpu())
