"""Pins of the CPU oracle to facts other than itself.

Each test checks the oracle against something fixed by the page or by
mathematics: a hand-worked example, a closed form, a statistical law, a
library routine computing the same quantity another way, brute force on
tiny inputs, or an identity printed on the page.  Page cited as [MF]:
"BitNet b1.58: Mathematical Foundations of 1.58-Bit Ternary Quantization,
Absmean Scaling, and Multiplication-Free LLM Architectures".
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from workloads import Problem, bf16_bits, draw

RNG = np.random.default_rng(1234)


def _bits(x):
    return bf16_bits(torch.as_tensor(np.asarray(x, dtype=np.float32)).to(torch.bfloat16))


# ------------------------------------------------------------- worked example

def test_worked_example(golden_dir):
    """Hand-derived example from the formulas of [MF] §2 (the page prints none)."""
    ex = json.load(open(os.path.join(golden_dir, "worked_example.json")))
    W = np.array(ex["W"], dtype=np.float32)
    X = _bits(ex["X"])
    out = oracle.forward(W, X, eps=ex["eps"], norm_eps=ex["norm_eps"])
    assert out["gamma"] == ex["gamma"]
    np.testing.assert_array_equal(out["wq"], np.array(ex["W_ternary"]))
    assert abs(out["inv_rms"][0] - ex["inv_rms"]) < 2e-6
    assert abs(out["beta"][0] - ex["beta"]) < 2e-6
    np.testing.assert_array_equal(out["xq"], np.array(ex["X_int8"]))
    np.testing.assert_array_equal(out["rowsum"], np.array(ex["rowsum"]))
    np.testing.assert_array_equal(out["acc"], np.array(ex["acc"]))
    np.testing.assert_allclose(out["y"], np.array(ex["Y"]), rtol=2e-6)


# ------------------------------------------------------------------- bf16

def test_bf16_conversions_match_torch():
    x = np.concatenate([RNG.standard_normal(2000).astype(np.float32) * 10,
                        np.array([0.0, -0.0, 1.0, 1.00390625, 1.0078125,
                                  1.005859375, 1.001953125, 3.0e-39, 65504.0],
                                 dtype=np.float32)])
    mine = oracle.f32_to_bf16_bits(x)
    ref = bf16_bits(torch.from_numpy(x).to(torch.bfloat16))
    np.testing.assert_array_equal(mine, ref)
    back = oracle.bf16_bits_to_f32(ref)
    np.testing.assert_array_equal(
        back, torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy())


# ------------------------------------------------------------------ gamma

def test_gamma_constant_magnitude():
    """|W_ij| = c everywhere => gamma = c exactly ([MF] §2, absmean)."""
    c = np.float32(0.0234375)  # exactly representable
    signs = RNG.choice([-1.0, 1.0], size=(48, 256)).astype(np.float32)
    assert oracle.absmean_gamma(signs * c) == float(c)


def test_gamma_half_normal_mean():
    """E|W| = sigma*sqrt(2/pi) for W ~ N(0, sigma^2) (half-normal mean)."""
    for sigma, seed in ((0.02, 0), (0.015, 3)):
        W = draw(Problem("h", 1024, 1024, 1, sigma, 0.0, 1.0, seed))[0].numpy()
        g = oracle.absmean_gamma(W)
        mean = sigma * math.sqrt(2 / math.pi)
        se = sigma * math.sqrt(1 - 2 / math.pi) / math.sqrt(W.size)
        assert abs(g - mean) < 5 * se, (g, mean, se)


def test_gamma_sum_against_exact_sum():
    """The double sum agrees with math.fsum (correctly rounded) to 1e-12."""
    W = (RNG.standard_normal((64, 512)) * 0.02).astype(np.float32)
    exact = math.fsum(abs(float(v)) for v in W.ravel())
    assert abs(oracle.abs_sum(W) - exact) <= 1e-12 * exact
    assert oracle.absmean_gamma(W) == np.float32(exact / W.size)


def test_gamma_homogeneous_and_sign_free():
    W = (RNG.standard_normal((32, 256)) * 0.02).astype(np.float32)
    g = oracle.absmean_gamma(W)
    assert oracle.absmean_gamma(-W) == g
    assert oracle.absmean_gamma(W * np.float32(4.0)) == np.float32(4.0) * np.float32(g)
    assert abs(oracle.absmean_gamma(np.ascontiguousarray(W.T)) - g) <= 1e-7 * g


# ------------------------------------------------------------- ternarise

def test_ternary_alphabet_and_gaussian_zero_fraction():
    """W~ in {-1,0,1}; for Gaussian W the zero fraction is
    P(|Z| < sqrt(2/pi)/2) = erf(1/(2 sqrt(pi))) = 0.3101 and +-1 split evenly."""
    W = draw(Problem("z", 2048, 1024, 1, 0.02, 0.0, 1.0, 7))[0].numpy()
    wq = oracle.ternarize(W, oracle.absmean_gamma(W))
    assert set(np.unique(wq).tolist()) <= {-1, 0, 1}
    p0 = math.erf(1 / (2 * math.sqrt(math.pi)))
    frac0 = float((wq == 0).mean())
    se = math.sqrt(p0 * (1 - p0) / wq.size)
    assert abs(frac0 - p0) < 6 * se, (frac0, p0)
    fp, fm = float((wq == 1).mean()), float((wq == -1).mean())
    assert abs(fp - fm) < 12 * se


def test_roundclip_ties_and_clip():
    """RoundClip(z) = max(-1, min(1, floor(z + 0.5))): halves round up ([MF] §2).
    With gamma = 1 and eps = 0 the divisor is exactly 1, so z = W."""
    W = np.array([[0.5, -0.5, 1.5, -1.5, 0.49999997, -0.50000006, 7.0, -7.0,
                   0.0, -0.0, 1.0, -1.0]], dtype=np.float32)
    got = oracle.ternarize(W, 1.0, 0.0)[0].tolist()
    assert got == [1, 0, 1, -1, 0, -1, 1, -1, 0, 0, 1, -1]


def test_ternarize_is_nearest_level_with_ties_up():
    """Second formulation: the code is the level in {-1,0,1} nearest to
    z = fl32(W / fl32(gamma + eps)), ties to the larger level."""
    W = (RNG.standard_normal(4096) * 0.02).astype(np.float32)
    gamma, eps = 0.0159, 1e-5
    wq = oracle.ternarize(W[None, :], gamma, eps)[0]
    z = W / (np.float32(gamma) + np.float32(eps))            # binary32 as in [MF]
    levels = np.array([-1.0, 0.0, 1.0])
    d = np.abs(z.astype(np.float64)[:, None] - levels[None, :])
    best = np.where(d == d.min(axis=1, keepdims=True), levels[None, :], -np.inf).max(axis=1)
    np.testing.assert_array_equal(wq, best.astype(np.int8))


def test_zero_weights():
    W = np.zeros((16, 256), dtype=np.float32)
    g = oracle.absmean_gamma(W)
    assert g == 0.0
    assert not oracle.ternarize(W, g).any()


# ----------------------------------------------------------------- packing

def test_pack_layout_golden(golden_dir):
    ex = json.load(open(os.path.join(golden_dir, "packed_layout.json")))
    n, k = ex["d_out"], ex["d_in"]
    assert (oracle.pack(np.zeros((n, k), np.int8)) == 0x55555555).all()
    for c in ex["cases"]:
        wq = np.zeros((n, k), np.int8)
        wq[c["o"], c["k"]] = c["w"]
        p = oracle.pack(wq)
        expect = np.full(p.shape, 0x55555555, dtype=np.uint32)
        expect[c["word"]] = int(c["value"], 16)
        np.testing.assert_array_equal(p, expect, err_msg=str(c))


@pytest.mark.parametrize("shape", [(16, 256), (32, 512), (48, 768), (144, 2560)])
def test_pack_roundtrip(shape):
    wq = RNG.integers(-1, 2, size=shape).astype(np.int8)
    p = oracle.pack(wq)
    assert p.size == shape[0] * shape[1] // 16
    np.testing.assert_array_equal(oracle.unpack(p, *shape), wq)
    for o in (0, shape[0] - 1, shape[0] // 3):
        np.testing.assert_array_equal(oracle.unpack_row(p, *shape, o), wq[o])


# ------------------------------------------------------ base-3 packing ---

def test_base3_layout_golden(golden_dir):
    ex = json.load(open(os.path.join(golden_dir, "base3_layout.json")))
    n, k = ex["d_out"], ex["d_in"]
    zero = oracle.pack_base3(np.zeros((n, k), np.int8))
    assert zero.size == ex["bytes"] and (zero == 121).all()
    for c in ex["cases"]:
        wq = np.zeros((n, k), np.int8)
        wq[c["o"], c["k"]] = c["w"]
        p = oracle.pack_base3(wq)
        expect = np.full(p.shape, 121, dtype=np.uint8)
        expect[c["byte"]] = c["value"]
        np.testing.assert_array_equal(p, expect, err_msg=str(c))


def test_base3_constant_matrices():
    """All -1 packs to 0, all +1 to 242 = 2 (1 + 3 + 9 + 27 + 81); with a
    ragged width the padding columns hold W~ = 0 (digit 1)."""
    assert (oracle.pack_base3(np.full((16, 320), -1, np.int8)) == 0).all()
    assert (oracle.pack_base3(np.full((16, 320), 1, np.int8)) == 242).all()
    # d_in = 256: tile 1 covers columns 160..319, of which 256..319 are padding:
    # groups 0..3 (columns 160..239) and 4 (240..255 real, 256..259 padding).
    p = oracle.pack_base3(np.full((16, 256), -1, np.int8)).reshape(2, 16, 32)
    assert (p[0] == 0).all()
    assert (p[1][:, :16] == 0).all()                  # groups 0..3: all real
    # group 4: columns 240 + 4i + j, real for i < 4, padding (digit 1) for i = 4
    assert (p[1][:, 16:20] == 81).all()
    assert (p[1][:, 20:] == 121).all()                # groups 5..7: all padding


@pytest.mark.parametrize("shape", [(16, 160), (16, 256), (32, 512), (48, 2560), (16, 4096),
                                   (32, 11008)])
def test_base3_roundtrip_and_size(shape):
    wq = RNG.integers(-1, 2, size=shape).astype(np.int8)
    p = oracle.pack_base3(wq)
    kp = -(-shape[1] // 160) * 160
    assert oracle.base3_cols(shape[1]) == kp
    assert p.size == shape[0] * kp // 5              # 8/5 = 1.6 bits per padded weight
    assert p.max() <= 242
    np.testing.assert_array_equal(oracle.unpack_base3(p, *shape), wq)
    # The code histogram survives packing: count the digits of every byte.
    digits = np.stack([(p.astype(np.int64) // 3 ** i) % 3 for i in range(5)], axis=-1)
    counts = np.bincount(digits.ravel(), minlength=3)
    want = np.bincount((wq + 1).ravel(), minlength=3)
    want[1] += shape[0] * (kp - shape[1])            # padding columns are W~ = 0
    np.testing.assert_array_equal(counts, want)


def test_base3_is_a_bijection_on_a_tile():
    """Every (row, column) of a 16 x 160 tile owns its own (byte, digit)."""
    seen = set()
    base = oracle.pack_base3(np.zeros((16, 160), np.int8)).astype(np.int64)
    for o in range(16):
        for k in range(160):
            wq = np.zeros((16, 160), np.int8)
            wq[o, k] = 1
            d = oracle.pack_base3(wq).astype(np.int64) - base
            nz = np.flatnonzero(d)
            assert nz.size == 1
            power = int(round(math.log(d[nz[0]], 3)))
            assert 3 ** power == d[nz[0]] and 0 <= power < 5
            seen.add((int(nz[0]), power))
    assert len(seen) == 16 * 160


def test_base3_rejects_bad_input():
    with pytest.raises(ValueError):
        oracle.pack_base3(np.full((16, 160), 2, np.int8))
    with pytest.raises(ValueError):
        oracle.pack_base3(np.zeros((8, 160), np.int8))
    bad = oracle.pack_base3(np.zeros((16, 160), np.int8))
    bad[7] = 243
    with pytest.raises(ValueError):
        oracle.unpack_base3(bad, 16, 160)
    pad = oracle.pack_base3(np.zeros((16, 256), np.int8))
    pad[-1] = 0                                      # padding column set to -1
    with pytest.raises(ValueError):
        oracle.unpack_base3(pad, 16, 256)


# ------------------------------------------------------- W1A4 (binary) ---

def test_binarize_signs():
    """Sign code of the W1 regime: +1 for W >= 0 (both zeros), -1 below."""
    W = np.array([0.0, -0.0, 1e-38, -1e-38, 3.5, -2.0, 1e-45, -1e-45], np.float32)
    np.testing.assert_array_equal(oracle.binarize(W), [1, 1, 1, -1, 1, -1, 1, -1])
    G = (RNG.standard_normal(100000) * 0.02).astype(np.float32)
    b = oracle.binarize(G)
    assert set(np.unique(b)) == {-1, 1}
    assert abs((b == 1).mean() - 0.5) < 0.01                # symmetric distribution


def test_absmean_is_least_squares_scale_of_sign_code():
    """The absmean gamma minimises sum (W - a sign W)^2 over a: the derivative
    sum |W| - N a vanishes at a = gamma, and nearby scales fit worse."""
    W = (RNG.standard_normal((64, 512)) * 0.02).astype(np.float32)
    g = oracle.absmean_gamma(W)
    s = oracle.binarize(W).astype(np.float64)
    w = W.astype(np.float64)
    f = lambda a: float(((w - a * s) ** 2).sum())
    assert abs(float((s * (w - g * s)).sum())) <= 1e-6 * float(np.abs(w).sum())
    assert f(g) < f(g * 1.01) and f(g) < f(g * 0.99)


def test_w1_layout_golden(golden_dir):
    ex = json.load(open(os.path.join(golden_dir, "w1_layout.json")))
    n, k = ex["d_out"], ex["d_in"]
    zero = oracle.pack_w1(np.full((n, k), -1, np.int8))
    assert zero.size == ex["words"] and not zero.any()
    for c in ex["cases"]:
        wq = np.full((n, k), -1, np.int8)
        wq[c["o"], c["k"]] = 1
        p = oracle.pack_w1(wq)
        expect = np.zeros(p.shape, dtype=np.uint32)
        expect[c["word"]] = int(c["value"], 16)
        np.testing.assert_array_equal(p, expect, err_msg=str(c))


@pytest.mark.parametrize("shape", [(16, 256), (32, 512), (48, 2560), (16, 4096), (32, 11008)])
def test_w1_roundtrip_and_size(shape):
    wq = (RNG.integers(0, 2, size=shape) * 2 - 1).astype(np.int8)
    p = oracle.pack_w1(wq)
    kp = -(-shape[1] // 512) * 512
    assert oracle.w1_cols(shape[1]) == kp
    assert p.size == shape[0] * kp // 32                 # one bit per padded weight
    np.testing.assert_array_equal(oracle.unpack_w1(p, *shape), wq)
    # The number of +1 codes survives packing.
    ones = sum(bin(int(v)).count("1") for v in p)
    assert ones == int((wq == 1).sum())
    if shape[1] % 512 == 0:                               # no padding: every bit set
        assert (oracle.pack_w1(np.ones(shape, np.int8)) == 0xFFFFFFFF).all()


def test_w1_is_a_bijection_on_a_tile():
    seen = set()
    for o in range(16):
        for k in range(512):
            wq = np.full((16, 512), -1, np.int8)
            wq[o, k] = 1
            p = oracle.pack_w1(wq)
            nz = np.flatnonzero(p)
            assert nz.size == 1 and bin(int(p[nz[0]])).count("1") == 1
            seen.add((int(nz[0]), int(p[nz[0]]).bit_length() - 1))
    assert len(seen) == 16 * 512


def test_w1_rejects_bad_input():
    with pytest.raises(ValueError):
        oracle.pack_w1(np.zeros((16, 512), np.int8))          # 0 is not a binary code
    pad = oracle.pack_w1(np.full((16, 256), -1, np.int8))
    pad[15] = 1                                               # column 480: padding
    with pytest.raises(ValueError):
        oracle.unpack_w1(pad, 16, 256)


def test_quant_act_4bit():
    """A4: Q_b = 2^3 levels, codes in [-7, 7], the absmax element of a token at
    +-7, q the integer nearest to v = fl32(n * fl32(7 / (beta + eps))) with ties
    upward; act_bits = 8 is the default quantiser."""
    X = draw(Problem("a4", 512, 16, 5, 0.02, 0.01, 50.0, 4))[1]
    bits = bf16_bits(X)
    xq, beta, rowsum, r = oracle.quant_act(bits, act_bits=4)
    assert xq.min() >= -7 and xq.max() <= 7
    np.testing.assert_array_equal(rowsum, xq.astype(np.int64).sum(axis=1))
    xf = X.float().numpy()
    for t in range(5):
        n = xf[t] * np.float32(r[t])
        assert abs(int(xq[t][np.argmax(np.abs(n))])) == 7
        s = np.float32(7.0) / (np.float32(beta[t]) + np.float32(1e-5))
        v = (n * s).astype(np.float64)
        cand = np.stack([np.floor(v), np.floor(v) + 1])
        d = np.abs(v[None] - cand)
        q = np.where(d[1] <= d[0], cand[1], cand[0])
        np.testing.assert_array_equal(xq[t], np.clip(q, -7, 7).astype(np.int8))
    q8 = oracle.quant_act(bits, act_bits=8)
    q0 = oracle.quant_act(bits)
    for a, b in zip(q8, q0):
        np.testing.assert_array_equal(a, b)


def test_w1a4_forward_against_dequantised_product():
    """Y = (X~ W~^T) beta gamma / 7 equals the fp64 product of the dequantised
    operands (X~ beta / 7) and (gamma W~)."""
    W, X = draw(Problem("w1a4", 256, 16, 3, 0.02, 0.01, 50.0, 7))
    Wn = W.numpy()
    g = oracle.absmean_gamma(Wn)
    wq = oracle.binarize(Wn)
    xq, beta, _, _ = oracle.quant_act(bf16_bits(X), act_bits=4)
    y = oracle.rescale(oracle.int_matmul(wq, xq), g, beta, act_bits=4)
    ref = (xq.astype(np.float64) * beta.astype(np.float64)[:, None] / 7.0) @ \
          (float(g) * wq.astype(np.float64)).T
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-15)


def test_pack_exhaustive_groups():
    """All 81 joint values of the four codes that share one byte (same s)
    and of the four that share one 2-bit slot across bytes (same j)."""
    import itertools
    for combo in itertools.product((-1, 0, 1), repeat=4):
        for pos in (lambda i: i, lambda i: 4 * i):     # same-s group / same-j group
            wq = np.zeros((16, 256), np.int8)
            for i, v in enumerate(combo):
                wq[5, 32 + pos(i)] = v
            np.testing.assert_array_equal(
                oracle.unpack(oracle.pack(wq), 16, 256), wq)


def test_pack_rejects_bad_input():
    with pytest.raises(ValueError):
        oracle.pack(np.full((16, 256), 2, np.int8))
    with pytest.raises(ValueError):
        oracle.pack(np.zeros((16, 128), np.int8))
    p = oracle.pack(np.zeros((16, 256), np.int8))
    p[7] |= 3  # plant the unused code 3
    with pytest.raises(ValueError):
        oracle.unpack(p, 16, 256)


# ------------------------------------------------------- activation quant

def test_inv_rms_matches_torch_rms_norm():
    """The reciprocal RMS agrees with torch.nn.functional.rms_norm (float64),
    whose output is x * r, to 1e-7."""
    X = draw(Problem("r", 2560, 16, 8, 0.02, 0.005, 100.0, 11))[1]
    bits = bf16_bits(X)
    x64 = X.to(torch.float64)
    y = torch.nn.functional.rms_norm(x64, (x64.shape[1],), eps=float(np.float32(1e-5)))
    for t in range(X.shape[0]):
        k = int(torch.argmax(x64[t].abs()))
        lib_r = float(y[t, k] / x64[t, k])
        assert abs(oracle.inv_rms(bits[t]) - lib_r) <= 1e-7 * lib_r


def test_quant_act_invariants():
    X = draw(Problem("a", 2560, 16, 8, 0.02, 0.005, 100.0, 5))[1]
    bits = bf16_bits(X)
    xq, beta, rowsum, r = oracle.quant_act(bits)
    assert xq.min() >= -127 and xq.max() <= 127
    np.testing.assert_array_equal(rowsum, xq.astype(np.int64).sum(axis=1))
    xf = X.float().numpy()
    for t in range(xq.shape[0]):
        k = int(np.argmax(np.abs(xf[t])))
        assert abs(int(xq[t, k])) == 127                    # absmax channel -> +-Qb-1
        assert np.all((xq[t] == 0) | (np.sign(xq[t]) == np.sign(xf[t])))
        np.testing.assert_allclose(beta[t], np.abs(xf[t]).max() * r[t], rtol=2e-7)


def test_quant_act_nearest_integer():
    """Second formulation: q is the integer nearest to v = fl32(n * s),
    ties upward, clipped to [-127, 127]."""
    X = draw(Problem("n", 512, 16, 4, 0.02, 0.01, 50.0, 2))[1]
    bits = bf16_bits(X)
    xq, beta, _, r = oracle.quant_act(bits)
    xf = X.float().numpy()
    for t in range(4):
        n = xf[t] * np.float32(r[t])
        s = np.float32(127.0) / (np.float32(beta[t]) + np.float32(1e-5))
        v = (n * s).astype(np.float64)
        cand = np.stack([np.floor(v), np.floor(v) + 1])
        d = np.abs(v[None] - cand)
        q = np.where(d[1] <= d[0], cand[1], cand[0])
        np.testing.assert_array_equal(xq[t], np.clip(q, -127, 127).astype(np.int8))


def test_quant_act_scale_invariance():
    """With eps = 0 the codes of 2^m x equal the codes of x, with and
    without RMSNorm (norm_eps = 0 too)."""
    X = draw(Problem("s", 512, 16, 4, 0.02, 0.01, 50.0, 9))[1]
    for rmsnorm in (False, True):
        base = oracle.quant_act(bf16_bits(X), rmsnorm=rmsnorm, eps=0.0, norm_eps=0.0)[0]
        for m in (-3, 1, 5):
            Xs = (X.float() * 2.0 ** m).to(torch.bfloat16)
            got = oracle.quant_act(bf16_bits(Xs), rmsnorm=rmsnorm, eps=0.0,
                                   norm_eps=0.0)[0]
            np.testing.assert_array_equal(got, base)
        g = np.full(512, 4.0, np.float32)
        got = oracle.quant_act(bf16_bits(X), gain=g, rmsnorm=True, eps=0.0,
                               norm_eps=0.0)[0]
        np.testing.assert_array_equal(got, oracle.quant_act(
            bf16_bits(X), rmsnorm=True, eps=0.0, norm_eps=0.0)[0])


def test_quant_act_special_tokens():
    K = 256
    zero = np.zeros((1, K), np.float32)
    const = np.full((1, K), -3.0, np.float32)
    onehot = np.zeros((1, K), np.float32)
    onehot[0, 77] = 2.5
    xq, beta, S, r = oracle.quant_act(_bits(np.concatenate([zero, const, onehot])))
    assert beta[0] == 0 and not xq[0].any() and S[0] == 0
    assert (xq[1] == -127).all() and S[1] == -127 * K
    assert xq[2, 77] == 127 and np.count_nonzero(xq[2]) == 1
    # reciprocal rms of a one-hot token is 1/sqrt(v^2/K + eps): closed form
    assert abs(r[2] - 1 / math.sqrt(2.5 ** 2 / K + float(np.float32(1e-5)))) < 1e-6


def test_quant_act_supplied_inv_rms_is_used():
    X = draw(Problem("u", 512, 16, 3, 0.02, 0.01, 50.0, 4))[1]
    bits = bf16_bits(X)
    _, _, _, r = oracle.quant_act(bits)
    a = oracle.quant_act(bits, inv_rms_in=r)
    b = oracle.quant_act(bits)
    for u, v in zip(a, b):
        np.testing.assert_array_equal(u, v)
    c = oracle.quant_act(bits, inv_rms_in=r * 2)
    np.testing.assert_array_equal(c[3], r * 2)


# ------------------------------------------------------------------ product

@pytest.mark.parametrize("T,N,K", [(1, 16, 256), (3, 48, 512), (5, 32, 768)])
def test_int_matmul_brute_force(T, N, K):
    wq = RNG.integers(-1, 2, size=(N, K)).astype(np.int8)
    xq = RNG.integers(-127, 128, size=(T, K)).astype(np.int8)
    acc = oracle.int_matmul(wq, xq)
    np.testing.assert_array_equal(acc, xq.astype(np.int64) @ wq.astype(np.int64).T)
    # The OpenMP build (every host core, used for the timed CPU baseline)
    # computes the same exact sums.
    np.testing.assert_array_equal(oracle.int_matmul(wq, xq, parallel=True), acc)


def test_masked_add_identity_exhaustive():
    """[MF] §6: accumulator += (x XOR sign) - sign where W != 0.  Over every
    legal int8 activation and every ternary weight this equals w * x."""
    for w in (-1, 0, 1):
        for x in range(-127, 128):
            got = oracle.dot_masked_add(np.array([w], np.int8), np.array([x], np.int8))
            assert got == w * x


def test_masked_add_matches_int_matmul():
    wq = RNG.integers(-1, 2, size=(8, 1024)).astype(np.int8)
    xq = RNG.integers(-127, 128, size=(2, 1024)).astype(np.int8)
    acc = oracle.int_matmul(wq, xq)
    for t in range(2):
        for o in range(8):
            assert oracle.dot_masked_add(wq[o], xq[t]) == acc[t, o]


def test_forward_equals_float_matmul_of_dequantised_operands():
    """Y = (X~ W~^T) beta gamma / 127 equals the fp64 product of the
    dequantised operands (gamma W~) and (beta X~ / 127) ([MF] §2)."""
    p = Problem("f", 512, 48, 4, 0.02, 0.01, 50.0, 6)
    W, X = draw(p)
    out = oracle.forward(W.numpy(), bf16_bits(X))
    Wd = out["gamma"] * out["wq"].astype(np.float64)
    Xd = out["beta"].astype(np.float64)[:, None] * out["xq"].astype(np.float64) / 127.0
    np.testing.assert_allclose(out["y"], Xd @ Wd.T, rtol=1e-12, atol=1e-15)


def test_forward_special_cases():
    K, N = 256, 16
    W = (RNG.standard_normal((N, K)) * 0.02).astype(np.float32)
    # zero weights -> y = 0
    z = oracle.forward(np.zeros((N, K), np.float32), _bits(RNG.standard_normal((2, K))))
    assert not z["y"].any()
    # zero activations -> y = 0
    z = oracle.forward(W, _bits(np.zeros((2, K))))
    assert not z["y"].any()
    # one-hot activation v e_j without RMSNorm: y_o = gamma * W~[o][j] * v
    x = np.zeros((1, K), np.float32)
    x[0, 9] = -1.5
    g = oracle.absmean_gamma(W)
    wq = oracle.ternarize(W, g)
    xq, beta, _, _ = oracle.quant_act(_bits(x), rmsnorm=False)
    y = oracle.rescale(oracle.int_matmul(wq, xq), g, beta)[0]
    np.testing.assert_allclose(y, g * wq[:, 9] * -1.5, rtol=1e-6)


# ------------------------------------------------- dense bf16 (context) ---

def test_dense_bf16_brute_force():
    """Y = X W^T of bf16 operands against pure-Python loops over exact fractions."""
    from fractions import Fraction
    W = _bits(RNG.standard_normal((3, 5)) * 0.5)
    X = _bits(RNG.standard_normal((2, 5)) * 3.0)
    Wf = oracle.bf16_bits_to_f32(W).astype(np.float64)
    Xf = oracle.bf16_bits_to_f32(X).astype(np.float64)
    y = oracle.dense_bf16(W, X)
    for t in range(2):
        for o in range(3):
            exact = sum(Fraction(float(Wf[o, k])) * Fraction(float(Xf[t, k])) for k in range(5))
            assert abs(Fraction(y[t, o]) - exact) <= abs(exact) * Fraction(1, 2 ** 50)


def test_dense_bf16_against_numpy_and_identity():
    W = _bits(RNG.standard_normal((16, 256)) * 0.02)
    X = _bits(RNG.standard_normal((3, 256)))
    y = oracle.dense_bf16(W, X)
    ref = oracle.bf16_bits_to_f32(X).astype(np.float64) @ \
        oracle.bf16_bits_to_f32(W).astype(np.float64).T
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-15)
    # W = identity rows: Y reproduces X exactly.
    eye = _bits(np.eye(256, dtype=np.float32)[:16])
    np.testing.assert_array_equal(oracle.dense_bf16(eye, X),
                                  oracle.bf16_bits_to_f32(X)[:, :16].astype(np.float64))
    # One output through the single-dot entry point equals the full product.
    assert oracle.dense_bf16_dot(W[5], X[2]) == y[2, 5]


# ------------------------------------------------- per-tensor absmax (NEXT) ---

def test_per_tensor_worked_example():
    """Hand-derived: X = [[1, -2], [4, 0.5]], no RMSNorm, beta = 4 for both
    tokens, scale = 127 / (4 + 1e-5) = 31.7499...; 1 -> floor(32.25) = 32,
    -2 -> floor(-63.0) = -63, 4 -> 127, 0.5 -> floor(16.37) = 16."""
    X = _bits([[1.0, -2.0], [4.0, 0.5]])
    xq, beta, rs, _ = oracle.quant_act(X, rmsnorm=False, per_tensor=True)
    np.testing.assert_array_equal(xq, [[32, -63], [127, 16]])
    np.testing.assert_array_equal(beta, [4.0, 4.0])
    np.testing.assert_array_equal(rs, [-31, 143])
    # Per token the first row would use its own beta = 2 instead.
    xq1, beta1, _, _ = oracle.quant_act(X, rmsnorm=False, per_tensor=False)
    np.testing.assert_array_equal(beta1, [2.0, 4.0])
    assert xq1[0, 1] == -127


@pytest.mark.parametrize("rmsnorm", [False, True])
def test_per_tensor_properties(rmsnorm):
    W, X = draw(Problem("pt", 512, 16, 6, 0.02, 0.01, 50.0, 9))
    xb = bf16_bits(X)
    xq_t, beta_t, _, r_t = oracle.quant_act(xb, rmsnorm=rmsnorm)
    xq, beta, rs, r = oracle.quant_act(xb, rmsnorm=rmsnorm, per_tensor=True)
    np.testing.assert_array_equal(r, r_t)                 # the normalisation is per token
    assert np.all(beta == beta_t.max())                   # one beta: the largest per-token one
    np.testing.assert_array_equal(rs, xq.astype(np.int64).sum(axis=1))
    top = int(np.argmax(beta_t))
    np.testing.assert_array_equal(xq[top], xq_t[top])     # that token is unchanged
    assert np.abs(xq[top]).max() == 127
    # Every other token's largest code is its own absmax on the shared scale.
    scale = np.float32(127.0) / (np.float32(beta[0]) + np.float32(1e-5))
    for t in range(6):
        expect = np.floor(np.float64(np.float32(beta_t[t] * scale)) + 0.5)
        assert np.abs(xq[t]).max() == min(expect, 127)
    # One token: the two scopes coincide.
    a = oracle.quant_act(xb[:1], rmsnorm=rmsnorm, per_tensor=True)
    b = oracle.quant_act(xb[:1], rmsnorm=rmsnorm, per_tensor=False)
    for u, v in zip(a, b):
        np.testing.assert_array_equal(u, v)


def test_per_tensor_scale_invariance():
    """Without RMSNorm and with eps = 0, scaling all of X by 2^m (exact in
    bf16) leaves the per-tensor codes unchanged."""
    _, X = draw(Problem("ps", 256, 16, 4, 0.02, 0.02, 30.0, 4))
    base = oracle.quant_act(bf16_bits(X), rmsnorm=False, eps=0.0, per_tensor=True)[0]
    for m in (-3, 5):
        Xs = (X.float() * (2.0 ** m)).to(torch.bfloat16)
        np.testing.assert_array_equal(
            oracle.quant_act(bf16_bits(Xs), rmsnorm=False, eps=0.0, per_tensor=True)[0], base)


# --------------------------------------------- backward, STE (NEXT-2) ---

def _tiny_backward_case(T=3, N=32, K=256, seed=6):
    W, X = draw(Problem("bw", K, N, T, 0.02, 0.01, 50.0, seed))
    Wn = W.numpy()
    g = oracle.absmean_gamma(Wn)
    wq = oracle.ternarize(Wn, g, 1e-5)
    xq, beta, _, _ = oracle.quant_act(bf16_bits(X))
    dY = bf16_bits(torch.randn(T, N, generator=torch.Generator().manual_seed(seed + 1))
                   .to(torch.bfloat16))
    return wq, g, xq, beta, dY


def test_dequant_operand_matches_torch_rounding():
    """X^ = bf16(fl32(q * fl32(beta / 127))) against torch's own bf16 rounding."""
    for beta in (0.37, 3.1415, 127.0, 1e-3):
        s = np.float32(beta) / np.float32(127.0)
        for q in (-127, -64, -1, 0, 1, 5, 99, 127):
            ref = torch.tensor(np.float32(q) * s, dtype=torch.float32).to(torch.bfloat16)
            assert oracle.dequant_act_bf16(q, beta) == int(ref.view(torch.int16).item()) & 0xFFFF


def test_backward_is_the_gradient_of_the_forward():
    """The inference forward (int_matmul + rescale) is linear in the codes, so
    raising one activation code by 1 changes L = sum(dY * Y) by
    dX[t][k] * beta_t / 127, and raising one weight code by 1 changes it by
    dW[o][k] up to the bf16 rounding of X^ (2^-8 relative per term)."""
    wq, g, xq, beta, dY = _tiny_backward_case()
    dX, dW = oracle.backward(wq, g, xq, beta, dY)
    dYf = oracle.bf16_bits_to_f32(dY).astype(np.float64)

    def loss(w, x):
        return float((dYf * oracle.rescale(oracle.int_matmul(w, x), g, beta)).sum())

    base = loss(wq, xq)
    rng = np.random.default_rng(0)
    for _ in range(8):
        t, k = int(rng.integers(0, xq.shape[0])), int(rng.integers(0, xq.shape[1]))
        x2 = xq.copy()
        x2[t, k] += 1 if x2[t, k] < 127 else -1
        step = float(int(x2[t, k]) - int(xq[t, k])) * float(beta[t]) / 127.0
        assert abs((loss(wq, x2) - base) - dX[t, k] * step) <= 1e-9 * (abs(base) + 1)
    mag = np.abs(dYf).T @ np.abs(xq.astype(np.float64) * beta[:, None] / 127.0) * g
    for _ in range(8):
        o, k = int(rng.integers(0, wq.shape[0])), int(rng.integers(0, wq.shape[1]))
        w2 = wq.copy()
        w2[o, k] += 1 if w2[o, k] < 1 else -1
        step = float(int(w2[o, k]) - int(wq[o, k]))
        assert abs((loss(w2, xq) - base) - dW[o, k] * step) <= 2.0 ** -8 * mag[o, k] + 1e-12


def test_backward_exact_fractions_and_special_cases():
    from fractions import Fraction
    wq, g, xq, beta, dY = _tiny_backward_case(T=2, N=16, K=256, seed=9)
    dX, dW = oracle.backward(wq, g, xq, beta, dY)
    dYf = oracle.bf16_bits_to_f32(dY)
    for t, k in ((0, 3), (1, 200)):
        exact = sum(Fraction(float(dYf[t, o])) * int(wq[o, k]) for o in range(16)) * Fraction(g)
        assert abs(Fraction(dX[t, k]) - exact) <= abs(exact) * Fraction(1, 2 ** 50)
    # One-hot dY: dX is gamma times one weight row; dW is gamma times one X^ row.
    oh = np.zeros_like(dY)
    oh[1, 5] = 0x3F80                                   # bf16 1.0
    dX1, dW1 = oracle.backward(wq, g, xq, beta, oh)
    np.testing.assert_array_equal(dX1[0], 0.0)
    np.testing.assert_array_equal(dX1[1], g * wq[5].astype(np.float64))
    xh = np.array([oracle.bf16_bits_to_f32(np.array([oracle.dequant_act_bf16(q, beta[1])],
                                                     dtype=np.uint16))[0] for q in xq[1]])
    np.testing.assert_array_equal(dW1[5], g * xh.astype(np.float64))
    assert not dW1[np.arange(16) != 5].any()
    z0, z1 = oracle.backward(wq, g, xq, beta, np.zeros_like(dY))
    assert not z0.any() and not z1.any()


def test_backward_rejects_mismatched_shapes():
    wq, g, xq, beta, dY = _tiny_backward_case(T=3, N=16, K=256, seed=2)
    with pytest.raises(ValueError):
        oracle.backward(wq, g, xq[:2], beta[:2], dY)          # tokens disagree
    with pytest.raises(ValueError):
        oracle.backward(wq[:8], g, xq, beta, dY)              # outputs disagree
    dX, dW = oracle.backward(wq, g, None, None, dY, want_dw=False)
    assert dW is None and dX.shape == (3, 256)
