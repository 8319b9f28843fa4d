"""CPU oracle for the BitNet b1.58 BitLinear forward path.

TEST INFRASTRUCTURE ONLY.  The tests, the smoke check and the benchmark's CPU
baseline leg are the only callers; the CUDA library never imports, links or
executes anything here, and this package imports nothing from it.

The arithmetic lives in ``bitlinear_oracle.c`` (plain scalar C, compiled with
``-ffp-contract=off`` and no fast-math).  This module only compiles it, loads
it with ctypes and marshals numpy arrays in and out.

Page cited throughout as [MF]: "BitNet b1.58: Mathematical Foundations of
1.58-Bit Ternary Quantization, Absmean Scaling, and Multiplication-Free LLM
Architectures", section 2 (weight absmean quantisation, activation absmax
quantisation, the linear transformation and rescaling) and section 6
(vectorized ternary GEMV: sign/zero masks, masked addition).

Parity pins: every function here is pinned by ``tests/test_oracle_pins.py``
against closed forms, library routines, hand-worked fixtures and brute force;
none is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "bitlinear_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
# The same source built with OpenMP: int_matmul's independent outputs are
# split over the host's cores.  Only the benchmark's CPU baseline uses it.
_LIB_OMP = os.path.join(_HERE, "liboracle_omp.so")

QB_MINUS_1 = 127  # [MF] §2: Q_b - 1, multiplier and clip bound of the activation codes


def _compile(out: str, extra, force: bool) -> str:
    if (not force and os.path.exists(out)
            and os.path.getmtime(out) >= os.path.getmtime(_SRC)):
        return out
    tmp = out + ".tmp.%d" % os.getpid()
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
           "-fno-fast-math", "-fno-unsafe-math-optimizations", "-Wall", "-Wextra",
           "-Wno-unknown-pragmas", *extra, _SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (plain, and the OpenMP build of the same
    source); returns the path of the plain shared object."""
    _compile(_LIB_OMP, ["-fopenmp"], force)
    return _compile(_LIB, [], force)


_lib = None
_lib_omp = None


def _load(parallel: bool = False):
    global _lib, _lib_omp
    if parallel:
        if _lib_omp is None:
            build()
            lib = ctypes.CDLL(_LIB_OMP)
            _declare(lib)
            _lib_omp = lib
        return _lib_omp
    if _lib is None:
        lib = ctypes.CDLL(build())
        _declare(lib)
        _lib = lib
    return _lib


def threads(parallel: bool = True) -> int:
    """Threads the oracle's parallel loops use (1 for the plain build)."""
    return int(_load(parallel).oracle_threads())


def _declare(lib):
    """Argument and result types of every exported oracle function."""
    i64, f32, i32 = ctypes.c_int64, ctypes.c_float, ctypes.c_int
    vp = ctypes.c_void_p
    lib.oracle_bf16_to_f32.argtypes = [ctypes.c_uint16]
    lib.oracle_bf16_to_f32.restype = f32
    lib.oracle_f32_to_bf16.argtypes = [f32]
    lib.oracle_f32_to_bf16.restype = ctypes.c_uint16
    lib.oracle_abs_sum.argtypes = [vp, i64, i64]
    lib.oracle_abs_sum.restype = ctypes.c_double
    lib.oracle_absmean_gamma.argtypes = [vp, i64, i64]
    lib.oracle_absmean_gamma.restype = f32
    lib.oracle_ternarize.argtypes = [vp, i64, f32, f32, vp]
    lib.oracle_ternarize.restype = None
    lib.oracle_pack.argtypes = [vp, i64, i64, vp]
    lib.oracle_pack.restype = i32
    lib.oracle_unpack.argtypes = [vp, i64, i64, vp]
    lib.oracle_unpack.restype = i32
    lib.oracle_unpack_row.argtypes = [vp, i64, i64, i64, vp]
    lib.oracle_unpack_row.restype = i32
    lib.oracle_base3_cols.argtypes = [i64]
    lib.oracle_base3_cols.restype = i64
    lib.oracle_pack_base3.argtypes = [vp, i64, i64, vp]
    lib.oracle_pack_base3.restype = i32
    lib.oracle_unpack_base3.argtypes = [vp, i64, i64, vp]
    lib.oracle_unpack_base3.restype = i32
    lib.oracle_binarize.argtypes = [vp, i64, vp]
    lib.oracle_binarize.restype = None
    lib.oracle_w1_cols.argtypes = [i64]
    lib.oracle_w1_cols.restype = i64
    lib.oracle_pack_w1.argtypes = [vp, i64, i64, vp]
    lib.oracle_pack_w1.restype = i32
    lib.oracle_unpack_w1.argtypes = [vp, i64, i64, vp]
    lib.oracle_unpack_w1.restype = i32
    lib.oracle_quant_act_bits.argtypes = [vp, i64, i64, vp, i32, i32, i32, f32, f32, vp,
                                          vp, vp, vp, vp]
    lib.oracle_quant_act_bits.restype = None
    lib.oracle_rescale_bits.argtypes = [vp, i64, i64, f32, vp, i32, vp]
    lib.oracle_rescale_bits.restype = None
    lib.oracle_inv_rms.argtypes = [vp, i64, f32]
    lib.oracle_inv_rms.restype = f32
    lib.oracle_quant_act.argtypes = [vp, i64, i64, vp, i32, i32, f32, f32, vp,
                                     vp, vp, vp, vp]
    lib.oracle_quant_act.restype = None
    lib.oracle_int_matmul.argtypes = [vp, vp, i64, i64, i64, vp]
    lib.oracle_int_matmul.restype = None
    lib.oracle_dot_masked_add.argtypes = [vp, vp, i64]
    lib.oracle_dot_masked_add.restype = ctypes.c_int32
    lib.oracle_rescale.argtypes = [vp, i64, i64, f32, vp, vp]
    lib.oracle_rescale.restype = None
    lib.oracle_dequant_act_bf16.argtypes = [ctypes.c_int8, f32]
    lib.oracle_dequant_act_bf16.restype = ctypes.c_uint16
    lib.oracle_backward.argtypes = [vp, f32, vp, vp, vp, i64, i64, i64, vp, vp]
    lib.oracle_backward.restype = None
    lib.oracle_dense_bf16_dot.argtypes = [vp, vp, i64]
    lib.oracle_dense_bf16_dot.restype = ctypes.c_double
    lib.oracle_dense_bf16.argtypes = [vp, vp, i64, i64, i64, vp]
    lib.oracle_dense_bf16.restype = None
    lib.oracle_threads.argtypes = []
    lib.oracle_threads.restype = ctypes.c_int


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# ------------------------------------------------------------------ bf16 ---

def bf16_bits_to_f32(bits) -> np.ndarray:
    """Exact widening of bf16 bit patterns (uint16) to float32."""
    lib = _load()
    b = _c(bits, np.uint16).ravel()
    return np.array([lib.oracle_bf16_to_f32(int(v)) for v in b],
                    dtype=np.float32).reshape(np.shape(bits))


def f32_to_bf16_bits(x) -> np.ndarray:
    """float32 -> bf16 bit patterns, round to nearest even."""
    lib = _load()
    a = _c(x, np.float32).ravel()
    return np.array([lib.oracle_f32_to_bf16(float(v)) for v in a],
                    dtype=np.uint16).reshape(np.shape(x))


# ---------------------------------------------------- weight quantisation ---

def abs_sum(W) -> float:
    W = _c(W, np.float32)
    return _load().oracle_abs_sum(_ptr(W), W.shape[0], W.shape[1])


def absmean_gamma(W) -> float:
    """gamma = mean |W_ij| over the whole tensor ([MF] §2)."""
    W = _c(W, np.float32)
    return float(_load().oracle_absmean_gamma(_ptr(W), W.shape[0], W.shape[1]))


def ternarize(W, gamma: float, eps: float = 1e-5) -> np.ndarray:
    """W~ = RoundClip(W / (gamma + eps), -1, 1) in int8 ([MF] §2)."""
    W = _c(W, np.float32)
    out = np.empty(W.shape, dtype=np.int8)
    _load().oracle_ternarize(_ptr(W), W.size, gamma, eps, _ptr(out))
    return out


def pack(wq) -> np.ndarray:
    """Ternary codes [d_out][d_in] -> packed uint32 words (tile layout)."""
    wq = _c(wq, np.int8)
    n, k = wq.shape
    out = np.empty(n * k // 16 if (n % 16 == 0 and k % 256 == 0) else 0,
                   dtype=np.uint32)
    rc = _load().oracle_pack(_ptr(wq), n, k, _ptr(out) if out.size else None)
    if rc != 0:
        raise ValueError("oracle_pack: shape not a whole number of 16x256 tiles "
                         "or a code outside {-1,0,1}")
    return out


def unpack(packed, d_out: int, d_in: int) -> np.ndarray:
    packed = _c(packed, np.uint32)
    out = np.empty((d_out, d_in), dtype=np.int8)
    rc = _load().oracle_unpack(_ptr(packed), d_out, d_in, _ptr(out))
    if rc != 0:
        raise ValueError("oracle_unpack: invalid code 3 or bad shape")
    return out


def unpack_row(packed, d_out: int, d_in: int, o: int) -> np.ndarray:
    packed = _c(packed, np.uint32)
    out = np.empty(d_in, dtype=np.int8)
    rc = _load().oracle_unpack_row(_ptr(packed), d_out, d_in, o, _ptr(out))
    if rc != 0:
        raise ValueError("oracle_unpack_row: invalid code 3 or bad index")
    return out


def binarize(W) -> np.ndarray:
    """W1 codes: +1 where W >= 0, -1 elsewhere (the sign code of [MF] section 1
    read for the W1A4 regime)."""
    W = _c(W, np.float32)
    out = np.empty(W.shape, dtype=np.int8)
    _load().oracle_binarize(_ptr(W), W.size, _ptr(out))
    return out


def w1_cols(d_in: int) -> int:
    """Row width of the 1-bit format: d_in padded to a multiple of 512."""
    return int(_load().oracle_w1_cols(d_in))


def pack_w1(wq) -> np.ndarray:
    """Binary codes [d_out][d_in] in {-1, +1} -> uint32 words, one bit per
    weight, in 16 x 512 tiles."""
    wq = _c(wq, np.int8)
    n, k = wq.shape
    out = np.empty(n * w1_cols(k) // 32 if (n % 16 == 0 and k >= 1) else 0, dtype=np.uint32)
    rc = _load().oracle_pack_w1(_ptr(wq), n, k, _ptr(out) if out.size else None)
    if rc != 0:
        raise ValueError("oracle_pack_w1: d_out not a multiple of 16, or a code not +-1")
    return out


def unpack_w1(packed, d_out: int, d_in: int) -> np.ndarray:
    packed = _c(packed, np.uint32)
    if d_out % 16 or d_in < 1 or packed.size != d_out * w1_cols(d_in) // 32:
        raise ValueError("unpack_w1: size does not match the shape")
    out = np.empty((d_out, d_in), dtype=np.int8)
    rc = _load().oracle_unpack_w1(_ptr(packed), d_out, d_in, _ptr(out))
    if rc != 0:
        raise ValueError("oracle_unpack_w1: a padding bit is set")
    return out


def base3_cols(d_in: int) -> int:
    """Row width of the base-3 format: d_in padded to a multiple of 160."""
    return int(_load().oracle_base3_cols(d_in))


def pack_base3(wq) -> np.ndarray:
    """Ternary codes [d_out][d_in] -> base-3 bytes, five codes per byte
    ([MF] section 4), in 16 x 160 tiles."""
    wq = _c(wq, np.int8)
    n, k = wq.shape
    out = np.empty(n * base3_cols(k) // 5 if (n % 16 == 0 and k >= 1) else 0, dtype=np.uint8)
    rc = _load().oracle_pack_base3(_ptr(wq), n, k, _ptr(out) if out.size else None)
    if rc != 0:
        raise ValueError("oracle_pack_base3: d_out not a multiple of 16, or a code "
                         "outside {-1,0,1}")
    return out


def unpack_base3(packed, d_out: int, d_in: int) -> np.ndarray:
    packed = _c(packed, np.uint8)
    if d_out % 16 or d_in < 1 or packed.size != d_out * base3_cols(d_in) // 5:
        raise ValueError("unpack_base3: size does not match the shape")
    out = np.empty((d_out, d_in), dtype=np.int8)
    rc = _load().oracle_unpack_base3(_ptr(packed), d_out, d_in, _ptr(out))
    if rc != 0:
        raise ValueError("oracle_unpack_base3: byte above 242 or a nonzero padding code")
    return out


# ------------------------------------------------ activation quantisation ---

def inv_rms(x_bf16_bits, norm_eps: float = 1e-5) -> float:
    """1 / sqrt(mean(x^2) + norm_eps) of one token, in double, rounded to f32."""
    x = _c(x_bf16_bits, np.uint16)
    return float(_load().oracle_inv_rms(_ptr(x), x.size, norm_eps))


def quant_act(X_bf16_bits, gain=None, rmsnorm: bool = True, eps: float = 1e-5,
              norm_eps: float = 1e-5, inv_rms_in=None, per_tensor: bool = False,
              act_bits: int = 8):
    """Absmax quantisation to act_bits-bit codes (8: [-127, 127]; 4: [-7, 7]),
    per token (or per tensor), optional RMSNorm first ([MF] §2).

    Returns (xq int8 [T][K], beta f32 [T], rowsum int32 [T], inv_rms f32 [T]);
    with per_tensor every beta[t] is the one absmax of the whole X.
    """
    if act_bits not in (4, 8):
        raise ValueError("act_bits must be 4 or 8")
    X = _c(X_bf16_bits, np.uint16)
    T, K = X.shape
    g = None if gain is None else _c(gain, np.float32)
    r_in = None if inv_rms_in is None else _c(inv_rms_in, np.float32)
    xq = np.empty((T, K), dtype=np.int8)
    beta = np.empty(T, dtype=np.float32)
    rowsum = np.empty(T, dtype=np.int32)
    rms_out = np.empty(T, dtype=np.float32)
    _load().oracle_quant_act_bits(_ptr(X), T, K, _ptr(g), int(bool(rmsnorm)),
                                  int(bool(per_tensor)), act_bits, eps, norm_eps, _ptr(r_in),
                                  _ptr(xq), _ptr(beta), _ptr(rowsum), _ptr(rms_out))
    return xq, beta, rowsum, rms_out


# ----------------------------------------------------- product / rescale ---

def int_matmul(wq, xq, parallel: bool = False) -> np.ndarray:
    """acc[t][o] = sum_k W~[o][k] X~[t][k] in int32 ([MF] §2).  parallel: the
    OpenMP build (same arithmetic, outputs split over the host's cores)."""
    wq = _c(wq, np.int8)
    xq = _c(xq, np.int8)
    N, K = wq.shape
    T = xq.shape[0]
    acc = np.empty((T, N), dtype=np.int32)
    _load(parallel).oracle_int_matmul(_ptr(wq), _ptr(xq), T, N, K, _ptr(acc))
    return acc


def dot_masked_add(wrow, xrow) -> int:
    """Sign-mask / zero-mask masked-add dot product ([MF] §6)."""
    w = _c(wrow, np.int8)
    x = _c(xrow, np.int8)
    return int(_load().oracle_dot_masked_add(_ptr(w), _ptr(x), w.size))


def rescale(acc, gamma: float, beta, act_bits: int = 8) -> np.ndarray:
    """Y = acc * beta * gamma / (Q_b - 1), Q_b = 2^(act_bits - 1), in float64
    ([MF] §2)."""
    acc = _c(acc, np.int32)
    beta = _c(beta, np.float32)
    T, N = acc.shape
    y = np.empty((T, N), dtype=np.float64)
    _load().oracle_rescale_bits(_ptr(acc), T, N, gamma, _ptr(beta), act_bits, _ptr(y))
    return y


# ------------------------------------------------ dense bf16 (context) ---

def dense_bf16(W_bits, X_bits) -> np.ndarray:
    """Y = X W^T of bf16 bit patterns, in double (the layer BitLinear replaces)."""
    W = _c(W_bits, np.uint16)
    X = _c(X_bits, np.uint16)
    N, K = W.shape
    T = X.shape[0]
    y = np.empty((T, N), dtype=np.float64)
    _load().oracle_dense_bf16(_ptr(W), _ptr(X), T, N, K, _ptr(y))
    return y


def dense_bf16_dot(w_bits, x_bits) -> float:
    """One output of dense_bf16: sum_k w_k x_k in double, index order."""
    w = _c(w_bits, np.uint16)
    x = _c(x_bits, np.uint16)
    return float(_load().oracle_dense_bf16_dot(_ptr(w), _ptr(x), w.size))


# ------------------------------------------------ backward (STE, [MF] §3) ---

def dequant_act_bf16(q: int, beta: float) -> int:
    """X^ of one code: bf16 bits of fl32(q * fl32(beta / 127))."""
    return int(_load().oracle_dequant_act_bf16(int(q), float(beta)))


def backward(wq, gamma: float, xq, beta, dY_bits, want_dx: bool = True, want_dw: bool = True):
    """Straight-through-estimator gradients ([MF] §3): returns (dX [T][K],
    dW [N][K]) in double, either None when not asked for."""
    wq = _c(wq, np.int8)
    dY = _c(dY_bits, np.uint16)
    N, K = wq.shape
    T = dY.shape[0]
    if dY.ndim != 2 or dY.shape[1] != N:
        raise ValueError("dY must be [T][N] with N = wq.shape[0]")
    if want_dw:
        xq = _c(xq, np.int8)
        beta = _c(beta, np.float32)
        if xq.shape != (T, K) or beta.shape != (T,):
            raise ValueError("xq must be [T][K] and beta [T], T = dY.shape[0]")
    else:
        xq = beta = None
    dX = np.empty((T, K), dtype=np.float64) if want_dx else None
    dW = np.empty((N, K), dtype=np.float64) if want_dw else None
    _load().oracle_backward(_ptr(wq), gamma, _ptr(xq), _ptr(beta), _ptr(dY), T, N, K,
                            _ptr(dX), _ptr(dW))
    return dX, dW


def forward(W, X_bf16_bits, eps: float = 1e-5, norm_eps: float = 1e-5, gain=None,
            rmsnorm: bool = True, gamma=None, inv_rms_in=None):
    """The whole BitLinear forward on the CPU: returns a dict of every stage."""
    g = absmean_gamma(W) if gamma is None else float(gamma)
    wq = ternarize(W, g, eps)
    xq, beta, rowsum, r = quant_act(X_bf16_bits, gain, rmsnorm, eps, norm_eps,
                                    inv_rms_in)
    acc = int_matmul(wq, xq)
    y = rescale(acc, g, beta)
    return dict(gamma=g, wq=wq, xq=xq, beta=beta, rowsum=rowsum, inv_rms=r, acc=acc,
                y=y)
