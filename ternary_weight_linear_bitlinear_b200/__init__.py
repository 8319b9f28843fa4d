"""Python binding of the sm_100a BitNet b1.58 BitLinear library.

Argument marshalling only: every step of the computation runs in the CUDA
kernels of ``libbitlinear.so`` (C ABI in ``include/bitlinear.h``).  PyTorch
provides device memory and the current CUDA stream.  There is no CPU
fallback: if the library is missing, or no sm_100 device is present, every
call raises.

The operation ("BitNet b1.58: Mathematical Foundations of 1.58-Bit Ternary
Quantization, Absmean Scaling, and Multiplication-Free LLM Architectures",
section 2): gamma = mean|W|, W~ = RoundClip(W/(gamma+eps), -1, 1); per-token
beta = max|RMSNorm(x)|, X~ = RoundClip(x 127/(beta+eps), -127, 127);
Y = (X~ W~^T) beta gamma / 127 with int32 accumulation.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libbitlinear.so")

OUT_F32 = 0
OUT_BF16 = 1
RMSNORM = 1
STATIC_WEIGHTS = 2
PER_TENSOR_ABSMAX = 4
ACT_4BIT = 8

OK = 0
ERR_INVALID_ARG = 1
ERR_MISALIGNED = 2
ERR_UNSUPPORTED_SHAPE = 3
ERR_CUDA = 4
ERR_TIMEOUT = 5
ERR_DEVICE = 6

# Every exported entry point with (restype, argtypes), as in bitlinear.h.
_vp, _i64, _f32, _u32, _int = (ctypes.c_void_p, ctypes.c_int64, ctypes.c_float,
                               ctypes.c_uint32, ctypes.c_int)
SIGNATURES = {
    "bitlinear_version": (_int, []),
    "bitlinear_status_string": (ctypes.c_char_p, [_int]),
    "bitlinear_packed_words": (ctypes.c_size_t, [_i64, _i64]),
    "bitlinear_packed_bytes": (ctypes.c_size_t, [_i64, _i64]),
    "bitlinear_pack_workspace_bytes": (ctypes.c_size_t, [_i64, _i64]),
    "bitlinear_pack_weights": (_int, [_vp, _i64, _i64, _f32, _vp, _vp, ctypes.c_size_t,
                                      _vp, _vp, _vp]),
    "bitlinear_pack_weights_noalloc": (_int, [_vp, _i64, _i64, _f32, _vp, _vp, _vp]),
    "bitlinear_quant_act": (_int, [_vp, _i64, _i64, _vp, _u32, _f32, _f32, _vp, _vp, _vp,
                                   _vp, _vp, _vp]),
    "bitlinear_forward": (_int, [_vp, _vp, _i64, _i64, _vp, _vp, _vp, _i64, _vp, _int,
                                 _vp, _vp, ctypes.c_size_t, _vp]),
    "bitlinear_decode_workspace_bytes": (ctypes.c_size_t, [_i64, _i64]),
    "bitlinear_set_decode_split": (_int, [_int]),
    "bitlinear_set_decode_kernel": (_int, [_int]),
    "bitlinear_linear": (_int, [_vp, _vp, _i64, _i64, _vp, _i64, _vp, _u32, _f32, _f32, _vp,
                                _vp, _vp, _vp, _vp, _int, _vp, ctypes.c_size_t, _vp]),
    "bitlinear_base3_bytes": (ctypes.c_size_t, [_i64, _i64]),
    "bitlinear_repack_base3": (_int, [_vp, _i64, _i64, _vp, _vp]),
    "bitlinear_forward_base3": (_int, [_vp, _vp, _i64, _i64, _vp, _vp, _vp, _i64, _vp, _int,
                                       _vp, _vp, ctypes.c_size_t, _vp]),
    "bitlinear_linear_base3": (_int, [_vp, _vp, _i64, _i64, _vp, _i64, _vp, _u32, _f32, _f32, _vp,
                                      _vp, _vp, _vp, _vp, _int, _vp, ctypes.c_size_t, _vp]),
    "bitlinear_w1_packed_bytes": (ctypes.c_size_t, [_i64, _i64]),
    "bitlinear_pack_weights_w1": (_int, [_vp, _i64, _i64, _vp, _vp, ctypes.c_size_t, _vp, _vp,
                                         _vp]),
    "bitlinear_forward_w1": (_int, [_vp, _vp, _i64, _i64, _vp, _vp, _vp, _i64, _int, _vp, _int,
                                    _vp, _vp, ctypes.c_size_t, _vp]),
    "bitlinear_linear_w1": (_int, [_vp, _vp, _i64, _i64, _vp, _i64, _vp, _u32, _f32, _f32, _vp,
                                   _vp, _vp, _vp, _vp, _int, _vp, ctypes.c_size_t, _vp]),
    "bitlinear_dense_bf16_forward": (_int, [_vp, _i64, _i64, _vp, _i64, _vp, _int, _vp]),
    "bitlinear_backward_workspace_bytes": (ctypes.c_size_t, [_i64, _i64, _i64, _int, _int]),
    "bitlinear_backward": (_int, [_vp, _vp, _i64, _i64, _vp, _vp, _i64, _vp, _vp, _vp, _int, _vp,
                                  ctypes.c_size_t, _vp]),
    "bitlinear_linear_plan_create": (_int, [_vp, _vp, _i64, _i64, _i64, _vp, _u32, _f32, _f32,
                                            _vp, _vp, _vp, _vp, _int,
                                            ctypes.POINTER(ctypes.c_void_p)]),
    "bitlinear_linear_plan_run": (_int, [_vp, _vp, _vp]),
    "bitlinear_plan_destroy": (None, [_vp]),
    "bitlinear_device_error": (_int, [_vp, _int]),
    "bitlinear_get_last_device_error": (_int, [_vp]),
    "bitlinear_set_wait_limit_ns": (_int, [ctypes.c_uint64]),
    "bitlinear_wait_probe": (_int, [ctypes.c_uint64, _vp]),
}


class BitLinearError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__("%s: %s (status %d)" % (where, status_string(status), status))


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded library; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                "libbitlinear.so is not built (run python -m "
                "ternary_weight_linear_bitlinear_b200.build); there is no fallback")
        l = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(l, name)
            f.restype = res
            f.argtypes = args
        _lib = l
    return _lib


def status_string(status: int) -> str:
    return lib().bitlinear_status_string(status).decode()


def _check(status: int, where: str):
    if status != OK:
        raise BitLinearError(status, where)


def _ptr(t):
    # ctypes converts the integer address through the declared c_void_p.
    return None if t is None else t.data_ptr()


def _stream():
    return torch.cuda.current_stream().cuda_stream


def _need(t, dtype, name):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError("%s must be a CUDA tensor" % name)
    if t.dtype != dtype:
        raise TypeError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)


@dataclass
class PackedTernary:
    """Packed ternary weights of one BitLinear (layout in bitlinear.h)."""
    packed: torch.Tensor    # int32 [d_out * d_in / 16] (uint32 bit patterns)
    gamma: torch.Tensor     # float32 [1]
    d_out: int
    d_in: int


@dataclass
class PackedTernaryBase3:
    """The same ternary weights in the base-3 format, five codes per byte
    (layout in bitlinear.h); decode only (1 <= T <= 16)."""
    packed: torch.Tensor    # uint8 [base3_bytes(d_out, d_in)]
    gamma: torch.Tensor     # float32 [1], shared with the 2-bit weights
    d_out: int
    d_in: int


@dataclass
class PackedBinary:
    """Sign-binarised weights of the W1A4 regime, one bit per weight (layout
    in bitlinear.h); decode only (1 <= T <= 16)."""
    packed: torch.Tensor    # int32 [w1_packed_bytes(d_out, d_in) / 4] (uint32 patterns)
    gamma: torch.Tensor     # float32 [1], absmean scale
    d_out: int
    d_in: int


def _entry(w, name: str):
    """The entry point for w's format: name, name + '_base3' or name + '_w1'."""
    if isinstance(w, PackedTernaryBase3):
        full = name + "_base3"
    elif isinstance(w, PackedBinary):
        full = name + "_w1"
    else:
        full = name
    return getattr(lib(), full), full


def w1_packed_bytes(d_out: int, d_in: int) -> int:
    return int(lib().bitlinear_w1_packed_bytes(d_out, d_in))


def pack_weights_w1(W: torch.Tensor, gamma: torch.Tensor = None) -> PackedBinary:
    """Sign-binarise and pack fp32 latent weights [d_out][d_in] (W1)."""
    _need(W, torch.float32, "W")
    d_out, d_in = W.shape
    n = w1_packed_bytes(d_out, d_in)
    if n == 0:
        _check(ERR_UNSUPPORTED_SHAPE, "pack_weights_w1")
    out = PackedBinary(torch.empty(n // 4, dtype=torch.int32, device=W.device),
                       torch.empty(1, dtype=torch.float32, device=W.device), d_out, d_in)
    ws = None
    if gamma is None:
        ws = torch.empty(max(pack_workspace_bytes(d_out, d_in), 8), dtype=torch.uint8,
                         device=W.device)
    else:
        _need(gamma, torch.float32, "gamma")
    st = lib().bitlinear_pack_weights_w1(_ptr(W), d_out, d_in, _ptr(gamma), _ptr(ws),
                                         0 if ws is None else ws.numel(), _ptr(out.packed),
                                         _ptr(out.gamma), _stream())
    _check(st, "bitlinear_pack_weights_w1")
    return out


def base3_bytes(d_out: int, d_in: int) -> int:
    return int(lib().bitlinear_base3_bytes(d_out, d_in))


def repack_base3(w: PackedTernary, out: torch.Tensor = None) -> PackedTernaryBase3:
    """2-bit packed weights -> the base-3 format (exact; gamma shared)."""
    n = base3_bytes(w.d_out, w.d_in)
    if n == 0:
        _check(ERR_UNSUPPORTED_SHAPE, "repack_base3")
    if out is None:
        out = torch.empty(n, dtype=torch.uint8, device=w.packed.device)
    st = lib().bitlinear_repack_base3(_ptr(w.packed), w.d_out, w.d_in, _ptr(out), _stream())
    _check(st, "bitlinear_repack_base3")
    return PackedTernaryBase3(out, w.gamma, w.d_out, w.d_in)


def packed_words(d_out: int, d_in: int) -> int:
    return int(lib().bitlinear_packed_words(d_out, d_in))


def packed_bytes(d_out: int, d_in: int) -> int:
    return int(lib().bitlinear_packed_bytes(d_out, d_in))


def pack_workspace_bytes(d_out: int, d_in: int) -> int:
    return int(lib().bitlinear_pack_workspace_bytes(d_out, d_in))


def pack_weights(W: torch.Tensor, eps: float = 1e-5, gamma: torch.Tensor = None,
                 out: PackedTernary = None) -> PackedTernary:
    """Absmean-ternarise and pack fp32 latent weights [d_out][d_in]."""
    _need(W, torch.float32, "W")
    d_out, d_in = W.shape
    if out is None:
        n = packed_words(d_out, d_in)
        if n == 0:
            _check(ERR_UNSUPPORTED_SHAPE, "pack_weights")
        out = PackedTernary(torch.empty(n, dtype=torch.int32, device=W.device),
                            torch.empty(1, dtype=torch.float32, device=W.device), d_out, d_in)
    ws = None
    if gamma is None:
        ws = torch.empty(max(pack_workspace_bytes(d_out, d_in), 8), dtype=torch.uint8,
                         device=W.device)
    else:
        _need(gamma, torch.float32, "gamma")
    st = lib().bitlinear_pack_weights(_ptr(W), d_out, d_in, eps, _ptr(gamma), _ptr(ws),
                                      0 if ws is None else ws.numel(), _ptr(out.packed),
                                      _ptr(out.gamma), _stream())
    _check(st, "bitlinear_pack_weights")
    return out


def quant_act(X: torch.Tensor, gain: torch.Tensor = None, rmsnorm: bool = True,
              eps: float = 1e-5, norm_eps: float = 1e-5, inv_rms: torch.Tensor = None,
              per_tensor: bool = False, act_bits: int = 8, outs=None):
    """Fused RMSNorm + absmax int8 codes of bf16 X [T][d_in], with one beta
    per token (default) or one for the whole tensor (per_tensor).

    Returns (Xq int8 [T][d_in], beta f32 [T], rowsum int32 [T], inv_rms f32 [T]),
    inv_rms being the per-token reciprocal RMS used (or given).  ``outs``, if
    given, is that tuple of caller-owned tensors to write instead.
    """
    _need(X, torch.bfloat16, "X")
    T, d_in = X.shape
    dev = X.device
    if outs is not None:
        Xq, beta, rowsum, rms_out = outs
        _need(Xq, torch.int8, "Xq")
        _need(beta, torch.float32, "beta")
        _need(rowsum, torch.int32, "rowsum")
        _need(rms_out, torch.float32, "inv_rms_out")
    else:
        Xq = torch.empty((T, d_in), dtype=torch.int8, device=dev)
        beta = torch.empty(T, dtype=torch.float32, device=dev)
        rowsum = torch.empty(T, dtype=torch.int32, device=dev)
        rms_out = torch.empty(T, dtype=torch.float32, device=dev)
    if gain is not None:
        _need(gain, torch.float32, "gain")
    if inv_rms is not None:
        _need(inv_rms, torch.float32, "inv_rms")
    flags = ((RMSNORM if rmsnorm else 0) | (PER_TENSOR_ABSMAX if per_tensor else 0)
             | (ACT_4BIT if act_bits == 4 else 0))
    st = lib().bitlinear_quant_act(_ptr(X), T, d_in, _ptr(gain), flags,
                                   eps, norm_eps, _ptr(inv_rms), _ptr(Xq), _ptr(beta),
                                   _ptr(rowsum), _ptr(rms_out), _stream())
    _check(st, "bitlinear_quant_act")
    return Xq, beta, rowsum, rms_out


SPLIT_AUTO, SPLIT_ALWAYS, SPLIT_NEVER = 0, 1, 2


def set_decode_split(mode: int) -> None:
    """When decode calls with a split workspace split their units:
    SPLIT_AUTO (default), SPLIT_ALWAYS (tests) or SPLIT_NEVER; process-wide."""
    _check(lib().bitlinear_set_decode_split(mode), "bitlinear_set_decode_split")


DECODE_AUTO, DECODE_WARP_MMA, DECODE_TCGEN05 = 0, 1, 2


def set_decode_kernel(mode: int) -> None:
    """Which product kernel 2-bit decode calls (T <= 16) use: DECODE_AUTO
    (default), DECODE_WARP_MMA or DECODE_TCGEN05; process-wide."""
    _check(lib().bitlinear_set_decode_kernel(mode), "bitlinear_set_decode_kernel")


def decode_workspace_bytes(d_out: int, T: int) -> int:
    """Bytes of the split workspace of a decode product (0 unless 1 <= T <= 16)."""
    return int(lib().bitlinear_decode_workspace_bytes(d_out, T))


def decode_workspace(d_out: int, T: int, device=None):
    """A zero-filled split workspace for decode products with d_out outputs
    and up to T tokens (None when T > 16), on `device` (default: the current
    CUDA device), zeroed on that device's current stream.  The kernels leave
    it zero, so one workspace serves every call on one stream; calls that may
    overlap on the GPU need their own."""
    n = decode_workspace_bytes(d_out, min(max(T, 1), 16)) if T <= 16 else 0
    if n == 0:
        return None
    if device is None:
        device = torch.device("cuda", torch.cuda.current_device())
    return torch.zeros(n, dtype=torch.uint8, device=device)


def _ws_args(workspace):
    if workspace is None:
        return None, 0
    if workspace.device.type != "cuda" or not workspace.is_contiguous():
        raise TypeError("workspace must be a contiguous CUDA tensor")
    return workspace.data_ptr(), workspace.numel() * workspace.element_size()


def forward(w, Xq: torch.Tensor, beta: torch.Tensor, rowsum: torch.Tensor,
            out_dtype=torch.float32, want_acc: bool = False, out: torch.Tensor = None,
            act_bits: int = 8, acc: torch.Tensor = None, workspace: torch.Tensor = None):
    """Y = (X~ W~^T) gamma beta / (Q_b - 1); returns Y (and the int32 acc if
    asked, written to ``acc`` when that tensor is given).  w is a
    PackedTernary, PackedTernaryBase3 or PackedBinary; act_bits (4 or 8, the
    width the codes were made with) applies to PackedBinary.  workspace: an
    optional split workspace (decode_workspace) for T <= 16."""
    _need(Xq, torch.int8, "Xq")
    T = Xq.shape[0]
    dev = Xq.device
    if out is None:
        out = torch.empty((T, w.d_out), dtype=out_dtype, device=dev)
    od = OUT_BF16 if out.dtype == torch.bfloat16 else OUT_F32
    if acc is not None:
        _need(acc, torch.int32, "acc")
        want_acc = True
    elif want_acc:
        acc = torch.empty((T, w.d_out), dtype=torch.int32, device=dev)
    fn, name = _entry(w, "bitlinear_forward")
    wsp, wsn = _ws_args(workspace)
    if isinstance(w, PackedBinary):
        st = fn(_ptr(w.packed), _ptr(w.gamma), w.d_out, w.d_in, _ptr(Xq), _ptr(beta),
                _ptr(rowsum), T, act_bits, _ptr(out), od, _ptr(acc), wsp, wsn, _stream())
    else:
        if act_bits != 8:
            raise ValueError("act_bits != 8 needs binary weights")
        st = fn(_ptr(w.packed), _ptr(w.gamma), w.d_out, w.d_in, _ptr(Xq), _ptr(beta),
                _ptr(rowsum), T, _ptr(out), od, _ptr(acc), wsp, wsn, _stream())
    _check(st, name)
    return (out, acc) if want_acc else out


def linear(w, X: torch.Tensor, gain: torch.Tensor = None, rmsnorm: bool = True,
           eps: float = 1e-5, norm_eps: float = 1e-5, out_dtype=torch.float32,
           out: torch.Tensor = None, scratch=None, static_weights: bool = False,
           per_tensor: bool = False, act_bits: int = 8, inv_rms: torch.Tensor = None,
           workspace: torch.Tensor = None):
    """The whole BitLinear forward from bf16 X: quantise, then product.
    w is a PackedTernary, PackedTernaryBase3 or PackedBinary; act_bits = 4
    (PackedBinary only) makes it the W1A4 forward.

    static_weights: promise that no work still in flight on the stream
    writes w.packed or w.gamma (the product may then stream the weights
    before earlier work has finished).  per_tensor: one activation absmax for
    the whole X instead of one per token.  ``scratch`` = (Xq, beta, rowsum)
    receives the intermediates.  inv_rms: f32 [T] reciprocal RMS to use
    instead of computing it.  workspace: an optional split workspace
    (decode_workspace) for T <= 16.
    """
    _need(X, torch.bfloat16, "X")
    T = X.shape[0]
    dev = X.device
    if scratch is None:
        scratch = (torch.empty((T, w.d_in), dtype=torch.int8, device=dev),
                   torch.empty(T, dtype=torch.float32, device=dev),
                   torch.empty(T, dtype=torch.int32, device=dev))
    Xq, beta, rowsum = scratch
    if out is None:
        out = torch.empty((T, w.d_out), dtype=out_dtype, device=dev)
    od = OUT_BF16 if out.dtype == torch.bfloat16 else OUT_F32
    if gain is not None:
        _need(gain, torch.float32, "gain")
    if inv_rms is not None:
        _need(inv_rms, torch.float32, "inv_rms")
    flags = ((RMSNORM if rmsnorm else 0) | (STATIC_WEIGHTS if static_weights else 0)
             | (PER_TENSOR_ABSMAX if per_tensor else 0) | (ACT_4BIT if act_bits == 4 else 0))
    fn, name = _entry(w, "bitlinear_linear")
    wsp, wsn = _ws_args(workspace)
    st = fn(_ptr(w.packed), _ptr(w.gamma), w.d_out, w.d_in, _ptr(X), T, _ptr(gain), flags, eps,
            norm_eps, _ptr(inv_rms), _ptr(Xq), _ptr(beta), _ptr(rowsum), _ptr(out), od,
            wsp, wsn, _stream())
    _check(st, name)
    return out


class LinearPlan:
    """A bitlinear_linear call bound once (bitlinear_linear_plan_create): the
    weights, the scratch (Xq, beta, rowsum), the output, the flags and the
    CUDA stream (`stream`, default: the one current at construction).  The
    library validates the arguments and prepares the kernel launches at
    construction; each call passes X's address to bitlinear_linear_plan_run
    and returns the bound output tensor (overwritten by the next call).
    2-bit weights (PackedTernary); other formats bind bitlinear_linear_base3
    or bitlinear_linear_w1 each call.  For a serving loop that calls the same
    layer shape repeatedly."""

    def __init__(self, w, T: int, gain: torch.Tensor = None, rmsnorm: bool = True,
                 eps: float = 1e-5, norm_eps: float = 1e-5, out_dtype=torch.bfloat16,
                 out: torch.Tensor = None, scratch=None, static_weights: bool = False,
                 per_tensor: bool = False, device=None, act_bits: int = 8,
                 stream: torch.cuda.Stream = None):
        dev = device if device is not None else w.packed.device
        if scratch is None:
            scratch = (torch.empty((T, w.d_in), dtype=torch.int8, device=dev),
                       torch.empty(T, dtype=torch.float32, device=dev),
                       torch.empty(T, dtype=torch.int32, device=dev))
        if out is None:
            out = torch.empty((T, w.d_out), dtype=out_dtype, device=dev)
        if gain is not None:
            _need(gain, torch.float32, "gain")
        Xq, beta, rowsum = scratch
        _need(Xq, torch.int8, "Xq")
        flags = ((RMSNORM if rmsnorm else 0) | (STATIC_WEIGHTS if static_weights else 0)
                 | (PER_TENSOR_ABSMAX if per_tensor else 0) | (ACT_4BIT if act_bits == 4 else 0))
        od = OUT_BF16 if out.dtype == torch.bfloat16 else OUT_F32
        self.w, self.scratch, self.out, self.gain = w, scratch, out, gain   # keep alive
        self._shape = (T, w.d_in)
        self._stream = stream.cuda_stream if stream is not None else _stream()
        self._handle = None
        if isinstance(w, PackedTernary):
            h = ctypes.c_void_p()
            _check(lib().bitlinear_linear_plan_create(
                w.packed.data_ptr(), w.gamma.data_ptr(), w.d_out, w.d_in, T, _ptr(gain), flags,
                eps, norm_eps, Xq.data_ptr(), beta.data_ptr(), rowsum.data_ptr(), out.data_ptr(),
                od, ctypes.byref(h)), "bitlinear_linear_plan_create")
            self._handle = h
            self._run = lib().bitlinear_linear_plan_run
            self._name = "bitlinear_linear_plan_run"
        else:
            self._fn, self._name = _entry(w, "bitlinear_linear")
            self._pre = (w.packed.data_ptr(), w.gamma.data_ptr(), w.d_out, w.d_in)
            self._ws = decode_workspace(w.d_out, T, dev)   # the plan's own, as in the C plan
            if self._ws is not None and stream is not None:
                # zero-filled on the current stream: runs on `stream` come after it
                stream.wait_stream(torch.cuda.current_stream(self._ws.device))
            wsp, wsn = _ws_args(self._ws)
            self._post = (T, _ptr(gain), flags, eps, norm_eps, None, Xq.data_ptr(),
                          beta.data_ptr(), rowsum.data_ptr(), out.data_ptr(), od, wsp, wsn,
                          self._stream)

    def __call__(self, X: torch.Tensor) -> torch.Tensor:
        if X.dtype != torch.bfloat16 or tuple(X.shape) != self._shape or not X.is_contiguous():
            raise TypeError("X must be a contiguous bf16 tensor of shape %s" % (self._shape,))
        if self._handle is not None:
            st = self._run(self._handle, X.data_ptr(), self._stream)
        else:
            st = self._fn(*self._pre, X.data_ptr(), *self._post)
        if st != OK:
            raise BitLinearError(st, self._name)
        return self.out

    def __del__(self):
        h = getattr(self, "_handle", None)
        if h is not None and _lib is not None:
            _lib.bitlinear_plan_destroy(h)
            self._handle = None


class StepGraph:
    """A serving step captured once as a CUDA graph and replayed per call.

    fn() enqueues the step's work on the current stream: typically a copy of
    the step's inputs from pinned host memory into fixed device buffers, the
    LinearPlan calls of the layers, and a copy of the outputs back to pinned
    host memory.  Every address it uses must stay valid and fixed; a replay
    re-runs the same kernels and copies (the host buffers' current contents
    go in, the new outputs come out).  fn is captured on `stream` (default:
    a new stream), so LinearPlans called inside it must be bound to that
    stream; it runs once eagerly on the same stream before the capture."""

    def __init__(self, fn, stream: torch.cuda.Stream = None):
        self.stream = stream if stream is not None else torch.cuda.Stream()
        self.stream.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(self.stream):
            fn()
        torch.cuda.synchronize()
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph, stream=self.stream):
            fn()
        torch.cuda.synchronize()

    def __call__(self):
        self.graph.replay()


def backward(w: PackedTernary, Xq: torch.Tensor, beta: torch.Tensor, dY: torch.Tensor,
             want_dx: bool = True, want_dw: bool = True, out_dtype=torch.float32,
             workspace: torch.Tensor = None):
    """Straight-through-estimator gradients of the forward ([MF] §3):
    returns (dX [T][d_in], dW [d_out][d_in]), None for the one not asked for."""
    _need(dY, torch.bfloat16, "dY")
    T = dY.shape[0]
    dev = dY.device
    if want_dw:
        _need(Xq, torch.int8, "Xq")
        _need(beta, torch.float32, "beta")
    nbytes = int(lib().bitlinear_backward_workspace_bytes(w.d_out, w.d_in, T, int(want_dx),
                                                          int(want_dw)))
    if workspace is None:
        workspace = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=dev)
    dX = torch.empty((T, w.d_in), dtype=out_dtype, device=dev) if want_dx else None
    dW = torch.empty((w.d_out, w.d_in), dtype=out_dtype, device=dev) if want_dw else None
    od = OUT_BF16 if out_dtype == torch.bfloat16 else OUT_F32
    _check(lib().bitlinear_backward(_ptr(w.packed), _ptr(w.gamma), w.d_out, w.d_in,
                                    _ptr(Xq) if want_dw else None,
                                    _ptr(beta) if want_dw else None, T, _ptr(dY), _ptr(dX),
                                    _ptr(dW), od, _ptr(workspace), workspace.numel(), _stream()),
           "bitlinear_backward")
    return dX, dW


def dense_bf16_forward(W: torch.Tensor, X: torch.Tensor, out_dtype=torch.bfloat16,
                       out: torch.Tensor = None) -> torch.Tensor:
    """The dense bf16 layer Y = X W^T the ternary path replaces (context)."""
    _need(W, torch.bfloat16, "W")
    _need(X, torch.bfloat16, "X")
    d_out, d_in = W.shape
    T = X.shape[0]
    if X.shape[1] != d_in:
        raise ValueError("X must be [T][d_in]")
    if out is None:
        out = torch.empty((T, d_out), dtype=out_dtype, device=X.device)
    od = OUT_BF16 if out.dtype == torch.bfloat16 else OUT_F32
    _check(lib().bitlinear_dense_bf16_forward(_ptr(W), d_out, d_in, _ptr(X), T, _ptr(out), od,
                                              _stream()),
           "bitlinear_dense_bf16_forward")
    return out


def device_error(clear: bool = True) -> int:
    """Synchronise the current stream and return the device error status."""
    return int(lib().bitlinear_device_error(_stream(), 1 if clear else 0))


def get_last_device_error() -> int:
    """Synchronise the current stream, return the device error status, clear it."""
    return int(lib().bitlinear_get_last_device_error(_stream()))


def set_wait_limit_ns(limit_ns: int):
    _check(lib().bitlinear_set_wait_limit_ns(int(limit_ns)), "bitlinear_set_wait_limit_ns")


def wait_probe(limit_ns: int):
    _check(lib().bitlinear_wait_probe(int(limit_ns), _stream()), "bitlinear_wait_probe")
