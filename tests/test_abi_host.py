"""Host-side checks of the C ABI: no GPU needed, no kernel launched.

The library must load, export every entry point the header declares, and
reject bad arguments on the host before touching a device.
"""
import ctypes
import os
import re
import subprocess

import pytest
import torch

import ternary_weight_linear_bitlinear_b200 as bl
from ternary_weight_linear_bitlinear_b200 import build as blbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "bitlinear.h")


@pytest.fixture(scope="module")
def lib():
    blbuild.build()
    return bl.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(bitlinear_\w+)\s*\(", text)))


def test_header_declares_entry_points():
    names = declared_functions()
    for must in ("bitlinear_pack_weights", "bitlinear_quant_act", "bitlinear_forward"):
        assert must in names
    assert set(names) == set(bl.SIGNATURES), "binding and header disagree"


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", bl.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (bitlinear_\w+)$", out, flags=re.M))
    missing = set(declared_functions()) - exported
    assert not missing, missing
    for name in declared_functions():
        assert getattr(lib, name) is not None


def test_version_and_status_strings(lib):
    assert lib.bitlinear_version() == 3
    for code in range(0, 7):
        s = bl.status_string(code)
        assert s and s != "unknown status"
    assert bl.status_string(99) == "unknown status"


def test_packed_sizes(lib):
    assert bl.packed_words(6912, 2560) == 6912 * 2560 // 16
    assert bl.packed_words(11008, 4096) * 4 == 11272192
    assert bl.packed_words(4096, 11008) * 4 == 11272192
    assert bl.packed_words(16, 256) == 256
    assert bl.packed_words(15, 256) == 0          # d_out not a multiple of 16
    assert bl.packed_words(16, 128) == 0          # d_in not a multiple of 256
    assert bl.packed_words(16, 65536 + 256) == 0  # d_in too large
    # byte count of the scope table's boundary: 0.25 byte per weight
    assert bl.packed_bytes(6912, 2560) == 4423680
    assert bl.packed_bytes(8192, 28672) == 58720256
    assert bl.packed_bytes(15, 256) == 0
    assert bl.pack_workspace_bytes(6912, 2560) > 0
    assert bl.pack_workspace_bytes(16, 100) == 0


P = ctypes.c_void_p
S0 = ctypes.c_void_p(0)


def _fwd(lib, packed=0x10000, gamma=0x20000, d_out=64, d_in=256, xq=0x30000, beta=0x40000,
         rowsum=0x50000, T=4, Y=0x60000, od=0, acc=None, ws=None, ws_bytes=0):
    return lib.bitlinear_forward(P(packed), P(gamma), d_out, d_in, P(xq), P(beta), P(rowsum), T,
                                 P(Y), od, P(acc) if acc else None, P(ws) if ws else None,
                                 ws_bytes, S0)


def test_forward_validation(lib):
    assert _fwd(lib, packed=0) == bl.ERR_INVALID_ARG
    assert _fwd(lib, Y=0) == bl.ERR_INVALID_ARG
    assert _fwd(lib, d_in=200) == bl.ERR_UNSUPPORTED_SHAPE
    assert _fwd(lib, d_out=24) == bl.ERR_UNSUPPORTED_SHAPE
    assert _fwd(lib, T=-1) == bl.ERR_UNSUPPORTED_SHAPE
    assert _fwd(lib, od=7) == bl.ERR_INVALID_ARG
    assert _fwd(lib, packed=0x10008) == bl.ERR_MISALIGNED
    assert _fwd(lib, Y=0x60004) == bl.ERR_MISALIGNED
    assert _fwd(lib, xq=0x30001) == bl.ERR_MISALIGNED
    assert _fwd(lib, beta=0x40002) == bl.ERR_MISALIGNED
    # T = 0 is an empty problem: success, nothing enqueued, no device touched.
    assert _fwd(lib, T=0, xq=0, beta=0, rowsum=0) == bl.OK


def test_decode_workspace_rules(lib):
    """The split workspace: one 8-byte word per token and row of d_out plus a
    spare 16-row tile, rounded up to 128 rows, the total to 256 bytes; only
    for 1 <= T <= 16; a workspace that is too small or misaligned is refused
    before anything is enqueued."""
    nb = lib.bitlinear_decode_workspace_bytes
    for d_out, T in ((64, 4), (28672, 1), (28672, 16), (6912, 8), (16, 1), (6928, 3)):
        n_rt = d_out // 16
        rows = (16 * (n_rt + 1) + 127) // 128 * 128
        want = (8 * rows * T + 255) // 256 * 256
        assert nb(d_out, T) == want
        assert bl.decode_workspace_bytes(d_out, T) == nb(d_out, T)
    assert nb(64, 0) == 0 and nb(64, 17) == 0 and nb(24, 4) == 0 and nb(0, 4) == 0
    need = nb(64, 4)
    assert _fwd(lib, ws=0x70000, ws_bytes=need - 1) == bl.ERR_INVALID_ARG
    assert _fwd(lib, ws=0x70008, ws_bytes=need) == bl.ERR_MISALIGNED
    # T > 16 ignores the workspace's size (the prefill GEMM does not use it).
    if not torch.cuda.is_available():
        assert _fwd(lib, ws=0x70000, ws_bytes=need) == bl.ERR_DEVICE
    lin = lib.bitlinear_linear
    args = (P(0x10000), P(0x20000), 64, 256, P(0x30000), 4, None, 1, 1e-5, 1e-5, None,
            P(0x40000), P(0x50000), P(0x60000), P(0x80000), 0)
    assert lin(*args, P(0x70000), need - 4, S0) == bl.ERR_INVALID_ARG
    assert lin(*args, P(0x70004), need, S0) == bl.ERR_MISALIGNED
    assert lib.bitlinear_set_decode_split(3) == bl.ERR_INVALID_ARG
    assert lib.bitlinear_set_decode_split(-1) == bl.ERR_INVALID_ARG
    for mode in (bl.SPLIT_NEVER, bl.SPLIT_ALWAYS, bl.SPLIT_AUTO):
        assert lib.bitlinear_set_decode_split(mode) == bl.OK
    assert lib.bitlinear_set_decode_kernel(3) == bl.ERR_INVALID_ARG
    for mode in (bl.DECODE_WARP_MMA, bl.DECODE_TCGEN05, bl.DECODE_AUTO):
        assert lib.bitlinear_set_decode_kernel(mode) == bl.OK


def test_base3_sizes_and_validation(lib):
    """Five codes per byte on rows padded to 160 columns; base-3 entry points
    take 1 <= T <= 16 and validate like their 2-bit counterparts."""
    assert bl.base3_bytes(6912, 2560) == 6912 * 2560 // 5          # 2560 = 16 x 160
    assert bl.base3_bytes(28672, 8192) == 28672 * 8320 // 5        # 8192 -> 8320 columns
    assert bl.base3_bytes(16, 256) == 16 * 320 // 5
    assert bl.base3_bytes(15, 256) == 0 and bl.base3_bytes(16, 128) == 0
    f = lib.bitlinear_forward_base3

    def fwd(T=4, packed=0x10000, d_in=256, xq=0x30000):
        return f(P(packed), P(0x20000), 64, d_in, P(xq), P(0x40000), P(0x50000), T, P(0x60000),
                 0, None, None, 0, S0)

    assert fwd(T=17) == bl.ERR_UNSUPPORTED_SHAPE
    assert fwd(d_in=200) == bl.ERR_UNSUPPORTED_SHAPE
    assert fwd(packed=0) == bl.ERR_INVALID_ARG
    assert fwd(packed=0x10008) == bl.ERR_MISALIGNED
    assert fwd(T=0, xq=0) == bl.OK
    lin = lib.bitlinear_linear_base3
    assert lin(P(0x10000), P(0x20000), 64, 256, P(0x30000), 17, None, 1, 1e-5, 1e-5, None,
               P(0x40000), P(0x50000), P(0x60000), P(0x70000), 0, None, 0,
               S0) == bl.ERR_UNSUPPORTED_SHAPE
    assert lin(P(0x10000), P(0x20000), 64, 256, P(0x30000), 4, None, 8, 1e-5, 1e-5, None,
               P(0x40000), P(0x50000), P(0x60000), P(0x70000), 0, None, 0,
               S0) == bl.ERR_INVALID_ARG
    rp = lib.bitlinear_repack_base3
    assert rp(P(0x10000), 16, 128, P(0x20000), S0) == bl.ERR_UNSUPPORTED_SHAPE
    assert rp(P(0x10000), 16, 256, None, S0) == bl.ERR_INVALID_ARG
    assert rp(P(0x10000), 16, 256, P(0x20008), S0) == bl.ERR_MISALIGNED


def test_w1_sizes_and_validation(lib):
    """One bit per weight on rows padded to 512 columns; the W1 entry points
    take 1 <= T <= 16, act_bits 4 or 8, and the 4-bit flag only with binary
    weights."""
    assert bl.w1_packed_bytes(6912, 2560) == 6912 * 2560 // 8
    assert bl.w1_packed_bytes(4096, 11008) == 4096 * 11264 // 8
    assert bl.w1_packed_bytes(16, 256) == 16 * 512 // 8
    assert bl.w1_packed_bytes(15, 256) == 0
    f = lib.bitlinear_forward_w1

    def fwd(T=4, bits=4, d_in=256, packed=0x10000):
        return f(P(packed), P(0x20000), 64, d_in, P(0x30000), P(0x40000), P(0x50000), T, bits,
                 P(0x60000), 0, None, None, 0, S0)

    assert fwd(T=17) == bl.ERR_UNSUPPORTED_SHAPE
    assert fwd(bits=5) == bl.ERR_INVALID_ARG
    assert fwd(d_in=384) == bl.ERR_UNSUPPORTED_SHAPE
    assert fwd(packed=0x10004) == bl.ERR_MISALIGNED
    assert fwd(T=0) == bl.OK
    args = (P(0x10000), P(0x20000), 64, 256, P(0x30000), 4, None)
    tail = (1e-5, 1e-5, None, P(0x40000), P(0x50000), P(0x60000), P(0x70000), 0, None, 0, S0)
    assert lib.bitlinear_linear(*args, 1 | bl.ACT_4BIT, *tail) == bl.ERR_INVALID_ARG
    assert lib.bitlinear_linear_w1(*args, 16, *tail) == bl.ERR_INVALID_ARG
    # A supplied reciprocal RMS must be 4-byte aligned.
    tail_r = (1e-5, 1e-5, P(0x80002), P(0x40000), P(0x50000), P(0x60000), P(0x70000), 0, None, 0,
              S0)
    assert lib.bitlinear_linear(*args, 1, *tail_r) == bl.ERR_MISALIGNED
    pk = lib.bitlinear_pack_weights_w1
    assert pk(P(0x10000), 16, 128, None, P(0x20000), 1 << 20, P(0x30000), P(0x40000),
              S0) == bl.ERR_UNSUPPORTED_SHAPE
    assert pk(P(0x10000), 16, 256, None, None, 0, P(0x30000), P(0x40000),
              S0) == bl.ERR_INVALID_ARG
    assert pk(P(0x10000), 16, 256, None, P(0x20000), 1 << 20, P(0x30008), P(0x40000),
              S0) == bl.ERR_MISALIGNED


def test_quant_act_validation(lib):
    q = lib.bitlinear_quant_act
    args = dict(X=0x10000, T=2, d_in=512, gain=None, flags=1, eps=1e-5, neps=1e-5, rms=None,
                xq=0x20000, beta=0x30000, rs=0x40000, rmso=None)

    def call(**kw):
        a = dict(args, **kw)
        return q(P(a["X"]), a["T"], a["d_in"], P(a["gain"]) if a["gain"] else None, a["flags"],
                 a["eps"], a["neps"], P(a["rms"]) if a["rms"] else None, P(a["xq"]),
                 P(a["beta"]), P(a["rs"]), P(a["rmso"]) if a["rmso"] else None, S0)

    assert call(X=0) == bl.ERR_INVALID_ARG
    assert call(flags=16) == bl.ERR_INVALID_ARG                    # no such flag
    assert call(flags=1 | bl.ACT_4BIT) != bl.ERR_INVALID_ARG        # 4-bit codes
    assert call(flags=2) == bl.ERR_INVALID_ARG                     # bitlinear_linear's only
    assert call(flags=1 | bl.PER_TENSOR_ABSMAX) != bl.ERR_INVALID_ARG
    assert call(eps=float("nan")) == bl.ERR_INVALID_ARG
    assert call(neps=-1.0) == bl.ERR_INVALID_ARG
    assert call(d_in=300) == bl.ERR_UNSUPPORTED_SHAPE
    assert call(X=0x10002) == bl.ERR_MISALIGNED
    assert call(gain=0x50001) == bl.ERR_MISALIGNED
    assert call(T=0, X=0, xq=0) == bl.OK


def test_pack_validation(lib):
    p = lib.bitlinear_pack_weights
    ws = bl.pack_workspace_bytes(64, 256)
    assert p(None, 64, 256, 1e-5, None, P(0x1000), ws, P(0x2000), P(0x3000), S0) == bl.ERR_INVALID_ARG
    assert p(P(0x1000), 64, 100, 1e-5, None, P(0x1000), ws, P(0x2000), P(0x3000), S0) == bl.ERR_UNSUPPORTED_SHAPE
    assert p(P(0x1000), 64, 256, -1.0, None, P(0x1000), ws, P(0x2000), P(0x3000), S0) == bl.ERR_INVALID_ARG
    # Computing gamma needs a large enough workspace.
    assert p(P(0x1000), 64, 256, 1e-5, None, None, 0, P(0x2000), P(0x3000), S0) == bl.ERR_INVALID_ARG
    assert p(P(0x1000), 64, 256, 1e-5, None, P(0x1000), ws - 8, P(0x2000), P(0x3000), S0) == bl.ERR_INVALID_ARG
    assert p(P(0x1004), 64, 256, 1e-5, None, P(0x1000), ws, P(0x2000), P(0x3000), S0) == bl.ERR_MISALIGNED


def test_wait_limit_validation(lib):
    assert lib.bitlinear_set_wait_limit_ns(10) == bl.ERR_INVALID_ARG
    assert lib.bitlinear_wait_probe(10, S0) == bl.ERR_INVALID_ARG


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device path")
def test_no_device_fails_loudly(lib):
    """Without an sm_100 GPU a valid compute call reports ERR_DEVICE: there
    is no CPU fallback behind the C ABI."""
    assert _fwd(lib) == bl.ERR_DEVICE
    with pytest.raises((RuntimeError, TypeError)):
        bl.quant_act(torch.zeros(2, 256, dtype=torch.bfloat16))


def test_plan_validation(lib):
    """bitlinear_linear_plan_create checks the bound arguments like
    bitlinear_linear, before it looks at the device."""
    import ctypes as C
    h = C.c_void_p()
    mk = lib.bitlinear_linear_plan_create

    def create(d_in=256, T=4, flags=1, xq=0x30000, plan=True):
        return mk(P(0x10000), P(0x20000), 64, d_in, T, None, flags, 1e-5, 1e-5, P(xq),
                  P(0x40000), P(0x50000), P(0x60000), 0, C.byref(h) if plan else None)

    assert create(plan=False) == bl.ERR_INVALID_ARG
    assert create(d_in=300) == bl.ERR_UNSUPPORTED_SHAPE
    assert create(flags=bl.ACT_4BIT | 1) == bl.ERR_INVALID_ARG      # 2-bit weights only
    assert create(xq=0x30001) == bl.ERR_MISALIGNED
    assert lib.bitlinear_linear_plan_run(None, P(0x1000), S0) == bl.ERR_INVALID_ARG
    lib.bitlinear_plan_destroy(None)
    if not torch.cuda.is_available():
        assert create() == bl.ERR_DEVICE
        assert h.value is None
