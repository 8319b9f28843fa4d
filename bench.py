"""Benchmark of the BitLinear forward hot path on B200.

Prints ONE JSON line on rank 0.

Headline (decode): the single-token 2560 -> 6912 BitLinear forward (fused
RMSNorm + absmax int8 quantiser, then the ternary GEMV with the fused
rescale), reported as achieved HBM GB/s of algorithmic bytes.  One step is a
stack of ``LAYERS`` such forwards over distinct packed weight copies (the
projections of consecutive layers of one decode step), so each step streams
more packed weight bytes than the L2 holds and every weight byte comes from
HBM.  Steps are captured in a CUDA graph and timed with CUDA events.

Also in the line: the prefill forward (2048 tokens, 4096 -> 11008, bf16
out) as int8 tensor TOPS, the transformer-block and large decode
workloads, the roofline of the dominant kernel, the CPU oracle baseline,
an end-to-end number through the public API with host buffers, and SM
clocks sampled during the timed region.

``--impl reference`` times the CPU oracle instead (the reference arm).
Multi-GPU (torchrun): independent replicas, one per GPU, no collective on
the data path; time is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from workloads import ALL as WORKLOADS, Problem, bf16_bits, draw  # noqa: E402

METRIC = "decode GEMV achieved HBM GB/s (% of peak); prefill int8 TOPS (% of peak)"
HEADLINE = "decode_gemv_2560x6912_t1"
LAYERS = 64
L2_BYTES = 126 * 2 ** 20
EPS = 1e-5


# ----------------------------------------------------------------- peaks ---

def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        p = json.load(open(path))
        return dict(hbm=float(p["hbm_gbs"]), bf16=float(p["bf16_tflops"]),
                    bf16_sustained=float(p["bf16_tflops_sustained"]), source="measured")
    except Exception:
        return dict(hbm=6650.0, bf16=1590.0, bf16_sustained=1400.0, source="fallback")


# Dense int8 tensor throughput relative to dense bf16: NVIDIA's B200 figures
# (4.5 POPS int8 / 2.25 PFLOPS bf16, dense).
INT8_OVER_BF16 = 2.0


# ---------------------------------------------------------------- clocks ---

class ClockSampler:
    """nvidia-smi SM clock / throttle-reason sampler for the timed region."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = str(index)
        try:
            u = str(torch.cuda.get_device_properties(index).uuid)
            self.index = u if u.startswith("GPU-") else "GPU-" + u
        except Exception:
            pass
        self.proc = None
        self.lines = []
        self.marks = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.index, "--query-gpu=" + self.QUERY,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self._t = threading.Thread(target=self._read, daemon=True)
            self._t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def mark(self, on: bool):
        self.marks.append((time.time(), on))

    def stop(self):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        if not self.lines:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"],
                    "samples": 0}
        windows = []
        for i in range(0, len(self.marks) - 1, 2):
            windows.append((self.marks[i][0], self.marks[i + 1][0]))

        def inside(t):
            return any(a - 0.15 <= t <= b + 0.15 for a, b in windows)

        rows = []
        for t, line in self.lines:
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            rows.append((t, f))
        sel = [f for t, f in rows if inside(t)] or [f for _, f in rows]
        mhz = [float(f[1]) for f in sel if f[1].replace(".", "").isdigit()]
        mx = [float(f[2]) for f in sel if f[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for f in sel for i in range(4)
                          if f[5 + i].lower().startswith("active")})
        return {"sm_mhz": statistics.median(mhz) if mhz else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(sel)}


# ------------------------------------------------------- distributed ---

def dist_init(n_gpus, timeout_s: float = 120.0):
    """One process per GPU (torchrun sets RANK / WORLD_SIZE / LOCAL_RANK).
    NCCL where GPUs are visible; gloo on a host without them (the CPU
    reference arm, the host-side tests).  The short timeout makes ranks
    that wait on a departed peer end with an error instead of hanging."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        timeout = datetime.timedelta(seconds=timeout_s)
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=timeout,
                                    device_id=torch.device("cuda", local))
        else:
            dist.init_process_group("gloo", timeout=timeout)
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world) -> float:
    """Max of a per-rank time over all ranks (the slowest replica sets the job time)."""
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_value(bytes_per_step: float, world: int, ms_step: float) -> float:
    """Whole-job GB/s of independent replicas: every rank moves bytes_per_step
    per step, and the job's step time is the slowest rank's."""
    return bytes_per_step * world / (ms_step * 1e-3) / 1e9


# ------------------------------------------------------------ helpers ---

FUSED_MAX_CODE_BYTES = 32768   # bitlinear_linear fuses quantiser + GEMV up to T*d_in


def fused(p: Problem) -> bool:
    return p.tokens <= 8 and p.tokens * p.d_in <= FUSED_MAX_CODE_BYTES


def decode_bytes(p: Problem, out_bytes: int = 2, fmt: str = "2bit") -> dict:
    """Algorithmic bytes of one decode BitLinear forward (quantise + product).

    Fused (one kernel): packed W + bf16 X read + codes, beta, row sums written
    once + gamma + Y.  Two kernels: the codes, beta and row sums are also read
    back once by the product.  fmt: "2bit" (four codes per byte), "base3" (five
    codes per byte on rows padded to 160 columns) or "w1" (one bit per weight
    on rows padded to 512 columns)."""
    T, K, N = p.tokens, p.d_in, p.d_out
    if fmt == "base3":
        w = N * ((K + 159) // 160 * 160) // 5
    elif fmt == "w1":
        w = N * ((K + 511) // 512 * 512) // 8
    else:
        w = N * K // 4
    x = T * K * 2                    # bf16 activations
    inter = T * K + 8 * T            # codes, beta, row sums written
    y = T * N * out_bytes
    step = w + x + inter + 4 + y + (0 if fused(p) else inter)
    return dict(step=step, gemv=w + inter + 4 + y, weights=w, weights_and_acts=w + x + y)


def time_graph(g: torch.cuda.CUDAGraph, reps: int = 1) -> float:
    """Milliseconds of `reps` replays of g, CUDA events on the current stream."""
    s = torch.cuda.current_stream()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    a.record(s)
    for _ in range(reps):
        g.replay()
    b.record(s)
    b.synchronize()
    return a.elapsed_time(b)


def capture(fn):
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()  # one eager call on the side stream before capture
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    with torch.cuda.graph(g):
        fn()
    torch.cuda.synchronize()
    return g


DECODE_SOURCES = ("gemv.cu", "quant_common.cuh", "common.cuh", "decode_common.cuh")
GEMM_SOURCES = ("gemm_tc.cu", "common.cuh", "tc_common.cuh")


def source_sha(names):
    """First 16 hex digits of the SHA-256 of the named kernel sources, concatenated."""
    h = hashlib.sha256()
    for name in names:
        with open(os.path.join(ROOT, "ternary_weight_linear_bitlinear_b200", "csrc", name),
                  "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profile_traffic(summary_name: str, source):
    """DRAM bytes per launch from a committed ncu summary, or None when the
    summary was taken on a different version of the kernel sources."""
    path = os.path.join(ROOT, "profiles", summary_name)
    try:
        text = open(path).read()
    except OSError:
        return None
    m_sha = re.search(r"source_sha256_16:\s*([0-9a-f]+)", text)
    m_b = re.search(r"dram_bytes_per_launch:\s*([0-9.eE+]+)", text)
    if not m_sha or not m_b or m_sha.group(1) != source_sha(source):
        return None
    return float(m_b.group(1))


# ------------------------------------------------------ decode workload ---

class DecodeRun:
    """`layers` forwards per step over distinct packed weight copies."""

    def __init__(self, problems, layers, dev, out_dtype=torch.bfloat16, fmt="2bit"):
        import ternary_weight_linear_bitlinear_b200 as bl
        self.bl = bl
        self.fmt = fmt
        self.act_bits = 4 if fmt == "w1" else 8     # the W1A4 regime
        self.problems = problems
        self.dev = dev
        self.out_dtype = out_dtype
        self.layers = []      # (problem, PackedTernary, X, scratch, Y, split workspace)
        base = []
        for p in problems:
            W, X = draw(p)
            if fmt == "w1":
                w = bl.pack_weights_w1(W.to(dev))
            else:
                w = bl.pack_weights(W.to(dev), EPS)
            if fmt == "base3":
                w = bl.repack_base3(w)
            base.append((p, w, X.to(dev)))
            del W
        reps = max(1, layers // len(problems))
        for r in range(reps):
            for p, w0, X in base:
                if r == 0:
                    w = w0
                else:
                    w = type(w0)(w0.packed.clone(), w0.gamma.clone(), w0.d_out, w0.d_in)
                T = p.tokens
                scratch = (torch.empty((T, p.d_in), dtype=torch.int8, device=dev),
                           torch.empty(T, dtype=torch.float32, device=dev),
                           torch.empty(T, dtype=torch.int32, device=dev))
                Y = torch.empty((T, p.d_out), dtype=out_dtype, device=dev)
                ws = bl.decode_workspace(p.d_out, T, dev)
                self.layers.append((p, w, X, scratch, Y, ws))
        torch.cuda.synchronize()
        # Pre-quantised activations for the product-only timing.
        for p, w, X, scratch, Y, _ in self.layers:
            xq, beta, rowsum, _ = bl.quant_act(X, act_bits=self.act_bits)
            scratch[0].copy_(xq)
            scratch[1].copy_(beta)
            scratch[2].copy_(rowsum)
        torch.cuda.synchronize()

    def step(self):
        for p, w, X, scratch, Y, ws in self.layers:
            self.bl.linear(w, X, out=Y, scratch=scratch, static_weights=True,
                           act_bits=self.act_bits, workspace=ws)

    def product_only(self):
        for p, w, X, scratch, Y, ws in self.layers:
            self.bl.forward(w, scratch[0], scratch[1], scratch[2], out=Y, act_bits=self.act_bits,
                            workspace=ws)

    def bytes(self):
        ob = 2 if self.out_dtype == torch.bfloat16 else 4
        tot = dict(step=0, gemv=0, weights=0, weights_and_acts=0)
        for p, *_ in self.layers:
            for k, v in decode_bytes(p, ob, self.fmt).items():
                tot[k] += v
        return tot

    def weight_bytes_resident(self):
        return sum(w.packed.numel() * w.packed.element_size() for _, w, *_ in self.layers)


def run_decode(name, steps, warmup, dev, layers, world):
    wl = WORKLOADS[name]
    run = DecodeRun(wl.problems, layers, dev)
    nb = run.bytes()
    for _ in range(max(warmup, 3)):
        run.step()
    torch.cuda.synchronize()

    def k_steps(k):
        def f():
            for _ in range(k):
                run.step()
        return f

    g_warm = capture(k_steps(max(warmup, 3)))
    g_timed = capture(k_steps(steps))
    time_graph(g_warm)
    time_graph(g_timed)              # untimed pass: graph upload
    barrier(world)
    return run, nb, g_timed


def measure_product_only(run, steps):
    g = capture(lambda: [run.product_only() for _ in range(steps)])
    time_graph(g)
    ms = time_graph(g)
    launches = steps * len(run.layers)
    return ms / launches, launches


def measure_formats(dev, peaks, reps=5, workloads=None):
    """The base-3 weight format (five codes per byte) and the W1A4 regime
    (one bit per weight, 4-bit activation codes) against the 2-bit ternary
    format on the decode workloads, each over distinct weight copies of at
    least 4x the L2: microseconds per forward of the whole fused forward and of
    the product alone (codes precomputed), and the GB/s of each format's own
    bytes."""
    out = {}
    for name in workloads or ("decode_gemv_2560x6912_t1", "decode_block_4096_t1",
                              "large_gemv_8192x28672_t1", "large_gemv_8192x28672_t8"):
        wl = WORKLOADS[name]
        res = {}
        for fmt in ("2bit", "base3", "w1"):
            per = sum(decode_bytes(p, fmt=fmt)["weights"] for p in wl.problems)
            layers = max(len(wl.problems), int(np.ceil(4 * L2_BYTES / per)) * len(wl.problems))
            r = DecodeRun(wl.problems, layers, dev, fmt=fmt)
            g = capture(lambda: [r.step() for _ in range(reps)])
            time_graph(g)
            t = time_graph(g) / reps / len(r.layers)
            gp = capture(lambda: [r.product_only() for _ in range(reps)])
            time_graph(gp)
            tp = time_graph(gp) / reps / len(r.layers)
            b = r.bytes()
            n = len(r.layers)
            res[fmt] = {"us_per_forward": round(t * 1e3, 3),
                        "gbs_forward": round(b["step"] / n / (t * 1e-3) / 1e9, 1),
                        "us_product_only": round(tp * 1e3, 3),
                        "gbs_product_only": round(b["gemv"] / n / (tp * 1e-3) / 1e9, 1),
                        "frac_of_hbm_product_only": round(
                            b["gemv"] / n / (tp * 1e-3) / 1e9 / peaks["hbm"], 4),
                        "weight_bytes_per_forward": b["weights"] // n}
            del r, g, gp
            torch.cuda.empty_cache()
        for fmt in ("base3", "w1"):
            res[fmt]["speedup_forward_vs_2bit"] = round(res["2bit"]["us_per_forward"] /
                                                        res[fmt]["us_per_forward"], 3)
            res[fmt]["speedup_product_vs_2bit"] = round(res["2bit"]["us_product_only"] /
                                                        res[fmt]["us_product_only"], 3)
        out[name] = res
    return out


# ----------------------------------------------------- prefill workload ---

def time_each(fn, iters, flush):
    """Mean device time (ms) of fn(), each call timed alone with CUDA events
    after the L2 has been overwritten (outside the timed window)."""
    s = torch.cuda.current_stream()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(iters)]
    for a, b in evs:
        flush.zero_()
        a.record(s)
        fn()
        b.record(s)
    torch.cuda.synchronize()
    return sum(a.elapsed_time(b) for a, b in evs) / iters


def measure_prefill(steps, warmup, dev, peaks):
    """The prefill working set (~65 MB) fits in L2, so every timed call
    follows an L2 flush (a 2x L2 write) and is timed on its own."""
    import ternary_weight_linear_bitlinear_b200 as bl
    p = WORKLOADS["prefill_2048x4096x11008"].problems[0]
    W, X = draw(p)
    w = bl.pack_weights(W.to(dev), EPS)
    del W
    Xd = X.to(dev)
    T = p.tokens
    scratch = (torch.empty((T, p.d_in), dtype=torch.int8, device=dev),
               torch.empty(T, dtype=torch.float32, device=dev),
               torch.empty(T, dtype=torch.int32, device=dev))
    Y = torch.empty((T, p.d_out), dtype=torch.bfloat16, device=dev)
    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev)
    for _ in range(max(warmup, 3)):
        bl.linear(w, Xd, out=Y, scratch=scratch)
    torch.cuda.synchronize()
    ms_step = time_each(lambda: bl.linear(w, Xd, out=Y, scratch=scratch), steps, flush)
    ms_step_pt = time_each(lambda: bl.linear(w, Xd, out=Y, scratch=scratch, per_tensor=True),
                           steps, flush)
    ms_mm = time_each(lambda: bl.forward(w, scratch[0], scratch[1], scratch[2], out=Y), steps,
                      flush)
    # Context, not this library's path: the vendor int8 GEMM (cuBLASLt, through
    # torch._int_mm) on the same shape, int8 x int8 -> int32 with the weights
    # stored unpacked -- what this GPU's tensor cores reach on the contraction
    # alone under the same timing.
    vendor = None
    try:
        g = torch.Generator().manual_seed(5)
        w8 = torch.randint(-1, 2, (p.d_out, p.d_in), dtype=torch.int8, generator=g).to(dev)
        for _ in range(max(warmup, 3)):   # the library picks and sets up its kernel on first use
            torch._int_mm(scratch[0], w8.t())
        torch.cuda.synchronize()
        ms_lib = time_each(lambda: torch._int_mm(scratch[0], w8.t()), steps, flush)
        del w8
        vendor = {"impl": "cuBLASLt via torch._int_mm (int8 x int8 -> int32, unpacked weights)",
                  "ms": round(ms_lib, 4), "tops": None, "ours_over_vendor": None}
    except Exception as e:   # context only: its absence must not cost the measurement
        vendor = {"impl": "cuBLASLt via torch._int_mm", "unavailable": repr(e)[:200]}
    del flush
    ops = 2.0 * T * p.d_in * p.d_out
    tops = ops / (ms_mm * 1e-3) / 1e12
    if vendor.get("ms"):
        vendor["tops"] = round(ops / (vendor["ms"] * 1e-3) / 1e12, 1)
        vendor["ours_over_vendor"] = round(vendor["ms"] / ms_mm, 3)
    peak = peaks["bf16"] * INT8_OVER_BF16
    return {
        "workload": WORKLOADS["prefill_2048x4096x11008"].name,
        "tops_gemm": round(tops, 1), "unit": "TOPS (int8, 2 ops per MAC)",
        "ms_gemm": round(ms_mm, 4), "ms_step_with_quant": round(ms_step, 4),
        "tops_step": round(ops / (ms_step * 1e-3) / 1e12, 1),
        "ms_step_per_tensor_absmax": round(ms_step_pt, 4),
        "roofline": {"bound": "tensor", "achieved": round(tops, 1), "peak": round(peak, 1),
                     "unit": "TFLOP/s", "frac": round(tops / peak, 4),
                     "traffic": profile_traffic("gemm_tc_pair_prefill_2048x4096x11008.md",
                                                GEMM_SOURCES),
                     "peak_source": "%s bf16 burst x %.0f (nominal int8/bf16 dense ratio)"
                                    % (peaks["source"], INT8_OVER_BF16)},
        "frac_of_datasheet_4500": round(tops / 4500.0, 4),
        "vendor_int8_gemm_same_shape": vendor,
        "l2": "L2 overwritten before every timed call; each call timed alone",
        "gpu_launches": 7 * steps,
    }


# ------------------------------------------------------------ backward ---

def measure_backward(steps, dev, peaks):
    """The straight-through-estimator backward at the prefill shape (dX and
    dW: the bf16 expansion of W~ and dequantisation of X^, then two tcgen05
    bf16 GEMMs that read their operands in place), one call at a time after
    an L2 flush; beside it the dense bf16 layer's two gradient GEMMs with
    operands already in their K-major form (its weights kept in bf16)."""
    import ternary_weight_linear_bitlinear_b200 as bl
    p = WORKLOADS["prefill_2048x4096x11008"].problems[0]
    T, N, K = p.tokens, p.d_out, p.d_in
    W, X = draw(p)
    w = bl.pack_weights(W.to(dev), EPS)
    del W
    xq, beta, _, _ = bl.quant_act(X.to(dev))
    g = torch.Generator().manual_seed(3)
    dY = torch.randn(T, N, generator=g).to(torch.bfloat16).to(dev)
    nbytes = int(bl.lib().bitlinear_backward_workspace_bytes(N, K, T, 1, 1))
    ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    dX = torch.empty((T, K), dtype=torch.float32, device=dev)
    dW = torch.empty((N, K), dtype=torch.float32, device=dev)
    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev)

    def ours():
        bl._check(bl.lib().bitlinear_backward(
            bl._ptr(w.packed), bl._ptr(w.gamma), N, K, bl._ptr(xq), bl._ptr(beta), T,
            bl._ptr(dY), bl._ptr(dX), bl._ptr(dW), bl.OUT_F32, bl._ptr(ws), nbytes,
            bl._stream()), "bitlinear_backward")

    for _ in range(3):
        ours()
    ms = time_each(ours, steps, flush)
    flops = 4.0 * T * N * K
    # The dense bf16 layer's gradient GEMMs on pre-transposed operands.
    Wt = torch.randn(K, N, generator=g).to(torch.bfloat16).to(dev)
    Xt = torch.randn(K, T, generator=g).to(torch.bfloat16).to(dev)
    dYt = dY.t().contiguous()

    def dense():
        bl.dense_bf16_forward(Wt, dY, out_dtype=torch.float32, out=dX)
        bl.dense_bf16_forward(Xt, dYt, out_dtype=torch.float32, out=dW)

    for _ in range(3):
        dense()
    ms_dense = time_each(dense, steps, flush)
    del ws, flush, Wt, Xt, dYt
    torch.cuda.empty_cache()
    tflops = flops / (ms * 1e-3) / 1e12
    return {"workload": "prefill_2048x4096x11008 backward (dX, dW)",
            "ms": round(ms, 4), "tflops": round(tflops, 1),
            "roofline": {"bound": "tensor", "achieved": round(tflops, 1),
                         "peak": peaks["bf16"], "unit": "TFLOP/s",
                         "frac": round(tflops / peaks["bf16"], 4),
                         "peak_source": peaks["source"] + " bf16 burst"},
            "dense_bf16_gemms_ms": round(ms_dense, 4),
            "overhead_vs_dense": round(ms / ms_dense, 3),
            "gpu_launches": 4 * steps}


# ------------------------------------------------------- bf16 context ---

def measure_context_bf16(dev, peaks, decode_us: dict, prefill_ms: float):
    """The dense bf16 layer of the same shapes (bitlinear_dense_bf16_forward,
    hand-written kernels), timed the same way: decode forwards over distinct
    weight copies (more bytes than L2) in a CUDA graph; the prefill GEMM one
    call at a time after an L2 flush."""
    import ternary_weight_linear_bitlinear_b200 as bl
    out = {"kernel": "bitlinear_dense_bf16_forward (streaming GEMV for T <= 16, "
                     "tcgen05 kind::f16 GEMM above)"}
    g = torch.Generator().manual_seed(0)
    for name in ("decode_gemv_2560x6912_t1", "large_gemv_8192x28672_t1"):
        p = WORKLOADS[name].problems[0]
        wbytes = 2 * p.d_out * p.d_in
        copies = max(2, int(np.ceil(2 * L2_BYTES / wbytes)))
        Ws = [(torch.randn(p.d_out, p.d_in, generator=g) * p.sigma).to(torch.bfloat16).to(dev)
              for _ in range(copies)]
        X = torch.randn(p.tokens, p.d_in, generator=g).to(torch.bfloat16).to(dev)
        Y = torch.empty((p.tokens, p.d_out), dtype=torch.bfloat16, device=dev)
        reps = 8
        for W in Ws:
            bl.dense_bf16_forward(W, X, out=Y)
        gr = capture(lambda: [bl.dense_bf16_forward(W, X, out=Y) for _ in range(reps)
                              for W in Ws])
        time_graph(gr)
        us = time_graph(gr) * 1e3 / (reps * copies)
        nbytes = wbytes + 2 * p.tokens * p.d_in + 2 * p.tokens * p.d_out
        out[name] = {"us_per_forward": round(us, 3),
                     "gbs": round(nbytes / (us * 1e-6) / 1e9, 1),
                     "frac_of_hbm": round(nbytes / (us * 1e-6) / 1e9 / peaks["hbm"], 4),
                     "weight_bytes": wbytes}
        if name in decode_us:
            out[name]["ternary_speedup"] = round(us / decode_us[name], 2)
        del Ws, gr
        torch.cuda.empty_cache()
    p = WORKLOADS["prefill_2048x4096x11008"].problems[0]
    W = (torch.randn(p.d_out, p.d_in, generator=g) * p.sigma).to(torch.bfloat16).to(dev)
    X = torch.randn(p.tokens, p.d_in, generator=g).to(torch.bfloat16).to(dev)
    Y = torch.empty((p.tokens, p.d_out), dtype=torch.bfloat16, device=dev)
    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev)
    for _ in range(3):
        bl.dense_bf16_forward(W, X, out=Y)
    ms = time_each(lambda: bl.dense_bf16_forward(W, X, out=Y), 10, flush)
    tflops = 2.0 * p.tokens * p.d_in * p.d_out / (ms * 1e-3) / 1e12
    out["prefill_2048x4096x11008"] = {
        "ms": round(ms, 4), "tflops": round(tflops, 1),
        "frac_of_bf16_peak": round(tflops / peaks["bf16"], 4),
        "ternary_speedup": round(ms / prefill_ms, 2) if prefill_ms else None}
    del W, X, Y, flush
    torch.cuda.empty_cache()
    return out


# ------------------------------------------------------------ e2e ---

def measure_e2e(run, steps):
    """Through the public API with host buffers: every step copies its
    activations (all layers' X, one pinned host buffer) host -> device and
    reads all its outputs back device -> host, inside the timed region.  The
    step is a LinearPlan call per layer (arguments bound once), run as a
    StepGraph (the step captured once as a CUDA graph, copies included, and
    replayed): one step at a time on one stream, and double-buffered -- two
    steps in flight on two streams with their own buffers, each step's kernels
    ordered after the previous step's kernels (events), so that only the
    copies of one step overlap the kernels of the other; eagerly for
    comparison."""
    bl = run.bl
    dev = run.dev
    xs = [X for _, _, X, _, _, _ in run.layers]
    ys = [Y for _, _, _, _, Y, _ in run.layers]
    x_elems = [x.numel() for x in xs]
    y_elems = [y.numel() for y in ys]

    class Lane:
        """Pinned host X and Y, device buffers, scratch and plans of one step."""

        def __init__(self, stream):
            self.s = stream
            self.host_x = torch.cat([x.reshape(-1) for x in xs]).cpu().pin_memory()
            self.host_y = torch.empty(sum(y_elems), dtype=ys[0].dtype).pin_memory()
            self.dev_x = torch.empty_like(self.host_x, device=dev)
            self.dev_y = torch.empty(sum(y_elems), dtype=ys[0].dtype, device=dev)
            self.x_views, y_views, ox, oy = [], [], 0, 0
            for x, y, nx, ny in zip(xs, ys, x_elems, y_elems):
                self.x_views.append(self.dev_x[ox:ox + nx].view(x.shape))
                y_views.append(self.dev_y[oy:oy + ny].view(y.shape))
                ox += nx
                oy += ny
            self.plans = []
            for (p, w, X, _, _, _), Yv in zip(run.layers, y_views):
                T = X.shape[0]
                scratch = (torch.empty((T, p.d_in), dtype=torch.int8, device=dev),
                           torch.empty(T, dtype=torch.float32, device=dev),
                           torch.empty(T, dtype=torch.int32, device=dev))
                self.plans.append(bl.LinearPlan(w, T, out=Yv, scratch=scratch,
                                                static_weights=True, stream=stream))
            self.graph = None
            self.g_in = self.g_calls = self.g_out = None
            self.done = torch.cuda.Event()   # this step's kernels finished

        def copy_in(self):
            self.dev_x.copy_(self.host_x, non_blocking=True)

        def calls(self):
            for plan, X in zip(self.plans, self.x_views):
                plan(X)

        def copy_out(self):
            self.host_y.copy_(self.dev_y, non_blocking=True)

        def one(self):
            self.copy_in()
            self.calls()
            self.copy_out()

    lanes = [Lane(torch.cuda.Stream()), Lane(torch.cuda.Stream())]
    h2d = lanes[0].host_x.numel() * lanes[0].host_x.element_size()
    d2h = lanes[0].host_y.numel() * lanes[0].host_y.element_size()
    s0, s1 = lanes[0].s, lanes[1].s

    def timed(fn):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        a.record(s0)
        s1.wait_stream(s0)
        for i in range(steps):
            fn(i)
        s0.wait_stream(s1)
        b.record(s0)
        b.synchronize()
        return a.elapsed_time(b) / steps

    with torch.cuda.stream(s0):
        lanes[0].one()
        torch.cuda.synchronize()
        ms_eager = timed(lambda i: lanes[0].one())
    for lane in lanes:
        lane.graph = bl.StepGraph(lane.one, stream=lane.s)
        lane.g_in = bl.StepGraph(lane.copy_in, stream=lane.s)
        lane.g_calls = bl.StepGraph(lane.calls, stream=lane.s)
        lane.g_out = bl.StepGraph(lane.copy_out, stream=lane.s)
        lane.graph()
    torch.cuda.synchronize()

    def replay(lane):
        with torch.cuda.stream(lane.s):
            lane.graph()

    def pipelined(i):
        lane, prev = lanes[i % 2], lanes[(i + 1) % 2]
        with torch.cuda.stream(lane.s):
            lane.g_in()
            if i > 0:
                lane.s.wait_event(prev.done)   # kernels one step after another
            lane.g_calls()
            lane.done.record(lane.s)
            lane.g_out()

    ms_graph = timed(lambda i: replay(lanes[0]))
    ms_pipe = timed(pipelined)
    return ms_pipe, ms_graph, ms_eager, h2d, d2h


# -------------------------------------------------------- CPU oracle ---

def oracle_layer_step(p, wq, gamma, xb, parallel=False):
    import oracle
    xq, beta, rowsum, _ = oracle.quant_act(xb, eps=EPS)
    acc = oracle.int_matmul(wq, xq, parallel=parallel)
    return oracle.rescale(acc, gamma, beta)


def _oracle_prepared(name):
    import oracle
    oracle.build()
    prepared = []
    for p in WORKLOADS[name].problems:
        W, X = draw(p)
        Wn = W.numpy()
        g = oracle.absmean_gamma(Wn)
        prepared.append((p, oracle.ternarize(Wn, g, EPS), g, bf16_bits(X)))
        del W, Wn
    return prepared


def cpu_oracle_rate(name, seconds, parallel=False, max_layers=None):
    """Time the oracle on bounded samples of a decode workload: whole
    forwards (quantise, int32 product, rescale) for about `seconds`.  Returns
    (GB/s of algorithmic bytes, forwards done, seconds)."""
    prepared = _oracle_prepared(name)
    done, nbytes, t0 = 0, 0, time.perf_counter()
    while True:
        p, wq, g, xb = prepared[done % len(prepared)]
        oracle_layer_step(p, wq, g, xb, parallel)
        done += 1
        nbytes += decode_bytes(p)["step"]
        el = time.perf_counter() - t0
        if el >= seconds or (max_layers and done >= max_layers):
            break
    return nbytes / el / 1e9, done, el


def cpu_oracle_prefill(seconds):
    """The prefill product on the host's cores: the oracle's int32 product of
    the first tokens of the 2048-token workload (quantised once), growing the
    token count until a call takes about `seconds`.  Returns (TOPS, tokens,
    seconds of the last call)."""
    import oracle
    (p, wq, g, xb), = _oracle_prepared("prefill_2048x4096x11008")
    xq, _, _, _ = oracle.quant_act(xb, eps=EPS)
    T = 8
    while True:
        t0 = time.perf_counter()
        oracle.int_matmul(wq, xq[:T], parallel=True)
        el = time.perf_counter() - t0
        if el >= seconds / 4 or T >= p.tokens:
            break
        T = min(p.tokens, T * 4)
    return 2.0 * T * p.d_in * p.d_out / el / 1e12, T, el


def cpu_baseline_line(workload, seconds):
    """The CPU oracle on this host: every core (the OpenMP build of the same
    C source) on the headline, the large GEMV and a prefill sample, plus the
    single-thread rate on the headline."""
    import oracle
    threads = oracle.threads(parallel=True)
    rate, done, el = cpu_oracle_rate(workload, seconds / 3, parallel=True)
    rate1, done1, el1 = cpu_oracle_rate(workload, seconds / 3)
    rl, donel, ell = cpu_oracle_rate("large_gemv_8192x28672_t1", seconds / 6, parallel=True)
    tops, tp, elp = cpu_oracle_prefill(seconds / 6)
    shape = "x".join(workload.split("_")[2:3])
    return {
        "value": round(rate, 4), "unit": "GB/s", "cores": threads, "kind": "oracle",
        "host_cpus": len(os.sched_getaffinity(0)),
        "sample": "%d single-token %s BitLinear forwards (quantise + int32 product + rescale) "
                  "by the plain C oracle, its product split over %d OpenMP threads, %.1f s"
                  % (done, shape, threads, el),
        "single_thread": {"value": round(rate1, 4), "unit": "GB/s", "cores": 1,
                          "sample": "%d forwards, one thread, %.1f s" % (done1, el1)},
        "large_gemv_8192x28672_t1": {"value": round(rl, 4), "unit": "GB/s", "cores": threads,
                                     "sample": "%d forwards, %.1f s" % (donel, ell)},
        "prefill_2048x4096x11008": {"value": round(tops, 5), "unit": "TOPS", "cores": threads,
                                    "sample": "int32 product of the first %d of 2048 quantised "
                                              "tokens, %.2f s" % (tp, elp)},
    }


# -------------------------------------------------------------- main ---

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=HEADLINE, choices=sorted(WORKLOADS))
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-extras", action="store_true",
                    help="headline only (no prefill / other decode workloads)")
    ap.add_argument("--only-prefill", action="store_true",
                    help="time the prefill forward alone and print its JSON object")
    ap.add_argument("--only-formats", action="store_true",
                    help="time the 2-bit, base-3 and W1A4 decode formats alone, print their JSON")
    ap.add_argument("--formats-workload", default=None,
                    choices=["decode_gemv_2560x6912_t1", "decode_block_4096_t1",
                             "large_gemv_8192x28672_t1", "large_gemv_8192x28672_t8"],
                    help="with --only-formats: that one decode workload")
    ap.add_argument("--only-backward", action="store_true",
                    help="time the straight-through-estimator backward alone, print its JSON")
    args = ap.parse_args()
    warmup = max(args.warmup, 3)
    rank, world, local = dist_init(args.gpus)

    if args.impl == "reference":
        if rank == 0:
            reference_arm(args, warmup)
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return

    dev = torch.device("cuda", local)
    peaks = load_peaks()
    if args.only_prefill:
        res = measure_prefill(max(3, args.steps), warmup, dev, peaks)
        if rank == 0:
            print(json.dumps({"prefill": res}), flush=True)
        if world > 1:
            import torch.distributed as dist
            barrier(world)
            dist.destroy_process_group()
        return
    if args.only_formats:
        res = measure_formats(dev, peaks, workloads=[args.formats_workload]
                              if args.formats_workload else None)
        if rank == 0:
            print(json.dumps({"weight_formats": res}), flush=True)
        if world > 1:
            import torch.distributed as dist
            barrier(world)
            dist.destroy_process_group()
        return
    if args.only_backward:
        res = measure_backward(max(3, args.steps), dev, peaks)
        if rank == 0:
            print(json.dumps({"backward_ste": res}), flush=True)
        if world > 1:
            import torch.distributed as dist
            barrier(world)
            dist.destroy_process_group()
        return
    sampler = ClockSampler(local)
    sampler.start()

    run, nb, g_timed = run_decode(args.workload, args.steps, warmup, dev, LAYERS, world)
    barrier(world)
    torch.cuda.synchronize()
    sampler.mark(True)
    torch.cuda.nvtx.range_push("timed")
    ms = time_graph(g_timed)
    torch.cuda.nvtx.range_pop()
    sampler.mark(False)
    ms = max_over_ranks(ms, world)
    ms_step = ms / args.steps
    value = replica_value(nb["step"], world, ms_step)

    # The product kernel alone (pre-quantised codes), back to back.
    sampler.mark(True)
    gemv_ms, gemv_launches = measure_product_only(run, args.steps)
    sampler.mark(False)
    per_gemv_bytes = nb["gemv"] / len(run.layers)
    gemv_gbs = per_gemv_bytes / (gemv_ms * 1e-3) / 1e9
    traffic = profile_traffic("decode_kernel_2560x6912_t1.md", DECODE_SOURCES)
    one_kernel = all(fused(p) for p in run.problems)
    if one_kernel:
        # Each forward is one kernel: its average duration over the timed region.
        rf_kernel = "decode_kernel<fused> (quantise + GEMV + rescale, one launch per forward)"
        rf_bytes = nb["step"] / len(run.layers)
        rf_us = ms_step * 1e3 / len(run.layers)
        rf_launches = args.steps * len(run.layers)
    else:
        rf_kernel = "decode_kernel (GEMV + rescale)"
        rf_bytes, rf_us, rf_launches = per_gemv_bytes, gemv_ms * 1e3, gemv_launches
    rf_gbs = rf_bytes / (rf_us * 1e-6) / 1e9

    extras = {}
    if not args.no_extras:
        sampler.mark(True)
        extras["prefill"] = measure_prefill(max(10, min(args.steps, 50)), warmup, dev, peaks)
        sampler.mark(False)
        other = {}
        for name in ("decode_block_4096_t1", "decode_block_4096_t16", "large_gemv_8192x28672_t1",
                     "large_gemv_8192x28672_t8"):
            wl = WORKLOADS[name]
            per = sum(decode_bytes(p)["weights"] for p in wl.problems)
            layers = max(len(wl.problems), int(np.ceil(4 * L2_BYTES / per)) * len(wl.problems))
            r2 = DecodeRun(wl.problems, layers, dev)
            g2 = capture(lambda: [r2.step() for _ in range(5)])
            time_graph(g2)
            sampler.mark(True)
            t2 = time_graph(g2) / 5
            sampler.mark(False)
            b2 = r2.bytes()
            other[name] = {"gbs_step": round(b2["step"] / (t2 * 1e-3) / 1e9, 1),
                           "ms_per_pass": round(t2, 4), "forwards_per_pass": len(r2.layers),
                           "frac_of_hbm": round(b2["step"] / (t2 * 1e-3) / 1e9 / peaks["hbm"], 4)}
            del r2, g2
            torch.cuda.empty_cache()
        extras["decode_other"] = other
        sampler.mark(True)
        extras["weight_formats"] = measure_formats(dev, peaks)
        sampler.mark(False)
        sampler.mark(True)
        extras["backward_ste"] = measure_backward(10, dev, peaks)
        extras["context_bf16"] = measure_context_bf16(
            dev, peaks,
            {args.workload: ms_step * 1e3 / len(run.layers),
             "large_gemv_8192x28672_t1": other["large_gemv_8192x28672_t1"]["ms_per_pass"] * 1e3
             / other["large_gemv_8192x28672_t1"]["forwards_per_pass"]},
            extras["prefill"]["ms_gemm"])
        sampler.mark(False)

    e2e_ms, e2e_serial_ms, e2e_eager_ms, h2d, d2h = measure_e2e(run, max(4, min(args.steps, 20)))
    e2e_ms = max_over_ranks(e2e_ms, world)
    e2e_serial_ms = max_over_ranks(e2e_serial_ms, world)
    e2e_eager_ms = max_over_ranks(e2e_eager_ms, world)
    sampler.stop()
    status = run.bl.device_error(clear=True)

    cpu = None
    if rank == 0 and world == 1:
        cpu = cpu_baseline_line(args.workload, args.cpu_seconds)

    if rank == 0:
        clocks = sampler.summary()
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": warmup, "ms_per_step": round(ms_step, 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "int8", "data": "synthetic",
            "config": {
                "workload": args.workload, "forwards_per_step": len(run.layers),
                "tokens": run.problems[0].tokens, "d_in": run.problems[0].d_in,
                "d_out": run.problems[0].d_out, "out_dtype": "bf16",
                "bytes_per_step": nb["step"],
                "l2": "inputs larger than L2: each step streams %d distinct packed weight "
                      "copies (%.0f MB > %d MB L2)" % (len(run.layers),
                                                       run.weight_bytes_resident() / 1e6,
                                                       L2_BYTES // 2 ** 20),
                "parallelism": "replicas" if world > 1 else "single GPU",
                "static_weights": True,
                "timing": "CUDA graph of all timed steps, CUDA events, max over ranks"},
            "frac_of_hbm": round(value / world / peaks["hbm"], 4),
            "frac_of_datasheet_8000": round(value / world / 8000.0, 4),
            "gbs_weights_and_activations": round(nb["weights_and_acts"] * world /
                                                 (ms_step * 1e-3) / 1e9, 2),
            "roofline": {"bound": "hbm", "kernel": rf_kernel,
                         "achieved": round(rf_gbs, 1), "peak": peaks["hbm"],
                         "unit": "GB/s", "frac": round(rf_gbs / peaks["hbm"], 4),
                         "traffic": traffic, "algorithmic_bytes_per_launch": rf_bytes,
                         "avg_launch_us": round(rf_us, 3), "launches_timed": rf_launches,
                         "peak_source": peaks["source"] + " HBM copy bandwidth"},
            "product_only": {"kernel": "decode_kernel (GEMV + rescale, codes precomputed)",
                             "gbs": round(gemv_gbs, 1), "avg_launch_us": round(gemv_ms * 1e3, 3),
                             "launches": gemv_launches},
            "cpu_baseline": cpu,
            "e2e": {"value": round(replica_value(nb["step"], world, e2e_ms), 3),
                    "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": round(e2e_ms, 4),
                    "one_step_at_a_time": {
                        "value": round(replica_value(nb["step"], world, e2e_serial_ms), 3),
                        "ms_per_step": round(e2e_serial_ms, 4)},
                    "eager": {"value": round(replica_value(nb["step"], world, e2e_eager_ms), 3),
                              "ms_per_step": round(e2e_eager_ms, 4)},
                    "how": "public Python API: a LinearPlan per layer (bitlinear_linear with "
                           "bound arguments), the step replayed as a StepGraph (CUDA graph of "
                           "the copies and the calls); every step one copy of all its X in "
                           "from pinned host memory and one of all its Y out; double-buffered: "
                           "two steps in flight on two streams with their own buffers, each "
                           "step's kernels after the previous step's kernels, so only copies "
                           "overlap kernels"},
            "gpu_launches": (1 if one_kernel else 2) * len(run.layers) * args.steps,
            "clocks": clocks,
            "device_error": run.bl.status_string(status),
        }
        line.update(extras)
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        barrier(world)
        dist.destroy_process_group()


def reference_arm(args, warmup):
    """The CPU oracle timed on this host, same metric and unit.  A step is as
    many BitLinear forwards of the workload as the GPU arm's step (LAYERS,
    cycling through the workload's layers), unless K such steps would take
    more than about two minutes on this host; then fewer forwards per step,
    as config.forwards_per_step says."""
    import oracle
    wl = WORKLOADS[args.workload]
    prepared = _oracle_prepared(args.workload)
    threads = oracle.threads(parallel=True)
    per_step = max(1, LAYERS // len(prepared)) * len(prepared)
    t1 = time.perf_counter()
    for i in range(max(warmup, 1)):
        p, wq, g, xb = prepared[i % len(prepared)]
        oracle_layer_step(p, wq, g, xb, parallel=True)
    one = (time.perf_counter() - t1) / max(warmup, 1)
    budget_s = 120.0
    if args.steps * per_step * one > budget_s:
        per_step = max(1, int(budget_s / (args.steps * one)))
    nbytes = 0
    t0 = time.perf_counter()
    for i in range(args.steps * per_step):
        p, wq, g, xb = prepared[i % len(prepared)]
        oracle_layer_step(p, wq, g, xb, parallel=True)
        nbytes += decode_bytes(p)["step"]
    el = time.perf_counter() - t0
    value = nbytes / el / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": warmup,
        "ms_per_step": round(el * 1e3 / args.steps, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "int8", "data": "synthetic",
        "config": {"workload": args.workload, "forwards_per_step": per_step,
                   "tokens": wl.problems[0].tokens, "d_in": wl.problems[0].d_in,
                   "d_out": wl.problems[0].d_out},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": threads,
                         "kind": "oracle", "host_cpus": len(os.sched_getaffinity(0)),
                         "sample": "each step %d BitLinear forwards of the workload by the "
                                   "plain C oracle, its product split over %d OpenMP threads"
                                   % (per_step, threads)},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
