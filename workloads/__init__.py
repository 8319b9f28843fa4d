"""Seeded synthetic inputs for the BitLinear forward path.

This module holds no part of the method's arithmetic: it only draws random
numbers.  Both the CPU oracle and the CUDA library are fed from here, and
nothing here imports either of them.

Recipe (one ``torch.Generator('cpu')`` per problem, seeded, draws in order):
  1. ``W = randn(d_out, d_in) * sigma``            float32 latent weights
  2. ``X = randn(T, d_in)``                         float32 activations
  3. ``idx = randperm(d_in)[:round(frac * d_in)]``  outlier channels
  4. ``X[:, idx] *= factor``                        outlier scaling
  5. ``X -> bfloat16`` (round to nearest even)      the layer's input

The shapes and distributions are those of the workloads named below: a small
parity layer, a 2560->6912 decode GEMV, the seven BitLinears of one
4096-wide transformer block (decode, 1 and 16 tokens), a 8192->28672 decode
GEMV at 1/4/8 tokens and a 2048-token 4096->11008 prefill.  The
activation-outlier channels follow the outlier phenomenon described on "The
End of Matrix Multiplications: Welcome to Addition" (Technical Details: a few
latent dimensions far larger than the median).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch


@dataclass(frozen=True)
class Problem:
    """One BitLinear forward problem: d_in -> d_out at T tokens."""
    name: str
    d_in: int
    d_out: int
    tokens: int
    sigma: float
    outlier_frac: float
    outlier_factor: float
    seed: int
    out_dtype: str = "f32"          # "f32" or "bf16"


@dataclass(frozen=True)
class Workload:
    name: str
    problems: tuple = field(default_factory=tuple)
    description: str = ""


def draw(p: Problem):
    """Return (W float32 [d_out][d_in], X bfloat16 [T][d_in]) as CPU tensors."""
    g = torch.Generator(device="cpu").manual_seed(p.seed)
    W = torch.randn(p.d_out, p.d_in, generator=g, dtype=torch.float32) * p.sigma
    X = torch.randn(p.tokens, p.d_in, generator=g, dtype=torch.float32)
    n_out = int(round(p.outlier_frac * p.d_in))
    if n_out > 0:
        idx = torch.randperm(p.d_in, generator=g)[:n_out]
        X[:, idx] *= p.outlier_factor
    return W, X.to(torch.bfloat16)


def draw_weights(p: Problem):
    """Only the weight draw of ``draw`` (the first draw, so identical)."""
    g = torch.Generator(device="cpu").manual_seed(p.seed)
    return torch.randn(p.d_out, p.d_in, generator=g, dtype=torch.float32) * p.sigma


def bf16_bits(X: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> numpy uint16 bit patterns (no arithmetic)."""
    return X.contiguous().view(torch.int16).numpy().view(np.uint16)


# ----------------------------------------------------------- workloads ---

PARITY_LAYER = Workload(
    "parity_512x512_t4",
    (Problem("parity", 512, 512, 4, 0.02, 0.01, 50.0, 0),),
    "single BitLinear 512->512, 4 tokens, W ~ N(0, 0.02^2), 1% outlier "
    "channels x50, seed 0")

DECODE_GEMV = Workload(
    "decode_gemv_2560x6912_t1",
    (Problem("gemv", 2560, 6912, 1, 0.02, 0.005, 100.0, 0),),
    "decode GEMV 2560->6912, 1 token, W ~ N(0, 0.02^2), 0.5% outlier channels "
    "x100")


def _block(tokens: int) -> Workload:
    shapes = [("q", 4096, 4096), ("k", 4096, 4096), ("v", 4096, 4096),
              ("o", 4096, 4096), ("gate", 4096, 11008), ("up", 4096, 11008),
              ("down", 11008, 4096)]
    probs = tuple(Problem(n, di, do, tokens, 0.02, 0.005, 100.0, seed)
                  for seed, (n, di, do) in enumerate(shapes))
    return Workload("decode_block_4096_t%d" % tokens, probs,
                    "one transformer block's seven BitLinears (q,k,v,o "
                    "4096x4096; gate,up 4096->11008; down 11008->4096), "
                    "%d token(s), seeds 0..6" % tokens)


DECODE_BLOCK_T1 = _block(1)
DECODE_BLOCK_T16 = _block(16)


def _large(tokens: int) -> Workload:
    return Workload("large_gemv_8192x28672_t%d" % tokens,
                    (Problem("large", 8192, 28672, tokens, 0.015, 0.001, 1000.0,
                             0),),
                    "decode GEMV 8192->28672, %d token(s), W ~ N(0, 0.015^2), "
                    "0.1%% outlier channels x1000" % tokens)


LARGE_GEMV_T1 = _large(1)
LARGE_GEMV_T4 = _large(4)
LARGE_GEMV_T8 = _large(8)

PREFILL = Workload(
    "prefill_2048x4096x11008",
    (Problem("prefill", 4096, 11008, 2048, 0.02, 0.0, 1.0, 0, "bf16"),),
    "prefill GEMM, 2048 tokens x 4096 -> 11008, W ~ N(0, 0.02^2), "
    "X ~ N(0,1), bf16 output")

ALL = {w.name: w for w in (PARITY_LAYER, DECODE_GEMV, DECODE_BLOCK_T1,
                           DECODE_BLOCK_T16, LARGE_GEMV_T1, LARGE_GEMV_T4,
                           LARGE_GEMV_T8, PREFILL)}
