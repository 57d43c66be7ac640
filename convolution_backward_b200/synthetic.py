"""Seeded synthetic inputs for the dgrad workloads.

This module is the only code the CUDA path and the fp64 oracle share: it draws
dY and W from ``numpy.random.default_rng(seed)`` and rounds them to bf16 where a
workload is bf16.  It holds none of dgrad's arithmetic; the one shape rule it
needs (the forward convolution's output extent, which fixes dY's shape) is the
textbook one, Ho = floor((H + 2*pad_h - KH)/stride) + 1, with Wo from pad_w.

Recipe (one per workload, in this order):
  1. rng = numpy.random.default_rng(seed)
  2. dY: draw in float64 in logical NHWC order and shape (N, Ho, Wo, K)
  3. W : draw in float64 in its storage layout ((K, C) pointwise, (KH, KW, C) depthwise,
     (KH, KW, K, C) dense)
  4. cast to float32; for bf16 workloads round to bf16, for f16 ones to IEEE half,
     both with round-to-nearest-even.
Distributions: "normal" is N(0, var) with ``var`` the variance (std = sqrt(var));
"uniform" is U[-1, 1].  A workload with several problems (the non-square and
strided depthwise set) draws each problem from a fresh generator with the same
seed, in the listed order.
"""
from __future__ import annotations

from dataclasses import dataclass, field
import math

import numpy as np


@dataclass(frozen=True)
class Problem:
    name: str
    kind: str            # "pointwise" | "depthwise" | "dense" | "grouped"
    dtype: str           # "f32" | "bf16" | "f16"
    N: int
    H: int
    W: int
    C: int               # dX channels
    K: int               # dY channels
    KH: int = 1
    KW: int = 1
    stride: int = 1
    pad_h: int = 0
    pad_w: int = 0
    seed: int = 0
    dy_dist: str = "normal"
    dy_var: float = 1.0
    w_dist: str = "normal"
    w_var: float = 1.0
    variant: str = ""    # "splitk": split-K pointwise entry point; "tc": tensor-core depthwise entry point;
    #                      "rotated": dgrad_depthwise forced to the FP32 rotated-filter kernels
    ngroups: int = 1     # groups of a "grouped" problem (K and C multiples of it)

    @property
    def Ho(self) -> int:
        return (self.H + 2 * self.pad_h - self.KH) // self.stride + 1

    @property
    def Wo(self) -> int:
        return (self.W + 2 * self.pad_w - self.KW) // self.stride + 1

    @property
    def groups(self) -> int:
        if self.kind == "depthwise":
            return self.C
        return self.ngroups if self.kind == "grouped" else 1

    @property
    def dy_shape(self):
        return (self.N, self.Ho, self.Wo, self.K)

    @property
    def w_shape(self):
        if self.kind == "pointwise":
            return (self.K, self.C)
        if self.kind == "dense":
            return (self.KH, self.KW, self.K, self.C)
        if self.kind == "grouped":
            return (self.KH, self.KW, self.K, self.C // self.ngroups)
        return (self.KH, self.KW, self.C)

    @property
    def dx_shape(self):
        return (self.N, self.H, self.W, self.C)

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == "f32" else 2

    def nominal_flops(self) -> int:
        """2 * N*Ho*Wo*K * (C/groups) * KH*KW: the forward-conv count, padded taps included."""
        return 2 * self.N * self.Ho * self.Wo * self.K * (self.C // self.groups) * self.KH * self.KW

    def algorithmic_bytes(self) -> int:
        """|dY| + |W| + |dX|, each moved once."""
        e = self.elem_bytes
        return e * (math.prod(self.dy_shape) + math.prod(self.w_shape) + math.prod(self.dx_shape))

    def replace(self, **kw) -> "Problem":
        d = dict(self.__dict__)
        d.update(kw)
        return Problem(**d)


# The five workloads.  Sizes, seeds and distributions are the ones the
# benchmark is quoted on; the fifth holds three problems drawn from seed 4.
# `variant` names the entry point the benchmark step calls: the three large
# stride-1 depthwise problems run through dgrad_depthwise_tc (tensor cores).
# Parity tests run every problem through dgrad_depthwise as well.
WORKLOADS: dict[str, list[Problem]] = {
    "pw_f32_small": [Problem("pw_f32_small", "pointwise", "f32", N=2, H=14, W=14, C=64, K=64,
                             seed=0, dy_dist="uniform", w_dist="uniform")],
    "dw3x3_bf16": [Problem("dw3x3_bf16", "depthwise", "bf16", N=8, H=56, W=56, C=128, K=128,
                           KH=3, KW=3, pad_h=1, pad_w=1, seed=1, w_var=1.0 / 9)],
    "pw_bf16": [Problem("pw_bf16", "pointwise", "bf16", N=32, H=28, W=28, C=256, K=512,
                        seed=2, w_var=1.0 / 512)],
    "dw31x31_bf16": [Problem("dw31x31_bf16", "depthwise", "bf16", N=16, H=64, W=64, C=384, K=384,
                             KH=31, KW=31, pad_h=15, pad_w=15, seed=3, w_var=1.0 / 961, variant="tc")],
    "dw_nonsquare_strided_bf16": [
        Problem("dw51x5_bf16", "depthwise", "bf16", N=8, H=64, W=64, C=768, K=768,
                KH=51, KW=5, pad_h=25, pad_w=2, seed=4, w_var=1.0 / 255, variant="tc"),
        Problem("dw5x51_bf16", "depthwise", "bf16", N=8, H=64, W=64, C=768, K=768,
                KH=5, KW=51, pad_h=2, pad_w=25, seed=4, w_var=1.0 / 255, variant="tc"),
        Problem("dw7x7s2_bf16", "depthwise", "bf16", N=32, H=112, W=112, C=96, K=96,
                KH=7, KW=7, stride=2, pad_h=3, pad_w=3, seed=4, w_var=1.0 / 49),
    ],
}

WORKLOAD_ORDER = ["pw_f32_small", "dw3x3_bf16", "pw_bf16", "dw31x31_bf16",
                  "dw_nonsquare_strided_bf16"]

# Extra workloads outside the benchmark suite (run with --workload NAME).
EXTRA_WORKLOADS: dict[str, list[Problem]] = {
    # small M, long K: 16 output tiles, split-K fills the GPU
    "pw_bf16_smallm_splitk": [Problem("pw_bf16_smallm_splitk", "pointwise", "bf16", N=2, H=14, W=14, C=512,
                                      K=2048, seed=5, w_var=1.0 / 2048, variant="splitk")],
    "pw_bf16_smallm": [Problem("pw_bf16_smallm", "pointwise", "bf16", N=2, H=14, W=14, C=512, K=2048,
                               seed=5, w_var=1.0 / 2048)],
    # dense (ungrouped) 3x3 dgrad through dgrad_dense, stride 1 and stride 2
    "dense3x3_bf16": [Problem("dense3x3_bf16", "dense", "bf16", N=32, H=28, W=28, C=256, K=256, KH=3, KW=3,
                              pad_h=1, pad_w=1, seed=6, w_var=1.0 / 2304)],
    "dense3x3s2_bf16": [Problem("dense3x3s2_bf16", "dense", "bf16", N=32, H=56, W=56, C=128, K=256, KH=3, KW=3,
                                stride=2, pad_h=1, pad_w=1, seed=7, w_var=1.0 / 2304)],
    # the large stride-1 depthwise problems through the FP32 rotated-filter kernel (dgrad_depthwise)
    "dw_large_fp32": [WORKLOADS["dw31x31_bf16"][0].replace(name="dw31x31_bf16_fp32", variant="rotated"),
                      WORKLOADS["dw_nonsquare_strided_bf16"][0].replace(name="dw51x5_bf16_fp32", variant="rotated"),
                      WORKLOADS["dw_nonsquare_strided_bf16"][1].replace(name="dw5x51_bf16_fp32",
                                                                        variant="rotated")],
}


def all_problems() -> list[Problem]:
    return [p for name in WORKLOAD_ORDER for p in WORKLOADS[name]]


def problem(name: str) -> Problem:
    for p in all_problems() + [q for v in EXTRA_WORKLOADS.values() for q in v]:
        if p.name == name:
            return p
    raise KeyError(name)


# ---------------------------------------------------------------- bf16 helpers

def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 (round to nearest, ties to even); return the uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    nan = (u & 0x7FFFFFFF) > 0x7F800000
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16) & 0xFFFF
    r = np.where(nan, (u >> 16) | 0x40, r)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to float32 exactly."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _draw(rng: np.random.Generator, shape, dist: str, var: float) -> np.ndarray:
    if dist == "uniform":
        return rng.uniform(-1.0, 1.0, size=shape)
    if dist == "normal":
        return rng.standard_normal(size=shape) * math.sqrt(var)
    raise ValueError(dist)


@dataclass
class Inputs:
    """One problem's inputs.  ``dy``/``w`` are float32 arrays holding exactly the
    values the kernels see (bf16- or f16-representable for 16-bit problems);
    ``dy_bits`` / ``w_bits`` are the 16-bit patterns (uint16) for 16-bit
    problems, else None."""
    problem: Problem
    dy: np.ndarray
    w: np.ndarray
    dy_bits: np.ndarray | None = None
    w_bits: np.ndarray | None = None
    extra: dict = field(default_factory=dict)


def make_inputs(p: Problem, seed: int | None = None) -> Inputs:
    """Draw dY then W for problem p (recipe in the module docstring)."""
    rng = np.random.default_rng(p.seed if seed is None else seed)
    dy64 = _draw(rng, p.dy_shape, p.dy_dist, p.dy_var)
    w64 = _draw(rng, p.w_shape, p.w_dist, p.w_var)
    dy32 = dy64.astype(np.float32)
    w32 = w64.astype(np.float32)
    if p.dtype == "f32":
        return Inputs(p, dy32, w32)
    if p.dtype == "f16":
        dyh = dy32.astype(np.float16)
        wh = w32.astype(np.float16)
        return Inputs(p, dyh.astype(np.float32), wh.astype(np.float32), dyh.view(np.uint16), wh.view(np.uint16))
    dyb = f32_to_bf16_bits(dy32)
    wb = f32_to_bf16_bits(w32)
    return Inputs(p, bf16_bits_to_f32(dyb), bf16_bits_to_f32(wb), dyb, wb)
