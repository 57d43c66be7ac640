"""Helpers for the GPU parity tests: device tensors from the seeded inputs,
oracle references and the comparison rules.

Tolerances (written out here, used by every parity test):
  normwise, the acceptance bar:
    bf16, f16 I/O : max|gpu - ref| / (max|ref| + 1e-6) <= 1e-2
    f32 I/O  : max|gpu - ref| / max|ref|          <= 1e-5
  elementwise, derived from the arithmetic (fp32 accumulation of n terms in any
  order, then one rounding of the output):
    |gpu - ref| <= u_out*|ref| + (1 + u_out) * n * 2^-24 * sum|terms| + eta_out
  with u_out = 2^-8 for a bf16 output (8 significant bits, round to nearest
  even: half an ulp is 2^-8 relative), 2^-11 for f16 (11 significant bits) and
  2^-24 for f32 (24 significant bits),
  n the number of products per output and sum|terms| the same dgrad
  evaluated on |dY| and |W| (by the oracle).  eta_out is the absolute error of
  rounding into the output format's subnormal range (gradual underflow: the
  rounding model fl(x) = x(1 + d) + e with |e| at most half the smallest
  subnormal): 2^-25 for f16, whose normals end at 2^-14; for bf16 and f32 it is
  below 1e-30, the floor the bound always carries.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from convolution_backward_b200 import synthetic

U_BF16 = 2.0 ** -8
U_F16 = 2.0 ** -11
U_F32 = 2.0 ** -24
ETA_F16 = 2.0 ** -25   # half the f16 subnormal spacing 2^-24


def to_dev(inp: synthetic.Inputs):
    """Device tensors (dY, W) holding exactly the values in inp."""
    p = inp.problem
    if p.dtype in ("bf16", "f16"):
        tt = torch.bfloat16 if p.dtype == "bf16" else torch.float16
        dy = torch.from_numpy(inp.dy_bits.view(np.int16)).view(tt).cuda()
        w = torch.from_numpy(inp.w_bits.view(np.int16)).view(tt).cuda()
    else:
        dy = torch.from_numpy(inp.dy).cuda()
        w = torch.from_numpy(inp.w).cuda()
    return dy.contiguous(), w.contiguous()


def run_gpu(p: synthetic.Problem, dy, w, mode="auto", out=None):
    import convolution_backward_b200 as cb
    if p.kind == "pointwise":
        return cb.pointwise(dy, w, out=out)
    if p.kind == "dense":
        return cb.dense(dy, w, H=p.H, Wd=p.W, stride=p.stride, pad_h=p.pad_h, pad_w=p.pad_w, out=out)
    if p.kind == "grouped":
        return cb.grouped(dy, w, p.ngroups, H=p.H, Wd=p.W, stride=p.stride, pad_h=p.pad_h, pad_w=p.pad_w,
                          out=out)
    return cb.depthwise(dy, w, H=p.H, Wd=p.W, stride=p.stride, pad_h=p.pad_h, pad_w=p.pad_w, mode=mode,
                        out=out)


def _oracle_kind(p: synthetic.Problem, w: np.ndarray):
    """The oracle's kind and filter for p: a dense W [KH][KW][K][C] goes in as the grouped layout
    (K, KH, KW, C) with one group (the same values, reordered)."""
    if p.kind in ("dense", "grouped"):
        return (dict(kind="grouped", groups=p.groups, C=p.C),
                np.ascontiguousarray(np.asarray(w).transpose(2, 0, 1, 3)))
    return dict(kind=p.kind), w


def oracle_full(p: synthetic.Problem, dy: np.ndarray, w: np.ndarray) -> np.ndarray:
    kw, w = _oracle_kind(p, w)
    return oracle.dgrad(dy, w, H=p.H, W=p.W, KH=p.KH, KW=p.KW, S=p.stride, ph=p.pad_h, pw=p.pad_w, **kw)


def oracle_points(p: synthetic.Problem, dy: np.ndarray, w: np.ndarray, pts) -> np.ndarray:
    kw, w = _oracle_kind(p, w)
    return oracle.dgrad_points(dy, w, pts, H=p.H, W=p.W, KH=p.KH, KW=p.KW, S=p.stride, ph=p.pad_h,
                               pw=p.pad_w, **kw)


def terms_per_output(p: synthetic.Problem) -> int:
    if p.kind == "pointwise":
        return p.K
    if p.kind in ("dense", "grouped"):
        return (p.K // p.groups) * p.KH * p.KW
    return p.KH * p.KW


def check(p: synthetic.Problem, got: np.ndarray, ref: np.ndarray, absref: np.ndarray, what: str = ""):
    """Apply both rules; raise AssertionError with the worst offender on failure."""
    got = np.asarray(got, dtype=np.float64)
    err = np.abs(got - ref)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    mx = float(np.max(np.abs(ref))) if ref.size else 0.0
    if p.dtype in ("bf16", "f16"):
        norm = float(err.max(initial=0.0)) / (mx + 1e-6)
        assert norm <= 1e-2, f"{what}: normwise error {norm:.3e} > 1e-2"
        u = U_BF16 if p.dtype == "bf16" else U_F16
    else:
        norm = float(err.max(initial=0.0)) / mx if mx > 0 else float(err.max(initial=0.0))
        assert norm <= 1e-5, f"{what}: normwise error {norm:.3e} > 1e-5"
        u = U_F32
    n = terms_per_output(p)
    eta = ETA_F16 if p.dtype == "f16" else 1e-30
    bound = u * np.abs(ref) + (1 + u) * n * U_F32 * absref + eta
    bad = err > bound
    if np.any(bad):
        i = int(np.argmax(err - bound))
        raise AssertionError(f"{what}: elementwise bound broken at flat index {i}: got {got.flat[i]!r}, "
                             f"ref {ref.flat[i]!r}, bound {bound.flat[i]!r} ({int(bad.sum())} elements)")
    return norm


def sample_points(p: synthetic.Problem, count: int, seed: int = 123):
    """Random (n,h,w,c) points plus the image corners and edges of a few channels."""
    r = np.random.default_rng(seed)
    pts = np.stack([r.integers(0, p.N, count), r.integers(0, p.H, count), r.integers(0, p.W, count),
                    r.integers(0, p.C, count)], axis=1)
    extra = []
    for n in (0, p.N - 1):
        for h in (0, 1, p.H // 2, p.H - 2, p.H - 1):
            for x in (0, 1, p.W // 2, p.W - 2, p.W - 1):
                for c in (0, 1, p.C - 2, p.C - 1):
                    extra.append((n, max(h, 0), max(x, 0), max(c, 0)))
    return np.concatenate([pts, np.array(extra, dtype=np.int64)], axis=0)


def gpu_to_np(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)
