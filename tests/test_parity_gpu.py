"""GPU parity: the CUDA kernels, called through the C ABI, against the fp64 oracle.

Small cases are compared element by element with the oracle over the whole
output; they span several tiles and ragged tails (M, K and C not multiples of
the tile sizes, channel counts not multiples of 32, odd image sizes).  The five
workloads run at full size with the launch configuration the benchmark times;
there the oracle evaluates a sample of outputs one by one (random points plus
corners and edges), and every element is also checked against cuDNN in fp32.
Tolerances are written out in gpu_helpers.
"""
import os

import numpy as np
import pytest

from convolution_backward_b200 import synthetic
from convolution_backward_b200.synthetic import Problem

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def _h():
    import gpu_helpers
    return gpu_helpers


def P(name, kind, dtype, N, H, W, C, K, KH=1, KW=1, S=1, ph=0, pw=0, seed=11):
    return Problem(name, kind, dtype, N=N, H=H, W=W, C=C, K=K, KH=KH, KW=KW, stride=S, pad_h=ph,
                   pad_w=pw, seed=seed, w_var=1.0 / (KH * KW) if kind == "depthwise" else 1.0 / K)


SMALL = [
    # pointwise bf16 (tcgen05): ragged M (598 = 4 tiles + 86), ragged K (200 = 3*64 + 8), ragged C
    P("pw_bf16_ragged", "pointwise", "bf16", 2, 13, 23, 264, 200, seed=21),
    P("pw_bf16_c40", "pointwise", "bf16", 1, 9, 15, 40, 72, seed=22),
    P("pw_bf16_k8_c8", "pointwise", "bf16", 3, 5, 7, 8, 8, seed=23),
    P("pw_bf16_one_row", "pointwise", "bf16", 1, 1, 1, 128, 64, seed=24),
    P("pw_bf16_256", "pointwise", "bf16", 4, 16, 20, 256, 512, seed=25),
    # pointwise f32
    P("pw_f32_ragged", "pointwise", "f32", 1, 7, 11, 20, 12, seed=26),
    P("pw_f32_wide", "pointwise", "f32", 2, 10, 9, 132, 100, seed=27),
    # depthwise stride 1 (rotated filter)
    P("dw3x3", "depthwise", "bf16", 2, 19, 23, 40, 40, 3, 3, 1, 1, 1, seed=31),
    P("dw31x31", "depthwise", "bf16", 1, 37, 45, 32, 32, 31, 31, 1, 15, 15, seed=32),
    P("dw51x5", "depthwise", "bf16", 1, 45, 30, 24, 24, 51, 5, 1, 25, 2, seed=33),
    P("dw5x51", "depthwise", "bf16", 1, 30, 45, 24, 24, 5, 51, 1, 2, 25, seed=34),
    P("dw7x7_nonsame", "depthwise", "bf16", 2, 17, 18, 16, 16, 7, 7, 1, 1, 5, seed=35),
    P("dw5x5_pw0", "depthwise", "bf16", 1, 12, 14, 48, 48, 5, 5, 1, 2, 0, seed=36),
    P("dw4x6_even", "depthwise", "bf16", 1, 11, 13, 8, 8, 4, 6, 1, 3, 0, seed=37),
    P("dw64x64_max", "depthwise", "bf16", 1, 70, 66, 8, 8, 64, 64, 1, 32, 31, seed=38),
    P("dw1x1", "depthwise", "bf16", 2, 5, 6, 16, 16, 1, 1, 1, 0, 0, seed=39),
    P("dw13x13", "depthwise", "bf16", 1, 33, 35, 64, 64, 13, 13, 1, 6, 6, seed=40),
    P("dw3x3_f32", "depthwise", "f32", 2, 9, 10, 12, 12, 3, 3, 1, 1, 1, seed=41),
    P("dw31x31_f32", "depthwise", "f32", 1, 20, 21, 8, 8, 31, 31, 1, 15, 15, seed=42),
    P("dw3x3_tiny_image", "depthwise", "bf16", 1, 1, 1, 8, 8, 3, 3, 1, 1, 1, seed=43),
    # depthwise strided (row streaming)
    P("dw7x7s2", "depthwise", "bf16", 2, 29, 27, 40, 40, 7, 7, 2, 3, 3, seed=51),
    P("dw3x3s2", "depthwise", "bf16", 1, 20, 21, 32, 32, 3, 3, 2, 1, 1, seed=52),
    P("dw5x3s3", "depthwise", "bf16", 1, 22, 19, 16, 16, 5, 3, 3, 2, 1, seed=53),
    P("dw2x2s3_gaps", "depthwise", "bf16", 1, 14, 13, 8, 8, 2, 2, 3, 0, 0, seed=54),
    P("dw31x31s2", "depthwise", "bf16", 1, 70, 66, 16, 16, 31, 31, 2, 15, 15, seed=55),
    P("dw7x7s2_f32", "depthwise", "f32", 1, 15, 16, 12, 12, 7, 7, 2, 3, 3, seed=56),
    P("dw64x64s1_rowstream", "depthwise", "bf16", 1, 66, 65, 8, 8, 64, 64, 1, 30, 33, seed=57),
]

ROWSTREAM_AT_S1 = {"dw3x3", "dw7x7_nonsame", "dw51x5", "dw5x5_pw0", "dw4x6_even", "dw64x64s1_rowstream",
                   "dw3x3_f32", "dw31x31"}


def _modes(p):
    if p.kind == "pointwise":
        return ["auto"]
    if p.stride > 1:
        return ["auto"]
    if p.name == "dw64x64s1_rowstream":
        return ["rowstream"]
    return ["auto", "rowstream"] if p.name in ROWSTREAM_AT_S1 else ["auto"]


CASES = [(p, m) for p in SMALL for m in _modes(p)]


@pytest.mark.parametrize("p,mode", CASES, ids=[f"{p.name}-{m}" for p, m in CASES])
def test_small_against_oracle(p, mode):
    h = _h()
    inp = synthetic.make_inputs(p)
    dy, w = h.to_dev(inp)
    got = h.gpu_to_np(h.run_gpu(p, dy, w, mode=mode))
    torch.cuda.synchronize()
    ref = h.oracle_full(p, inp.dy, inp.w)
    absref = h.oracle_full(p, np.abs(inp.dy), np.abs(inp.w))
    h.check(p, got, ref, absref, what=f"{p.name}/{mode}")
    import convolution_backward_b200 as cb
    cb.check_status()


PW_VARIANTS = [("pair", None), ("resident", None), ("pair", "128"), ("pair", "256"), ("stream", "64"),
               ("stream", "128"), ("stream", "256")]


@pytest.mark.parametrize("mode,bn", PW_VARIANTS, ids=[f"{m}-{b}" for m, b in PW_VARIANTS])
@pytest.mark.parametrize("shape", [(1, 23, 17, 328, 136), (2, 13, 23, 264, 200), (1, 9, 11, 64, 512),
                                   (3, 7, 5, 8, 8), (4, 16, 20, 256, 512)],
                         ids=["c328k136", "c264k200", "c64k512", "c8k8", "c256k512"])
def test_pointwise_kernels(mode, bn, shape, monkeypatch):
    """Every tcgen05 kernel (resident W; SM pair with 256 x 128 and 256 x 256 tiles; streaming W with
    BN = 64, 128, 256) on ragged problems."""
    h = _h()
    monkeypatch.setenv("DGRAD_PW_MODE", mode)
    if bn:
        monkeypatch.setenv("DGRAD_PW_BN", bn)
    N, H, W, C, K = shape
    p = P("pw_bf16_var", "pointwise", "bf16", N, H, W, C, K, seed=60)
    inp = synthetic.make_inputs(p)
    dy, w = h.to_dev(inp)
    got = h.gpu_to_np(h.run_gpu(p, dy, w))
    ref = h.oracle_full(p, inp.dy, inp.w)
    absref = h.oracle_full(p, np.abs(inp.dy), np.abs(inp.w))
    h.check(p, got, ref, absref, what=f"{mode}/BN={bn}")
    import convolution_backward_b200 as cb
    cb.check_status()


# Shapes where the SM-pair kernel has more tiles than pairs and splits the leftover ones in N:
# (N, H, W, C, K) with 75 tiles of 256 x 256 (one leftover tile, two halves), and with 80 tiles over
# two column blocks of which the second is ragged (C = 320: the upper halves of its leftover tiles
# lie wholly past C, so they load zeros and store nothing).
PW_SPLIT = [(2, 95, 100, 256, 136), (5, 40, 50, 320, 72)]


@pytest.mark.parametrize("shape", PW_SPLIT, ids=["75_tiles", "80_tiles_ragged_C"])
def test_pointwise_pair_split_last_round(shape):
    """The default pair kernel (256 x 256 tiles) where the last round's tiles are split in N."""
    h = _h()
    N, H, W, C, K = shape
    p = P("pw_bf16_split", "pointwise", "bf16", N, H, W, C, K, seed=61)
    inp = synthetic.make_inputs(p)
    dy, w = h.to_dev(inp)
    got = h.gpu_to_np(h.run_gpu(p, dy, w))
    ref = h.oracle_full(p, inp.dy, inp.w)
    absref = h.oracle_full(p, np.abs(inp.dy), np.abs(inp.w))
    h.check(p, got, ref, absref, what="pair, split last round")
    import convolution_backward_b200 as cb
    cb.check_status()


ROT_SMALL = [
    P("tile3x3", "depthwise", "bf16", 2, 19, 23, 40, 40, 3, 3, 1, 1, 1, seed=81),
    P("tile3x3_wide", "depthwise", "bf16", 1, 9, 150, 32, 32, 3, 3, 1, 0, 2, seed=82),
    P("tile5x5", "depthwise", "bf16", 1, 12, 14, 48, 48, 5, 5, 1, 2, 0, seed=83),
    P("tile7x7", "depthwise", "bf16", 2, 17, 18, 16, 16, 7, 7, 1, 1, 5, seed=84),
    P("tile7x7_same", "depthwise", "bf16", 1, 33, 31, 72, 72, 7, 7, 1, 3, 3, seed=85),
    P("tile3x3_1px", "depthwise", "bf16", 1, 1, 1, 8, 8, 3, 3, 1, 1, 1, seed=86),
]


@pytest.mark.parametrize("kernel", ["tile", "tile-direct-stores", "line"])
@pytest.mark.parametrize("p", ROT_SMALL, ids=[p.name for p in ROT_SMALL])
def test_rotated_small_filter_kernels(p, kernel, monkeypatch):
    """Small stride-1 filters through the halo-tile kernel and the line kernel."""
    h = _h()
    if kernel == "tile-direct-stores":
        monkeypatch.setenv("DGRAD_TILE_STORE", "direct")   # the tile kernel without its TMA-stored output tile
        kernel = "tile"
    monkeypatch.setenv("DGRAD_ROT_KERNEL", kernel)
    inp = synthetic.make_inputs(p)
    dy, w = h.to_dev(inp)
    got = h.gpu_to_np(h.run_gpu(p, dy, w))
    ref = h.oracle_full(p, inp.dy, inp.w)
    absref = h.oracle_full(p, np.abs(inp.dy), np.abs(inp.w))
    h.check(p, got, ref, absref, what=f"{p.name}/{kernel}")
    import convolution_backward_b200 as cb
    cb.check_status()


DW_F16 = [
    # stride 1: the halo-tile kernel (3x3, 5x5, 7x7) and the rotated-line kernel
    (P("f16_tile3x3", "depthwise", "f16", 2, 19, 23, 40, 40, 3, 3, 1, 1, 1, seed=301), {}),
    (P("f16_tile7x7", "depthwise", "f16", 1, 33, 31, 72, 72, 7, 7, 1, 3, 3, seed=302), {}),
    (P("f16_line5x5", "depthwise", "f16", 1, 12, 14, 48, 48, 5, 5, 1, 2, 0, seed=303), {"DGRAD_ROT_KERNEL": "line"}),
    (P("f16_line13x13", "depthwise", "f16", 1, 33, 35, 64, 64, 13, 13, 1, 6, 6, seed=304), {}),
    (P("f16_line51x5", "depthwise", "f16", 1, 45, 30, 24, 24, 51, 5, 1, 25, 2, seed=305), {}),
    (P("f16_line5x51", "depthwise", "f16", 1, 30, 45, 24, 24, 5, 51, 1, 2, 25, seed=306), {}),
    # strided: register ring (two and four columns per thread), shared ring, generic
    (P("f16_rs7x7s2", "depthwise", "f16", 2, 29, 27, 40, 40, 7, 7, 2, 3, 3, seed=307), {}),
    (P("f16_rs7x7s2_q4", "depthwise", "f16", 1, 23, 40, 16, 16, 7, 7, 2, 6, 1, seed=308), {"DGRAD_RS_Q": "4"}),
    (P("f16_rs5x5s2_smem", "depthwise", "f16", 2, 25, 26, 48, 48, 5, 5, 2, 2, 2, seed=309),
     {"DGRAD_RS_KERNEL": "smem"}),
    (P("f16_rs3x3s2", "depthwise", "f16", 1, 33, 34, 96, 96, 3, 3, 2, 1, 1, seed=310), {}),
    (P("f16_rs5x3s3", "depthwise", "f16", 1, 22, 19, 16, 16, 5, 3, 3, 2, 1, seed=311), {}),
    (P("f16_rs7x7s2_generic", "depthwise", "f16", 1, 30, 31, 32, 32, 7, 7, 2, 0, 0, seed=312),
     {"DGRAD_RS_GENERIC": "1"}),
]


@pytest.mark.parametrize("p,env", DW_F16, ids=[p.name for p, _ in DW_F16])
def test_depthwise_f16(p, env, monkeypatch):
    """fp16 I/O on the FMA depthwise kernels (dgrad_depthwise): every kernel family,
    f16 widened to fp32 on load, dX rounded once to f16."""
    h = _h()
    for k, v in env.items():
        monkeypatch.setenv(k, v)
    inp = synthetic.make_inputs(p)
    dy, w = h.to_dev(inp)
    got = h.gpu_to_np(h.run_gpu(p, dy, w))
    ref = h.oracle_full(p, inp.dy, inp.w)
    absref = h.oracle_full(p, np.abs(inp.dy), np.abs(inp.w))
    h.check(p, got, ref, absref, what=p.name)
    import convolution_backward_b200 as cb
    cb.check_status()


SPLITK = [
    (P("sk_small_m", "pointwise", "bf16", 2, 14, 14, 512, 2048, seed=91), [1, 2, 5, 0]),
    (P("sk_ragged", "pointwise", "bf16", 1, 7, 9, 136, 1000, seed=92), [3, 16, 0]),
    (P("sk_one_tile", "pointwise", "bf16", 1, 4, 4, 64, 4096, seed=93), [8, 64, 0]),
    (P("sk_k_lt_64", "pointwise", "bf16", 3, 5, 5, 264, 40, seed=94), [1, 0]),
    (P("sk_f16_small_m", "pointwise", "f16", 2, 14, 14, 512, 2048, seed=95), [2, 0]),
    (P("sk_f16_ragged", "pointwise", "f16", 1, 7, 9, 136, 1000, seed=96), [3, 0]),
]
SPLITK_CASES = [(p, s) for p, ss in SPLITK for s in ss]


@pytest.mark.parametrize("p,splits", SPLITK_CASES, ids=[f"{p.name}-s{s}" for p, s in SPLITK_CASES])
def test_pointwise_splitk(p, splits):
    """Split-K tcgen05 pointwise (NEXT-4), bf16 and f16: partial tiles in a caller workspace,
    deterministic reduction."""
    h = _h()
    import convolution_backward_b200 as cb
    inp = synthetic.make_inputs(p)
    dy, w = h.to_dev(inp)
    nbytes, used = cb.splitk_workspace_bytes(p.N, p.H, p.W, p.K, p.C, splits)
    ws = torch.full((nbytes // 4 + 4,), float("nan"), dtype=torch.float32, device="cuda")   # contents must not matter
    out = cb.pointwise_splitk(dy, w, splits=splits, workspace=ws)
    got = h.gpu_to_np(out)
    ref = h.oracle_full(p, inp.dy, inp.w)
    absref = h.oracle_full(p, np.abs(inp.dy), np.abs(inp.w))
    h.check(p, got, ref, absref, what=f"{p.name}/splits={splits}({used})")
    again = cb.pointwise_splitk(dy, w, splits=splits, workspace=ws)
    assert torch.equal(out, again)                      # deterministic
    cb.check_status()


TC_SMALL = [
    P("tc3x3", "depthwise", "bf16", 1, 10, 9, 8, 8, 3, 3, 1, 1, 1, seed=141),
    P("tc5x11_ragged_images", "depthwise", "bf16", 9, 7, 70, 8, 8, 5, 11, 1, 2, 5, seed=142),
    P("tc11x4_long_h", "depthwise", "bf16", 2, 70, 12, 8, 8, 11, 4, 1, 0, 3, seed=143),
    P("tc31x31", "depthwise", "bf16", 3, 20, 20, 16, 16, 31, 31, 1, 15, 15, seed=144),
    P("tc13x5", "depthwise", "bf16", 2, 16, 16, 8, 8, 13, 5, 1, 6, 2, seed=145),
    P("tc5x13", "depthwise", "bf16", 2, 16, 16, 8, 8, 5, 13, 1, 2, 6, seed=146),
    P("tc3x3_two_by_two_tiles", "depthwise", "bf16", 1, 70, 70, 8, 8, 3, 3, 1, 1, 1, seed=147),
    P("tc41x41", "depthwise", "bf16", 1, 12, 12, 8, 8, 41, 41, 1, 20, 20, seed=148),
    P("tc51x51_half_tile", "depthwise", "bf16", 1, 64, 64, 8, 8, 51, 51, 1, 25, 25, seed=149),
    P("tc31x31_c40", "depthwise", "bf16", 1, 37, 45, 40, 40, 31, 31, 1, 15, 15, seed=150),
    P("tc7x7_nonsame", "depthwise", "bf16", 2, 17, 18, 16, 16, 7, 7, 1, 1, 5, seed=151),
    P("tc1x1", "depthwise", "bf16", 2, 5, 6, 16, 16, 1, 1, 1, 0, 0, seed=152),
    P("tc51x5", "depthwise", "bf16", 1, 45, 30, 24, 24, 51, 5, 1, 25, 2, seed=153),
    P("tc64x64", "depthwise", "bf16", 1, 70, 66, 8, 8, 64, 64, 1, 32, 31, seed=155),
    P("tc17x17_nonsame", "depthwise", "bf16", 10, 40, 33, 16, 16, 17, 17, 1, 3, 11, seed=156),
    P("tc11x9_c136_ragged_x", "depthwise", "bf16", 3, 37, 70, 136, 136, 11, 9, 1, 5, 4, seed=157),
    P("tc9x9_tail_split", "depthwise", "bf16", 8, 20, 24, 152, 152, 9, 9, 1, 4, 4, seed=161),   # 152 planes
    P("tc31x31_f16", "depthwise", "f16", 3, 20, 20, 16, 16, 31, 31, 1, 15, 15, seed=162),
    P("tc51x5_f16", "depthwise", "f16", 1, 45, 30, 24, 24, 51, 5, 1, 25, 2, seed=163),
    P("tc9x21_c64_long_w", "depthwise", "bf16", 9, 66, 45, 64, 64, 9, 21, 1, 4, 10, seed=158),
    P("tc21x9_c192_long_h", "depthwise", "bf16", 2, 45, 67, 192, 192, 21, 9, 1, 10, 4, seed=159),
    P("tc5x51", "depthwise", "bf16", 1, 30, 45, 24, 24, 5, 51, 1, 2, 25, seed=154),
]


@pytest.mark.parametrize("p", TC_SMALL, ids=[p.name for p in TC_SMALL])
def test_depthwise_tensor_core(p):
    """Stride-1 depthwise on tcgen05 (banded-Toeplitz GEMMs, §8 NEXT-2) against the oracle; the
    workspace starts as NaN (its contents must not matter) and a second call gives identical bits."""
    h = _h()
    import convolution_backward_b200 as cb
    inp = synthetic.make_inputs(p)
    dy, w = h.to_dev(inp)
    nb = cb.depthwise_tc_workspace_bytes(p.N, p.H, p.W, p.C, p.KH, p.KW, p.pad_h, p.pad_w)
    ws = torch.full((nb // 2 + 8,), float("nan"), dtype=torch.bfloat16, device="cuda")
    out = cb.depthwise_tc(dy, w, H=p.H, Wd=p.W, pad_h=p.pad_h, pad_w=p.pad_w, workspace=ws)
    got = h.gpu_to_np(out)
    ref = h.oracle_full(p, inp.dy, inp.w)
    absref = h.oracle_full(p, np.abs(inp.dy), np.abs(inp.w))
    h.check(p, got, ref, absref, what=f"{p.name}/tc")
    again = cb.depthwise_tc(dy, w, H=p.H, Wd=p.W, pad_h=p.pad_h, pad_w=p.pad_w, workspace=ws)
    assert torch.equal(out, again)
    cb.check_status()


RS_FAST = [
    P("rs7x7s2_p3", "depthwise", "bf16", 2, 29, 27, 40, 40, 7, 7, 2, 3, 3, seed=71),
    P("rs7x7s2_p0", "depthwise", "bf16", 1, 30, 31, 32, 32, 7, 7, 2, 0, 0, seed=72),
    P("rs7x7s2_p6x1", "depthwise", "bf16", 1, 23, 40, 16, 16, 7, 7, 2, 6, 1, seed=73),
    P("rs7x7s2_wide", "depthwise", "bf16", 1, 12, 130, 64, 64, 7, 7, 2, 3, 3, seed=74),
    P("rs7x7s2_tall", "depthwise", "bf16", 1, 117, 9, 8, 8, 7, 7, 2, 3, 2, seed=75),
    P("rs5x5s2", "depthwise", "bf16", 2, 25, 26, 48, 48, 5, 5, 2, 2, 2, seed=76),
    P("rs3x3s2_p1", "depthwise", "bf16", 1, 33, 34, 96, 96, 3, 3, 2, 1, 1, seed=77),
    P("rs3x3s2_p0", "depthwise", "bf16", 1, 16, 17, 32, 32, 3, 3, 2, 0, 0, seed=78),
    P("rs7x7s2_tiny", "depthwise", "bf16", 1, 2, 3, 8, 8, 7, 7, 2, 3, 3, seed=79),
]


RS_VARIANTS = [("0", "reg", ""), ("0", "reg", "q4"), ("0", "reg", "direct"), ("0", "smem", ""), ("0", "smem", "alt"),
               ("1", "", "")]


@pytest.mark.parametrize("generic,kern,g", RS_VARIANTS,
                         ids=["reg-ring", "reg-ring-q4", "reg-ring-direct-stores", "smem-ring", "smem-ring-altG",
                              "generic"])
@pytest.mark.parametrize("p", RS_FAST, ids=[p.name for p in RS_FAST])
def test_rowstream_paths(p, generic, kern, g, monkeypatch):
    """Strided depthwise through every row-streaming kernel: accumulator ring in
    registers (two and four output columns per thread; final rows stored by TMA from
    shared memory, or stored directly), ring in shared memory (both step depths G), and
    the generic one."""
    h = _h()
    monkeypatch.setenv("DGRAD_RS_GENERIC", generic)
    if kern:
        monkeypatch.setenv("DGRAD_RS_KERNEL", kern)
    if g == "alt":
        monkeypatch.setenv("DGRAD_RS_G", {7: "1", 5: "1", 3: "2"}[p.KH])
    if g == "q4":
        monkeypatch.setenv("DGRAD_RS_Q", "4")
    if g == "direct":
        monkeypatch.setenv("DGRAD_RS_STORE", "direct")
    inp = synthetic.make_inputs(p)
    dy, w = h.to_dev(inp)
    got = h.gpu_to_np(h.run_gpu(p, dy, w))
    ref = h.oracle_full(p, inp.dy, inp.w)
    absref = h.oracle_full(p, np.abs(inp.dy), np.abs(inp.w))
    h.check(p, got, ref, absref, what=f"{p.name}/generic={generic}")
    import convolution_backward_b200 as cb
    cb.check_status()


def _torch_fp32_reference(p, dy, w):
    """dgrad by cuDNN / cuBLAS in fp32 with TF32 off (full-tensor property check)."""
    torch.backends.cudnn.allow_tf32 = False
    torch.backends.cuda.matmul.allow_tf32 = False
    dyf = dy.float()
    wf = w.float()
    if p.kind == "pointwise":
        return (dyf.reshape(-1, p.K) @ wf).reshape(p.N, p.H, p.W, p.C)
    wt = wf.permute(2, 0, 1).reshape(p.C, 1, p.KH, p.KW).contiguous()
    out = torch.nn.grad.conv2d_input((p.N, p.C, p.H, p.W), wt, dyf.permute(0, 3, 1, 2).contiguous(),
                                     stride=p.stride, padding=(p.pad_h, p.pad_w), groups=p.C)
    return out.permute(0, 2, 3, 1)


FULL = synthetic.all_problems()


@pytest.mark.parametrize("p", FULL, ids=[p.name for p in FULL])
def test_full_size_workloads(p):
    h = _h()
    inp = synthetic.make_inputs(p)
    dy, w = h.to_dev(inp)
    out = h.run_gpu(p, dy, w)
    torch.cuda.synchronize()
    if p.name == "pw_f32_small":
        got = h.gpu_to_np(out)
        ref = h.oracle_full(p, inp.dy, inp.w)
        absref = h.oracle_full(p, np.abs(inp.dy), np.abs(inp.w))
        h.check(p, got, ref, absref, what=p.name)
        return
    pts = h.sample_points(p, 3000)
    got = out.float()[pts[:, 0], pts[:, 1], pts[:, 2], pts[:, 3]].cpu().numpy().astype(np.float64)
    ref = h.oracle_points(p, inp.dy, inp.w, pts)
    absref = h.oracle_points(p, np.abs(inp.dy), np.abs(inp.w), pts)
    h.check(p, got, ref, absref, what=f"{p.name} sampled")
    # every element against cuDNN/cuBLAS fp32 with the normwise bar
    tref = _torch_fp32_reference(p, dy, w)
    err = (out.float() - tref).abs().max().item()
    assert err / (tref.abs().max().item() + 1e-6) <= 1e-2
    import convolution_backward_b200 as cb
    cb.check_status()


@pytest.mark.parametrize("p", [q for q in TC_SMALL if q.C >= 64], ids=[q.name for q in TC_SMALL if q.C >= 64])
def test_depthwise_tensor_core_cuda_transposes(p, monkeypatch):
    """The tensor-core path with its transposes on CUDA cores (DGRAD_TC_TRANSPOSE=cuda) instead of TMA."""
    h = _h()
    import convolution_backward_b200 as cb
    monkeypatch.setenv("DGRAD_TC_TRANSPOSE", "cuda")
    inp = synthetic.make_inputs(p)
    dy, w = h.to_dev(inp)
    out = cb.depthwise_tc(dy, w, H=p.H, Wd=p.W, pad_h=p.pad_h, pad_w=p.pad_w)
    got = h.gpu_to_np(out)
    ref = h.oracle_full(p, inp.dy, inp.w)
    absref = h.oracle_full(p, np.abs(inp.dy), np.abs(inp.w))
    h.check(p, got, ref, absref, what=f"{p.name}/cuda transposes")
    cb.check_status()


DENSE = [
    P("dense3x3_s1", "dense", "bf16", 2, 13, 21, 72, 40, 3, 3, 1, 1, 1, seed=171),
    P("dense1x1_s1", "dense", "bf16", 1, 9, 11, 64, 128, 1, 1, 1, 0, 0, seed=172),
    P("dense5x3_s1_nonsame", "dense", "bf16", 3, 17, 10, 136, 24, 5, 3, 1, 1, 2, seed=173),
    P("dense7x7_s1", "dense", "bf16", 1, 20, 19, 64, 64, 7, 7, 1, 3, 3, seed=174),
    P("dense3x3_s2", "dense", "bf16", 2, 15, 17, 48, 80, 3, 3, 2, 1, 1, seed=175),
    P("dense4x4_s2_even", "dense", "bf16", 1, 16, 18, 32, 16, 4, 4, 2, 1, 1, seed=176),
    P("dense1x1_s2", "dense", "bf16", 2, 14, 15, 40, 56, 1, 1, 2, 0, 0, seed=177),
    P("dense7x7_s2", "dense", "bf16", 1, 23, 22, 24, 32, 7, 7, 2, 3, 3, seed=178),
    P("dense5x5_s3", "dense", "bf16", 2, 19, 20, 16, 24, 5, 5, 3, 2, 2, seed=179),
    P("dense2x3_s2_gaps", "dense", "bf16", 1, 13, 14, 8, 8, 2, 3, 3, 0, 1, seed=180),
    P("dense3x3_k200_c264", "dense", "bf16", 1, 9, 9, 264, 200, 3, 3, 1, 1, 1, seed=181),
]


@pytest.mark.parametrize("bn", ["64", "128", "256"])
@pytest.mark.parametrize("p", DENSE, ids=[p.name for p in DENSE])
def test_dense_tensor_core(p, bn, monkeypatch):
    """Dense (ungrouped) KxK dgrad on tcgen05 by output phase (§8 NEXT-1), every channel tile width,
    against the oracle on whole outputs: strides 1-3, odd and even filters, padding that is not
    'same', ragged K, C, extents and tile edges."""
    h = _h()
    import convolution_backward_b200 as cb
    monkeypatch.setenv("DGRAD_DENSE_BN", bn)
    inp = synthetic.make_inputs(p)
    dy, w = h.to_dev(inp)
    got = h.gpu_to_np(h.run_gpu(p, dy, w))
    ref = h.oracle_full(p, inp.dy, inp.w)
    absref = h.oracle_full(p, np.abs(inp.dy), np.abs(inp.w))
    h.check(p, got, ref, absref, what=f"{p.name}/bn={bn}")
    cb.check_status()


GROUPED = [
    # grouped pointwise (1x1): per-group dY columns, W [K][C/groups]
    P("grouped1x1_g4", "grouped", "bf16", 2, 13, 17, 64, 128, seed=191).replace(ngroups=4),
    P("grouped1x1_g2_ragged", "grouped", "bf16", 1, 9, 23, 272, 144, seed=192).replace(ngroups=2),
    P("grouped1x1_g16_small", "grouped", "bf16", 1, 7, 9, 128, 256, seed=193).replace(ngroups=16),
    P("grouped3x3_g2", "grouped", "bf16", 2, 11, 14, 48, 80, 3, 3, 1, 1, 1, seed=194).replace(ngroups=2),
    P("grouped3x3_s2_g4", "grouped", "bf16", 1, 15, 16, 64, 32, 3, 3, 2, 1, 1, seed=195).replace(ngroups=4),
    P("grouped5x5_g8_k8", "grouped", "bf16", 1, 12, 13, 64, 64, 5, 5, 1, 2, 2, seed=196).replace(ngroups=8),
    # fp16 I/O
    P("dense3x3_f16", "dense", "f16", 2, 13, 21, 72, 40, 3, 3, 1, 1, 1, seed=197),
    P("grouped1x1_f16_g4", "grouped", "f16", 1, 11, 13, 128, 64, seed=198).replace(ngroups=4),
    P("dense3x3_s2_f16", "dense", "f16", 1, 15, 17, 48, 80, 3, 3, 2, 1, 1, seed=199),
]


@pytest.mark.parametrize("p", GROUPED, ids=[p.name for p in GROUPED])
def test_grouped_and_f16_tensor_core(p):
    """Grouped dgrad (1x1 = the grouped pointwise fast path) and fp16 I/O through the tap kernel (§8 NEXT-3),
    against the oracle on whole outputs."""
    h = _h()
    import convolution_backward_b200 as cb
    inp = synthetic.make_inputs(p)
    dy, w = h.to_dev(inp)
    got = h.gpu_to_np(h.run_gpu(p, dy, w))
    ref = h.oracle_full(p, inp.dy, inp.w)
    absref = h.oracle_full(p, np.abs(inp.dy), np.abs(inp.w))
    h.check(p, got, ref, absref, what=p.name)
    cb.check_status()


# fp32 pointwise on both tile heights: 64-row tiles (>= 64 tiles: 4096 and 4160+5 rows) and
# 16-row tiles (fewer tiles: 392 rows as in the small fp32 workload, and a ragged 77-row case)
PW_F32_TILES = [P("pw_f32_tall", "pointwise", "f32", 4, 32, 32, 64, 48, seed=191),
                P("pw_f32_tall_ragged", "pointwise", "f32", 5, 29, 29, 68, 36, seed=192),
                P("pw_f32_392", "pointwise", "f32", 2, 14, 14, 64, 64, seed=193),
                P("pw_f32_77", "pointwise", "f32", 1, 7, 11, 24, 20, seed=194)]


@pytest.mark.parametrize("p", PW_F32_TILES, ids=[q.name for q in PW_F32_TILES])
def test_pointwise_f32_tile_heights(p):
    """The fp32 FMA pointwise kernel with 64-row and with 16-row tiles against the oracle, every element
    within the fp32 bound."""
    h = _h()
    import convolution_backward_b200 as cb
    inp = synthetic.make_inputs(p)
    dy, w = h.to_dev(inp)
    got = h.gpu_to_np(h.run_gpu(p, dy, w))
    ref = h.oracle_full(p, inp.dy, inp.w)
    absref = h.oracle_full(p, np.abs(inp.dy), np.abs(inp.w))
    h.check(p, got, ref, absref, what=p.name)
    cb.check_status()


@pytest.mark.parametrize("shape", [(2, 13, 23, 264, 200), (1, 9, 11, 64, 512), (3, 7, 5, 8, 8)])
def test_pointwise_f16(shape):
    """dgrad_pointwise with fp16 I/O (routed to the tap kernel with one 1x1 tap)."""
    h = _h()
    import convolution_backward_b200 as cb
    N, H, W, C, K = shape
    p = P("pw_f16", "pointwise", "f16", N, H, W, C, K, seed=61)
    inp = synthetic.make_inputs(p)
    dy, w = h.to_dev(inp)
    got = h.gpu_to_np(cb.pointwise(dy, w))
    ref = h.oracle_full(p, inp.dy, inp.w)
    absref = h.oracle_full(p, np.abs(inp.dy), np.abs(inp.w))
    h.check(p, got, ref, absref, what=f"pointwise f16 {shape}")
    cb.check_status()


DENSE_LARGE = [P("dense3x3_s1_large", "dense", "bf16", 8, 28, 28, 256, 256, 3, 3, 1, 1, 1, seed=182),
               P("dense3x3_s2_large", "dense", "bf16", 8, 56, 56, 128, 256, 3, 3, 2, 1, 1, seed=183)]


@pytest.mark.parametrize("p", DENSE_LARGE, ids=[p.name for p in DENSE_LARGE])
def test_dense_tensor_core_sampled(p):
    """Larger dense problems (many tiles and k-blocks): sampled oracle points and every element against
    cuDNN in fp32."""
    h = _h()
    import convolution_backward_b200 as cb
    inp = synthetic.make_inputs(p)
    dy, w = h.to_dev(inp)
    out = h.run_gpu(p, dy, w)
    torch.cuda.synchronize()
    pts = h.sample_points(p, 2000)
    got = out.float()[pts[:, 0], pts[:, 1], pts[:, 2], pts[:, 3]].cpu().numpy().astype(np.float64)
    ref = h.oracle_points(p, inp.dy, inp.w, pts)
    absref = h.oracle_points(p, np.abs(inp.dy), np.abs(inp.w), pts)
    h.check(p, got, ref, absref, what=f"{p.name} sampled")
    wt = w.float().permute(2, 3, 0, 1).contiguous()      # (K, C, KH, KW): the forward weight
    tref = torch.nn.grad.conv2d_input((p.N, p.C, p.H, p.W), wt, dy.float().permute(0, 3, 1, 2).contiguous(),
                                      stride=p.stride, padding=(p.pad_h, p.pad_w)).permute(0, 2, 3, 1)
    err = (out.float() - tref).abs().max().item()
    assert err / (tref.abs().max().item() + 1e-6) <= 1e-2
    cb.check_status()


TC_TILES = ["0,2,32,1", "0,2,16,1", "0,4,16,2", "0,4,8,2", "0,8,8,4", "0,8,4,4", "1,4,16,2", "1,8,8,4"]


@pytest.mark.parametrize("tile", TC_TILES)
def test_depthwise_tensor_core_tile_shapes(tile, monkeypatch):
    """Every tile shape of the tensor-core depthwise kernel (orientation, row phases P, row groups NH,
    sub-tiles XT), forced through DGRAD_TC_TILE, on a ragged problem (N = 9, odd extents)."""
    h = _h()
    import convolution_backward_b200 as cb
    monkeypatch.setenv("DGRAD_TC_TILE", tile)
    p = P("tc_tile", "depthwise", "bf16", 9, 37, 41, 24, 24, 9, 7, 1, 4, 3, seed=160)
    inp = synthetic.make_inputs(p)
    dy, w = h.to_dev(inp)
    out = cb.depthwise_tc(dy, w, H=p.H, Wd=p.W, pad_h=p.pad_h, pad_w=p.pad_w)
    got = h.gpu_to_np(out)
    ref = h.oracle_full(p, inp.dy, inp.w)
    absref = h.oracle_full(p, np.abs(inp.dy), np.abs(inp.w))
    h.check(p, got, ref, absref, what=f"tile {tile}")
    cb.check_status()


TC_A_TMEM = [q for q in TC_SMALL if q.name in ("tc31x31", "tc51x5", "tc5x51", "tc17x17_nonsame", "tc64x64",
                                                 "tc11x9_c136_ragged_x", "tc31x31_f16")]


_TILE_PROBLEM = P("tc_tile", "depthwise", "bf16", 9, 37, 41, 24, 24, 9, 7, 1, 4, 3, seed=160)
TC_A_TMEM_CASES = [(q, "auto") for q in TC_A_TMEM] + [(_TILE_PROBLEM, t) for t in TC_TILES]


@pytest.mark.parametrize("case", TC_A_TMEM_CASES, ids=[f"{q.name}-{t}" for q, t in TC_A_TMEM_CASES])
def test_depthwise_tensor_core_a_in_tensor_memory(case, monkeypatch):
    """The planar tensor-core kernel with its Toeplitz operand A_i written into tensor memory by the
    builder warps (DGRAD_TC_A=tmem), the layout it falls back to when the shared-memory tables do not
    fit: the default tile of several problems, and every tile shape on a ragged problem."""
    p, tile = case
    h = _h()
    import convolution_backward_b200 as cb
    monkeypatch.setenv("DGRAD_TC_A", "tmem")
    if tile != "auto":
        monkeypatch.setenv("DGRAD_TC_TILE", tile)
    inp = synthetic.make_inputs(p)
    dy, w = h.to_dev(inp)
    out = cb.depthwise_tc(dy, w, H=p.H, Wd=p.W, pad_h=p.pad_h, pad_w=p.pad_w)
    got = h.gpu_to_np(out)
    ref = h.oracle_full(p, inp.dy, inp.w)
    absref = h.oracle_full(p, np.abs(inp.dy), np.abs(inp.w))
    h.check(p, got, ref, absref, what=f"{p.name}/A in tensor memory, tile {tile}")
    cb.check_status()


# More than 8 images (two or more image groups, ragged), two row tiles, two B panels (K clipped
# to 80), both orientations, f16.
TC_MANY_IMAGES = [
    P("tcn16_31x31", "depthwise", "bf16", 16, 20, 20, 16, 16, 31, 31, 1, 15, 15, seed=171),
    P("tcn13_9x7", "depthwise", "bf16", 13, 28, 36, 24, 24, 9, 7, 1, 4, 3, seed=172),
    P("tcn17_11x5_two_row_tiles", "depthwise", "bf16", 17, 100, 40, 8, 8, 11, 5, 1, 5, 2, seed=173),
    P("tcn10_5x9_two_panels", "depthwise", "bf16", 10, 68, 64, 8, 8, 5, 9, 1, 2, 8, seed=174),
    P("tcn12_51x5", "depthwise", "bf16", 12, 64, 64, 16, 16, 51, 5, 1, 25, 2, seed=175),
    P("tcn12_5x51", "depthwise", "bf16", 12, 64, 64, 16, 16, 5, 51, 1, 2, 25, seed=176),
    P("tcn11_17x17_f16", "depthwise", "f16", 11, 32, 48, 24, 24, 17, 17, 1, 8, 8, seed=177),
    P("tcn9_3x3_c40", "depthwise", "bf16", 9, 16, 24, 40, 40, 3, 3, 1, 1, 1, seed=178),
]


@pytest.mark.parametrize("amode", ["smem", "tmem"])
@pytest.mark.parametrize("p", TC_MANY_IMAGES, ids=[q.name for q in TC_MANY_IMAGES])
def test_depthwise_tensor_core_many_images(p, amode, monkeypatch):
    """The planar tensor-core kernel on problems with several image groups, with A_i as shared-memory
    tables (DGRAD_TC_A=smem) and in tensor memory (DGRAD_TC_A=tmem), against the oracle on every
    element; dX starts as NaN and a second call gives identical bits."""
    h = _h()
    import convolution_backward_b200 as cb
    monkeypatch.setenv("DGRAD_TC_A", amode)
    inp = synthetic.make_inputs(p)
    dy, w = h.to_dev(inp)
    out = torch.full(p.dx_shape, float("nan"), dtype=dy.dtype, device=dy.device)
    cb.depthwise_tc(dy, w, H=p.H, Wd=p.W, pad_h=p.pad_h, pad_w=p.pad_w, out=out)
    again = cb.depthwise_tc(dy, w, H=p.H, Wd=p.W, pad_h=p.pad_h, pad_w=p.pad_w)
    cb.check_status()
    assert torch.equal(out, again), f"{p.name}: two calls differ"
    got = h.gpu_to_np(out)
    ref = h.oracle_full(p, inp.dy, inp.w)
    absref = h.oracle_full(p, np.abs(inp.dy), np.abs(inp.w))
    h.check(p, got, ref, absref, what=f"{p.name}/A in {amode}")


# B-block layouts of the planar kernel: by default the blocks share the rows of zero padding
# above and below the image (written once by the kernel); DGRAD_TC_SHZ=0 gives each block its
# own, loaded by the TMA with the image rows.  Fewer shared-memory tables (DGRAD_TC_NA), with one or
# two filter-line buffers (DGRAD_TC_NFB), are the other layouts the planner can reach.
TC_LAYOUT_PROBLEMS = [q for q in TC_SMALL if q.name in ("tc31x31", "tc31x31_c40", "tc51x5", "tc17x17_nonsame",
                                                        "tc7x7_nonsame", "tc41x41")] + \
    [q for q in TC_MANY_IMAGES if q.name in ("tcn16_31x31", "tcn13_9x7", "tcn12_5x51")]
TC_LAYOUTS = {"own_zero_rows": {"DGRAD_TC_SHZ": "0"},
              "whole_tiles_per_cta": {"DGRAD_TC_SPLIT": "0"},
              "one_staging_box_per_half": {"DGRAD_TC_STG": "1"},
              "4_tables": {"DGRAD_TC_NA": "4"},
              "5_tables": {"DGRAD_TC_NA": "5"},
              "one_filter_buffer_4_tables": {"DGRAD_TC_NFB": "1", "DGRAD_TC_NA": "4"}}


@pytest.mark.parametrize("layout", list(TC_LAYOUTS))
@pytest.mark.parametrize("p", TC_LAYOUT_PROBLEMS, ids=[q.name for q in TC_LAYOUT_PROBLEMS])
def test_depthwise_tensor_core_b_layouts(p, layout, monkeypatch):
    """The planar tensor-core kernel with each B-block and table layout, against the oracle on every
    element; the workspace starts as NaN, and a call with the default layout gives identical bits."""
    h = _h()
    import convolution_backward_b200 as cb
    inp = synthetic.make_inputs(p)
    dy, w = h.to_dev(inp)
    nb = cb.depthwise_tc_workspace_bytes(p.N, p.H, p.W, p.C, p.KH, p.KW, p.pad_h, p.pad_w)
    ws = torch.full((nb // 2 + 8,), float("nan"), dtype=torch.bfloat16, device="cuda")
    base = cb.depthwise_tc(dy, w, H=p.H, Wd=p.W, pad_h=p.pad_h, pad_w=p.pad_w)
    for k, v in TC_LAYOUTS[layout].items():
        monkeypatch.setenv(k, v)
    out = cb.depthwise_tc(dy, w, H=p.H, Wd=p.W, pad_h=p.pad_h, pad_w=p.pad_w, workspace=ws)
    cb.check_status()
    got = h.gpu_to_np(out)
    ref = h.oracle_full(p, inp.dy, inp.w)
    absref = h.oracle_full(p, np.abs(inp.dy), np.abs(inp.w))
    h.check(p, got, ref, absref, what=f"{p.name}/{layout}")
    assert torch.equal(out, base), f"{p.name}: {layout} differs from the default layout"


# Balanced shift-step ranges: with A tables the CTAs take equal ranges of shift steps, and a tile
# two CTAs share passes an fp32 partial through the workspace.  DGRAD_TC_GRID caps the grid so that
# these small problems have more tiles than CTAs and split at many different steps.
TC_SPLIT_PROBLEMS = [q for q in TC_SMALL if q.name in ("tc31x31", "tc31x31_c40", "tc17x17_nonsame", "tc41x41",
                                                       "tc31x31_f16")] + \
    [q for q in TC_MANY_IMAGES if q.name in ("tcn16_31x31", "tcn11_17x17_f16")]


@pytest.mark.parametrize("transpose", ["tma", "cuda"])
@pytest.mark.parametrize("grid", [2, 3, 5, 7])
@pytest.mark.parametrize("p", TC_SPLIT_PROBLEMS, ids=[q.name for q in TC_SPLIT_PROBLEMS])
def test_depthwise_tensor_core_split_steps(p, grid, transpose, monkeypatch):
    """The planar tensor-core kernel with tiles split between CTAs at shift-step boundaries (a few
    CTAs for many tiles), through the TMA and the CUDA-core transposes (each clears the split flags),
    against the oracle on every element; the workspace starts as NaN and a second call gives
    identical bits."""
    h = _h()
    import convolution_backward_b200 as cb
    monkeypatch.setenv("DGRAD_TC_GRID", str(grid))
    if transpose == "cuda":
        monkeypatch.setenv("DGRAD_TC_TRANSPOSE", "cuda")
    inp = synthetic.make_inputs(p)
    dy, w = h.to_dev(inp)
    nb = cb.depthwise_tc_workspace_bytes(p.N, p.H, p.W, p.C, p.KH, p.KW, p.pad_h, p.pad_w)
    ws = torch.full((nb // 2 + 8,), float("nan"), dtype=torch.bfloat16, device="cuda")
    out = cb.depthwise_tc(dy, w, H=p.H, Wd=p.W, pad_h=p.pad_h, pad_w=p.pad_w, workspace=ws)
    again = cb.depthwise_tc(dy, w, H=p.H, Wd=p.W, pad_h=p.pad_h, pad_w=p.pad_w, workspace=ws)
    cb.check_status()
    assert torch.equal(out, again), f"{p.name}: two calls differ"
    got = h.gpu_to_np(out)
    ref = h.oracle_full(p, inp.dy, inp.w)
    absref = h.oracle_full(p, np.abs(inp.dy), np.abs(inp.w))
    h.check(p, got, ref, absref, what=f"{p.name}/split over {grid} CTAs ({transpose} transposes)")


TC_AUTO = [q for q in TC_SMALL if q.KH * q.KW > 49]


@pytest.mark.parametrize("p", TC_AUTO, ids=[q.name for q in TC_AUTO])
def test_depthwise_auto_tensor_core_nhwc(p):
    """dgrad_depthwise's automatic choice for large 16-bit stride-1 filters: the tensor-core kernel that
    reads NHWC dY and writes NHWC dX with no workspace (clusters of 8 channels), against the oracle on
    every element; dX starts as NaN and a second call gives identical bits."""
    h = _h()
    import convolution_backward_b200 as cb
    inp = synthetic.make_inputs(p)
    dy, w = h.to_dev(inp)
    out = torch.full(p.dx_shape, float("nan"), dtype=dy.dtype, device=dy.device)
    cb.depthwise(dy, w, H=p.H, Wd=p.W, pad_h=p.pad_h, pad_w=p.pad_w, out=out)
    again = cb.depthwise(dy, w, H=p.H, Wd=p.W, pad_h=p.pad_h, pad_w=p.pad_w)
    cb.check_status()
    assert torch.equal(out, again), f"{p.name}: two calls differ"
    got = h.gpu_to_np(out)
    ref = h.oracle_full(p, inp.dy, inp.w)
    absref = h.oracle_full(p, np.abs(inp.dy), np.abs(inp.w))
    h.check(p, got, ref, absref, what=f"{p.name}/auto")


@pytest.mark.parametrize("tile", TC_TILES)
def test_depthwise_auto_tensor_core_tile_shapes(tile, monkeypatch):
    """Every tile shape of the NHWC tensor-core kernel behind dgrad_depthwise (forced through
    DGRAD_TC_TILE) on a ragged problem: N = 9 (a partial image group), odd extents (a ragged last
    8-column group), several row tiles for the smaller shapes."""
    h = _h()
    import convolution_backward_b200 as cb
    monkeypatch.setenv("DGRAD_TC_TILE", tile)
    p = P("tc_tile_auto", "depthwise", "bf16", 9, 37, 41, 24, 24, 9, 7, 1, 4, 3, seed=160)
    inp = synthetic.make_inputs(p)
    dy, w = h.to_dev(inp)
    out = cb.depthwise(dy, w, H=p.H, Wd=p.W, pad_h=p.pad_h, pad_w=p.pad_w)
    got = h.gpu_to_np(out)
    ref = h.oracle_full(p, inp.dy, inp.w)
    absref = h.oracle_full(p, np.abs(inp.dy), np.abs(inp.w))
    h.check(p, got, ref, absref, what=f"auto tile {tile}")
    cb.check_status()


TC_FULL = [p for p in synthetic.all_problems() if p.variant == "tc"]


@pytest.mark.parametrize("entry", ["tc", "auto"])
@pytest.mark.parametrize("p", TC_FULL, ids=[p.name for p in TC_FULL])
def test_full_size_tensor_core_depthwise(p, entry):
    """The large stride-1 workloads through dgrad_depthwise_tc (planar, with a workspace: what the
    benchmark runs) and through dgrad_depthwise's automatic choice (NHWC, no workspace): sampled
    oracle points, and every element against cuDNN fp32."""
    h = _h()
    import convolution_backward_b200 as cb
    inp = synthetic.make_inputs(p)
    dy, w = h.to_dev(inp)
    if entry == "tc":
        out = cb.depthwise_tc(dy, w, H=p.H, Wd=p.W, pad_h=p.pad_h, pad_w=p.pad_w)
    else:
        out = cb.depthwise(dy, w, H=p.H, Wd=p.W, pad_h=p.pad_h, pad_w=p.pad_w)
    torch.cuda.synchronize()
    pts = h.sample_points(p, 3000)
    got = out.float()[pts[:, 0], pts[:, 1], pts[:, 2], pts[:, 3]].cpu().numpy().astype(np.float64)
    ref = h.oracle_points(p, inp.dy, inp.w, pts)
    absref = h.oracle_points(p, np.abs(inp.dy), np.abs(inp.w), pts)
    h.check(p, got, ref, absref, what=f"{p.name} sampled")
    tref = _torch_fp32_reference(p, dy, w)
    err = (out.float() - tref).abs().max().item()
    assert err / (tref.abs().max().item() + 1e-6) <= 1e-2
    cb.check_status()


def test_guard_bands_untouched():
    """dX sits between NaN canary bands; the kernels must write exactly dX."""
    h = _h()
    import convolution_backward_b200 as cb
    for p, mode in [(SMALL[0], "auto"), (SMALL[7], "auto"), (SMALL[7], "rowstream"), (SMALL[20], "auto"),
                    (SMALL[5], "auto")]:
        inp = synthetic.make_inputs(p)
        dy, w = h.to_dev(inp)
        n = int(np.prod(p.dx_shape))
        band = 4096
        dt = torch.bfloat16 if p.dtype == "bf16" else torch.float32
        buf = torch.full((band + n + band,), float("nan"), dtype=dt, device="cuda")
        out = buf[band:band + n].view(p.dx_shape)
        h.run_gpu(p, dy, w, mode=mode, out=out)
        torch.cuda.synchronize()
        assert torch.isnan(buf[:band]).all() and torch.isnan(buf[band + n:]).all(), p.name
        assert not torch.isnan(out).any(), p.name
        cb.check_status()


def test_empty_batch_gpu():
    import convolution_backward_b200 as cb
    dy = torch.empty((0, 8, 8, 16), dtype=torch.bfloat16, device="cuda")
    w = torch.randn(3, 3, 16, device="cuda").to(torch.bfloat16)
    out = cb.depthwise(dy, w, H=8, Wd=8, pad_h=1)
    assert out.shape == (0, 8, 8, 16)
    out = cb.pointwise(torch.empty((0, 4, 4, 16), dtype=torch.bfloat16, device="cuda"),
                       torch.randn(16, 8, device="cuda").to(torch.bfloat16))
    assert out.shape == (0, 4, 4, 8)
    out = cb.pointwise_splitk(torch.empty((0, 4, 4, 16), dtype=torch.bfloat16, device="cuda"),
                              torch.randn(16, 8, device="cuda").to(torch.bfloat16))   # automatic split count
    assert out.shape == (0, 4, 4, 8)
    cb.check_status()


def test_timeout_is_reported_not_hung():
    """A bounded wait that runs out is reported by dgrad_check_status, and the context stays usable."""
    import convolution_backward_b200 as cb
    cb.check_status()
    cb.selftest_timeout(20_000_000)
    with pytest.raises(cb.DgradError) as ei:
        cb.check_status()
    assert ei.value.status == 5
    cb.check_status()     # cleared
    h = _h()
    p = SMALL[7]
    inp = synthetic.make_inputs(p)
    dy, w = h.to_dev(inp)
    h.run_gpu(p, dy, w)
    cb.check_status()


def test_streams_are_respected():
    """Work enqueued on a side stream is ordered on that stream."""
    h = _h()
    import convolution_backward_b200 as cb
    p = SMALL[4]
    inp = synthetic.make_inputs(p)
    dy, w = h.to_dev(inp)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        out = cb.pointwise(dy, w)
    s.synchronize()
    ref = h.oracle_full(p, inp.dy, inp.w)
    absref = h.oracle_full(p, np.abs(inp.dy), np.abs(inp.w))
    h.check(p, h.gpu_to_np(out), ref, absref, what="side stream")


# --- every element of the full-size workloads against the oracle ----------------

EVERY = [p for p in synthetic.all_problems() if p.name in ("pw_bf16", "dw3x3_bf16", "dw7x7s2_bf16")]


def _oracle_whole(p, dy, w):
    import oracle
    if p.kind == "pointwise":
        return oracle.pointwise_matmul(dy, w)
    return oracle.depthwise_taps(dy, w, H=p.H, W=p.W, S=p.stride, ph=p.pad_h, pw=p.pad_w)


@pytest.mark.parametrize("p", EVERY, ids=[p.name for p in EVERY])
def test_full_size_every_element(p):
    """The benchmark's pointwise bf16, depthwise 3x3 and 7x7 stride-2 problems at full size, every
    element of dX against the fp64 oracle (whole-array form, pinned to the scatter loop) under the
    normwise bar and the elementwise bound."""
    h = _h()
    import convolution_backward_b200 as cb
    inp = synthetic.make_inputs(p)
    dy, w = h.to_dev(inp)
    out = h.run_gpu(p, dy, w)
    cb.check_status()
    got = h.gpu_to_np(out)
    ref = _oracle_whole(p, inp.dy, inp.w)
    absref = _oracle_whole(p, np.abs(inp.dy), np.abs(inp.w))
    h.check(p, got, ref, absref, what=f"{p.name} every element")


TC_EVERY_CHANNELS = (0, 1, 2, 3, 4, 5, 6, 7, 200, 201, 202, 203, 204, 205, 206, 207, -8, -7, -6, -5, -4, -3, -2, -1)


@pytest.mark.parametrize("entry", ["tc", "auto"])
@pytest.mark.parametrize("p", TC_FULL, ids=[p.name for p in TC_FULL])
def test_full_size_tensor_core_channel_subset(p, entry):
    """The large-filter workloads at full size: every image and every spatial position of 24 channels
    (the first, a middle and the last 8-channel block) against the fp64 oracle, through the planar
    tensor-core entry point and through dgrad_depthwise's automatic choice.  Depthwise channels are
    independent, so a channel subset is an exact sub-problem."""
    h = _h()
    import convolution_backward_b200 as cb
    inp = synthetic.make_inputs(p)
    dy, w = h.to_dev(inp)
    if entry == "tc":
        out = cb.depthwise_tc(dy, w, H=p.H, Wd=p.W, pad_h=p.pad_h, pad_w=p.pad_w)
    else:
        out = cb.depthwise(dy, w, H=p.H, Wd=p.W, pad_h=p.pad_h, pad_w=p.pad_w)
    cb.check_status()
    ch = np.array([c % p.C for c in TC_EVERY_CHANNELS])
    got = out.float()[..., torch.from_numpy(ch).cuda()].cpu().numpy().astype(np.float64)
    sub = p.replace(C=len(ch), K=len(ch))
    dys, ws = inp.dy[..., ch], inp.w[..., ch]
    ref = _oracle_whole(sub, dys, ws)
    absref = _oracle_whole(sub, np.abs(dys), np.abs(ws))
    h.check(sub, got, ref, absref, what=f"{p.name}/{entry} channels {list(ch[:3])}..")


def test_planted_dy_stride_mistake_is_caught():
    """The pages' lesson for the pointwise fast path (a mutated dY pixel stride must fail the numeric
    suite): dgrad_pointwise is handed a dY whose rows really lie K + 8 elements apart while the
    problem says K, as a kernel with a wrong stride would read it.  The parity check must fail."""
    h = _h()
    import ctypes
    import convolution_backward_b200 as cb
    p = P("pw_planted", "pointwise", "bf16", 2, 14, 14, 64, 64, seed=77)
    inp = synthetic.make_inputs(p)
    dy, w = h.to_dev(inp)
    M = p.N * p.H * p.W
    wide = torch.zeros((M, p.K + 8), dtype=dy.dtype, device=dy.device)
    wide[:, :p.K] = dy.reshape(M, p.K)
    out = torch.empty(p.dx_shape, dtype=dy.dtype, device=dy.device)
    prob = cb.Problem(p.N, p.H, p.W, p.C, p.K, 1, 1, 1, 0, 0)
    L = cb.lib()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert L.dgrad_pointwise(ctypes.byref(prob), 1, wide.data_ptr(), w.data_ptr(), out.data_ptr(), stream) == 0
    cb.check_status()
    got = h.gpu_to_np(out)
    ref = h.oracle_full(p, inp.dy, inp.w)
    absref = h.oracle_full(p, np.abs(inp.dy), np.abs(inp.w))
    with pytest.raises(AssertionError):
        h.check(p, got, ref, absref, what="planted dY stride")
    # and the same buffers read with the right layout pass
    h.check(p, h.gpu_to_np(cb.pointwise(dy, w)), ref, absref, what="right dY stride")
