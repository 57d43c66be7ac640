"""The debug build, libdgrad_debug.so: the same kernels compiled with -DDGRAD_DEBUG,
in which every hand-indexed store checks that it stays inside its output buffer
(a failed check skips the store and records DGRAD_ERR_BOUNDS).  It stands in
for a memory checker: each kernel family runs one ragged problem under it and
must give the oracle's result with a clean status word."""
import ctypes
import os

import numpy as np
import pytest

import convolution_backward_b200 as cb
from convolution_backward_b200 import synthetic
from convolution_backward_b200.synthetic import Problem

DEBUG_LIB = os.path.join(os.path.dirname(cb.library_path()), "libdgrad_debug.so")


def P(name, kind, dtype, N, H, W, C, K, KH=1, KW=1, S=1, ph=0, pw=0, seed=11):
    return Problem(name, kind, dtype, N=N, H=H, W=W, C=C, K=K, KH=KH, KW=KW, stride=S, pad_h=ph,
                   pad_w=pw, seed=seed, w_var=1.0 / (KH * KW) if kind == "depthwise" else 1.0 / K)


def test_debug_library_exports_the_same_symbols():
    if not os.path.exists(DEBUG_LIB):
        pytest.skip("libdgrad_debug.so not built")
    rel = ctypes.CDLL(cb.library_path())
    dbg = ctypes.CDLL(DEBUG_LIB)
    for name in ("dgrad_pointwise", "dgrad_depthwise", "dgrad_depthwise_tc", "dgrad_dense", "dgrad_grouped",
                 "dgrad_pointwise_splitk", "dgrad_pointwise_splitk_noalloc", "dgrad_check_status",
                 "dgrad_status_string"):
        assert hasattr(rel, name) and hasattr(dbg, name), name
    dbg.dgrad_status_string.restype = ctypes.c_char_p
    assert b"index check" in dbg.dgrad_status_string(6)


# One ragged problem per kernel family, with the tuning switch that selects it (tests run with
# DGRAD_TUNING=1, set in conftest.py).
CASES = [
    (P("pw_bf16_pair", "pointwise", "bf16", 2, 13, 23, 264, 200, seed=501), {}, "auto"),
    (P("pw_f32", "pointwise", "f32", 2, 7, 9, 44, 20, seed=502), {}, "auto"),
    (P("pw_f16_taps", "pointwise", "f16", 1, 9, 11, 40, 72, seed=503), {}, "auto"),
    (P("dw_tile_3x3", "depthwise", "bf16", 2, 17, 19, 40, 40, 3, 3, 1, 1, 1, seed=504), {}, "rotated"),
    (P("dw_tile_3x3_direct", "depthwise", "bf16", 2, 17, 19, 40, 40, 3, 3, 1, 1, 1, seed=504),
     {"DGRAD_TILE_STORE": "direct"}, "rotated"),
    (P("dw_rot_13x9_f32", "depthwise", "f32", 1, 21, 17, 36, 36, 13, 9, 1, 6, 4, seed=505), {}, "rotated"),
    (P("dw_rs_reg_7x7s2", "depthwise", "bf16", 2, 23, 29, 40, 40, 7, 7, 2, 3, 3, seed=506), {}, "rowstream"),
    (P("dw_rs_reg_7x7s2_direct", "depthwise", "bf16", 2, 23, 29, 40, 40, 7, 7, 2, 3, 3, seed=506),
     {"DGRAD_RS_STORE": "direct"}, "rowstream"),
    (P("dw_rs_smem_5x5s2", "depthwise", "bf16", 1, 19, 21, 24, 24, 5, 5, 2, 2, 2, seed=507),
     {"DGRAD_RS_KERNEL": "smem"}, "rowstream"),
    (P("dw_rs_generic_s3", "depthwise", "f16", 1, 17, 16, 16, 16, 5, 4, 3, 2, 1, seed=508),
     {"DGRAD_RS_GENERIC": "1"}, "rowstream"),
    (P("dw_nhwc_tc_11x9", "depthwise", "bf16", 9, 19, 21, 24, 24, 11, 9, 1, 5, 4, seed=509), {}, "auto"),
]


@pytest.mark.gpu
@pytest.mark.parametrize("case", CASES, ids=[c[0].name for c in CASES])
def test_kernels_under_the_debug_build(case, monkeypatch):
    if not os.path.exists(DEBUG_LIB):
        pytest.skip("libdgrad_debug.so not built")
    import gpu_helpers as h
    p, env, mode = case
    for k, v in env.items():
        monkeypatch.setenv(k, v)
    monkeypatch.setattr(cb, "_LIB_PATH", DEBUG_LIB)
    monkeypatch.setattr(cb, "_lib", None)
    inp = synthetic.make_inputs(p)
    dy, w = h.to_dev(inp)
    out = h.run_gpu(p, dy, w, mode=mode)
    cb.check_status()   # raises DgradError(DGRAD_ERR_BOUNDS) if any store index check failed
    got = h.gpu_to_np(out)
    ref = h.oracle_full(p, inp.dy, inp.w)
    absref = h.oracle_full(p, np.abs(inp.dy), np.abs(inp.w))
    h.check(p, got, ref, absref, what=f"{p.name} (debug build)")


@pytest.mark.gpu
def test_tensor_core_depthwise_planar_under_the_debug_build(monkeypatch):
    """The planar tensor-core path (its transposes on CUDA cores, whose stores are checked)."""
    if not os.path.exists(DEBUG_LIB):
        pytest.skip("libdgrad_debug.so not built")
    import gpu_helpers as h
    monkeypatch.setenv("DGRAD_TC_TRANSPOSE", "cuda")
    monkeypatch.setattr(cb, "_LIB_PATH", DEBUG_LIB)
    monkeypatch.setattr(cb, "_lib", None)
    p = P("dw_tc_planar_13x5", "depthwise", "bf16", 3, 18, 22, 64, 64, 13, 5, 1, 6, 2, seed=510)
    inp = synthetic.make_inputs(p)
    dy, w = h.to_dev(inp)
    out = cb.depthwise_tc(dy, w, H=p.H, Wd=p.W, pad_h=p.pad_h, pad_w=p.pad_w)
    cb.check_status()
    ref = h.oracle_full(p, inp.dy, inp.w)
    absref = h.oracle_full(p, np.abs(inp.dy), np.abs(inp.w))
    h.check(p, h.gpu_to_np(out), ref, absref, what=f"{p.name} (debug build)")
