"""Host-side checks of the C ABI that need no GPU.

- libdgrad.so loads and exports every function include/dgrad.h declares;
- dgrad_out_dims computes the forward extents (per-axis padding, pad_w = -1);
- every validation rule rejects before anything touches the GPU (the pointers
  passed here are never dereferenced: a rejected call launches nothing);
- an empty batch is a no-op.
"""
import ctypes
import os
import re

import pytest

import convolution_backward_b200 as cb

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", f) for f in os.listdir(os.path.join(ROOT, "include"))
           if f.endswith(".h")]

OK, INVALID, UNSUPPORTED, ALIGNMENT = 0, 1, 2, 3
FAKE = 0x10000   # 16-byte aligned, never dereferenced
BF16, F32 = 1, 0


def declared_functions():
    names = set()
    for h in HEADERS:
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"^\s*[A-Za-z_][\w\s\*]*?\b(dgrad_\w+)\s*\(", text, flags=re.M):
            names.add(m.group(1))
    return sorted(names)


def test_library_exports_every_declared_symbol():
    L = cb.lib()
    names = declared_functions()
    assert "dgrad_pointwise" in names and "dgrad_depthwise" in names
    for n in names:
        assert hasattr(L, n), f"libdgrad.so does not export {n}"


def test_status_strings():
    L = cb.lib()
    for code in range(6):
        s = L.dgrad_status_string(code)
        assert s and isinstance(s, bytes)
    assert L.dgrad_status_string(0) == b"ok"


@pytest.mark.parametrize("geom,expect", [
    ((56, 56, 3, 3, 1, 1, 1), (56, 56)),
    ((112, 112, 7, 7, 2, 3, 3), (56, 56)),
    ((64, 64, 51, 5, 1, 25, 2), (64, 64)),
    ((64, 64, 5, 51, 1, 2, 25), (64, 64)),
    ((10, 9, 3, 3, 1, 1, -1), (10, 9)),        # pad_w = -1 means pad_h
    ((10, 9, 3, 3, 1, 1, 0), (10, 7)),
    ((28, 28, 1, 1, 1, 0, 0), (28, 28)),
])
def test_out_dims(geom, expect):
    assert cb.out_dims(*geom) == expect


def _prob(N=1, H=8, W=8, C=16, K=16, KH=3, KW=3, S=1, ph=1, pw=1):
    return cb.Problem(N, H, W, C, K, KH, KW, S, ph, pw)


def _dw(prob, dtype=BF16, mode=0, ptrs=(FAKE, FAKE, FAKE)):
    return cb.lib().dgrad_depthwise(ctypes.byref(prob), dtype, mode, *ptrs, None)


def _pw(prob, dtype=BF16, ptrs=(FAKE, FAKE, FAKE)):
    return cb.lib().dgrad_pointwise(ctypes.byref(prob), dtype, *ptrs, None)


def test_null_problem_is_invalid():
    L = cb.lib()
    assert L.dgrad_pointwise(None, BF16, FAKE, FAKE, FAKE, None) == INVALID
    assert L.dgrad_depthwise(None, BF16, 0, FAKE, FAKE, FAKE, None) == INVALID
    ho = ctypes.c_int64()
    assert L.dgrad_out_dims(None, ctypes.byref(ho), ctypes.byref(ho)) == INVALID


@pytest.mark.parametrize("kw", [
    dict(H=0), dict(W=-1), dict(C=0), dict(K=0), dict(N=-1), dict(KH=0), dict(S=0),
    dict(ph=-1), dict(pw=-2), dict(pw=-7), dict(H=2, KH=7, ph=1),   # Ho < 1
])
def test_invalid_geometry(kw):
    assert _dw(_prob(**kw)) == INVALID


def test_bad_dtype_and_mode():
    assert _dw(_prob(), dtype=7) == INVALID
    assert _dw(_prob(), mode=9) == INVALID


def test_null_pointers_invalid():
    assert _dw(_prob(), ptrs=(0, FAKE, FAKE)) == INVALID
    assert _pw(_prob(KH=1, KW=1, ph=0, pw=0), ptrs=(FAKE, 0, FAKE)) == INVALID


@pytest.mark.parametrize("kw", [dict(KH=3, KW=3, ph=1, pw=1), dict(KH=1, KW=1, S=2, ph=0, pw=0),
                                dict(KH=1, KW=1, ph=1, pw=1), dict(KH=1, KW=1, ph=0, pw=1)])
def test_pointwise_refuses_other_shapes(kw):
    assert _pw(_prob(**kw)) == UNSUPPORTED


@pytest.mark.parametrize("kw,mode", [
    (dict(K=32, C=16), 0),                           # depth multiplier 2
    (dict(KH=65, ph=1, H=70), 0),                    # filter over 64 rows
    (dict(KW=65, pw=1, W=70), 0),
    (dict(S=2), 1),                                  # rotated mode at stride 2
    (dict(KH=3, ph=3, H=8), 0),                      # pad beyond KH-1
    (dict(KW=3, pw=3), 0),
    (dict(S=9, H=40, W=40), 2),                      # stride over 8
])
def test_depthwise_refusals(kw, mode):
    assert _dw(_prob(**kw), mode=mode) == UNSUPPORTED


def test_alignment():
    assert _dw(_prob(), ptrs=(FAKE + 2, FAKE, FAKE)) == ALIGNMENT
    assert _dw(_prob(), ptrs=(FAKE, FAKE, FAKE + 8)) == ALIGNMENT
    assert _dw(_prob(C=12, K=12)) == ALIGNMENT                  # 24-byte bf16 rows
    assert _dw(_prob(C=12, K=12), dtype=F32) != ALIGNMENT       # 48-byte f32 rows are fine
    p = _prob(KH=1, KW=1, ph=0, pw=0, K=20, C=16)
    assert _pw(p) == ALIGNMENT                                  # K*2 = 40 bytes
    assert _pw(_prob(KH=1, KW=1, ph=0, pw=0), ptrs=(FAKE, FAKE + 4, FAKE)) == ALIGNMENT


def test_empty_batch_is_noop():
    assert _dw(_prob(N=0), ptrs=(0, 0, 0)) == OK
    assert _pw(_prob(N=0, KH=1, KW=1, ph=0, pw=0), ptrs=(0, 0, 0)) == OK


def test_binding_refuses_cpu_tensors():
    torch = pytest.importorskip("torch")
    x = torch.zeros(1, 4, 4, 8, dtype=torch.bfloat16)
    w = torch.zeros(8, 8, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        cb.pointwise(x, w)
    with pytest.raises(ValueError):
        cb.depthwise(x, torch.zeros(3, 3, 8, dtype=torch.bfloat16), H=4, Wd=4, pad_h=1)


class _FakeCuda:
    """Stands in for a CUDA tensor on a machine without a GPU: the binding's
    argument checks only read these attributes before any library call."""

    def __init__(self, shape, dtype, index=0):
        import torch
        self.shape = tuple(shape)
        self.dtype = dtype
        self.device = torch.device("cuda", index)
        self.is_cuda = True

    def dim(self):
        return len(self.shape)

    def is_contiguous(self):
        return True


def test_binding_refuses_tensors_on_two_devices():
    torch = pytest.importorskip("torch")
    a = _FakeCuda((1, 4, 4, 8), torch.bfloat16, 0)
    b = _FakeCuda((8, 8), torch.bfloat16, 1)
    with pytest.raises(ValueError, match="same CUDA device"):
        cb._device_of(a, b)
    assert cb._device_of(a, _FakeCuda((8, 8), torch.bfloat16, 0)) == torch.device("cuda", 0)


def test_splitk_wrappers_refuse_mixed_dtypes():
    torch = pytest.importorskip("torch")
    dy = _FakeCuda((1, 4, 4, 64), torch.bfloat16)
    w = _FakeCuda((64, 64), torch.float32)
    out = _FakeCuda((1, 4, 4, 64), torch.bfloat16)
    with pytest.raises(TypeError):
        cb.pointwise_splitk(dy, w, splits=2)
    with pytest.raises(TypeError):
        cb.pointwise_splitk_noalloc(dy, w, out, splits=2)


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(cb, "_LIB_PATH", str(tmp_path / "absent.so"))
    monkeypatch.setattr(cb, "_lib", None)
    with pytest.raises(cb.DgradUnavailable):
        cb.lib()


def test_splitk_validation_and_workspace_size():
    L = cb.lib()
    p = _prob(N=2, H=14, W=14, C=64, K=256, KH=1, KW=1, ph=0, pw=0)
    nb = ctypes.c_size_t()
    used = ctypes.c_int()
    assert L.dgrad_pointwise_splitk_workspace(ctypes.byref(p), 4, ctypes.byref(nb), ctypes.byref(used)) == OK
    assert nb.value == 4 * 2 * 14 * 14 * 64 * 4 and used.value == 4
    assert L.dgrad_pointwise_splitk_workspace(ctypes.byref(p), 65, ctypes.byref(nb), None) == INVALID
    call = lambda prob, dtype=BF16, splits=4, ws_bytes=1 << 30: L.dgrad_pointwise_splitk(
        ctypes.byref(prob), dtype, splits, FAKE, FAKE, FAKE, FAKE, ws_bytes, None)
    assert call(p, dtype=F32) == UNSUPPORTED
    assert call(_prob()) == UNSUPPORTED                     # 3x3 is not pointwise
    assert call(p, splits=-1) == INVALID
    assert call(p, ws_bytes=nb.value - 16) == INVALID        # workspace too small
    assert L.dgrad_pointwise_splitk(ctypes.byref(p), BF16, 4, FAKE, FAKE, FAKE, 0, 1 << 30, None) == INVALID
    assert L.dgrad_pointwise_splitk(ctypes.byref(p), BF16, 4, FAKE, FAKE, FAKE, FAKE + 4, 1 << 30, None) == ALIGNMENT


def test_splitk_workspace_empty_batch():
    L = cb.lib()
    nb = ctypes.c_size_t(99)
    p = _prob(N=0, H=14, W=14, C=64, K=256, KH=1, KW=1, ph=0, pw=0)
    assert L.dgrad_pointwise_splitk_workspace(ctypes.byref(p), 3, ctypes.byref(nb), None) == OK
    assert nb.value == 0


def test_depthwise_tc_validation_and_workspace_size():
    L = cb.lib()
    nb = ctypes.c_size_t()
    p31 = cb.Problem(16, 64, 64, 384, 384, 31, 31, 1, 15, 15)
    assert L.dgrad_depthwise_tc_workspace(ctypes.byref(p31), ctypes.byref(nb)) == OK
    # planar dY + planar dX + packed filter lines (31 lines per channel of (Ks + 80) / 2 words,
    # Ks <= 144 the tile's MMA depth) + the split partials (one fp32 128 x 256 tile and one flag
    # per CTA, at most 148)
    planar = 2 * 384 * 64 * 16 * 64 * 2
    assert planar < nb.value <= planar + 384 * 31 * 112 * 4 + 148 * (128 * 256 * 4 + 4) + 512
    p51 = cb.Problem(8, 64, 64, 768, 768, 51, 5, 1, 25, 2)
    assert L.dgrad_depthwise_tc_workspace(ctypes.byref(p51), ctypes.byref(nb)) == OK
    assert L.dgrad_depthwise_tc_workspace(ctypes.byref(p51), None) == INVALID
    empty = cb.Problem(0, 64, 64, 384, 384, 31, 31, 1, 15, 15)
    assert L.dgrad_depthwise_tc_workspace(ctypes.byref(empty), ctypes.byref(nb)) == OK and nb.value == 0
    assert L.dgrad_depthwise_tc_workspace(ctypes.byref(cb.Problem(1, 64, 64, 32, 32, 64, 64, 1, 32, 32)),
                                          ctypes.byref(nb)) == OK
    # 64x64 at pad 6 on 64x64 planes: the input rows are 13 columns wide, so K is clipped to 16
    assert L.dgrad_depthwise_tc_workspace(ctypes.byref(cb.Problem(1, 64, 64, 32, 32, 64, 64, 1, 6, 6)),
                                          ctypes.byref(nb)) == OK
    refused = [cb.Problem(1, 128, 128, 32, 32, 64, 64, 1, 6, 6),   # 64x64 at pad 6, 128 wide: K = 144, no tile fits
               cb.Problem(1, 64, 64, 32, 32, 7, 7, 2, 3, 3),       # stride 2
               cb.Problem(1, 64, 64, 32, 64, 7, 7, 1, 3, 3),       # depth multiplier 2
               cb.Problem(1, 64, 64, 32, 32, 7, 7, 1, 7, 3)]       # pad beyond KH-1
    for q in refused:
        assert L.dgrad_depthwise_tc_workspace(ctypes.byref(q), ctypes.byref(nb)) == UNSUPPORTED
    call = lambda prob, dtype=BF16, ws=FAKE, ws_bytes=1 << 40: L.dgrad_depthwise_tc(
        ctypes.byref(prob), dtype, FAKE, FAKE, FAKE, ws, ws_bytes, None)
    assert call(p31, dtype=F32) == UNSUPPORTED
    assert call(p31, ws=0) == INVALID
    assert call(p31, ws=FAKE + 8) == ALIGNMENT
    assert L.dgrad_depthwise_tc_workspace(ctypes.byref(p31), ctypes.byref(nb)) == OK
    assert call(p31, ws_bytes=nb.value - 256) == INVALID
    assert L.dgrad_depthwise_tc(ctypes.byref(empty), BF16, 0, 0, 0, 0, 0, None) == OK


def test_dense_validation():
    L = cb.lib()
    p = cb.Problem(1, 8, 8, 16, 16, 3, 3, 1, 1, 1)
    call = lambda prob, dtype=BF16, ptrs=(FAKE, FAKE, FAKE): L.dgrad_dense(ctypes.byref(prob), dtype, *ptrs, None)
    assert call(p, dtype=F32) == UNSUPPORTED
    assert call(p, dtype=7) == INVALID
    assert call(cb.Problem(1, 8, 8, 16, 20, 3, 3, 1, 1, 1)) == ALIGNMENT      # K*2 = 40 bytes
    assert call(p, ptrs=(FAKE, FAKE + 4, FAKE)) == ALIGNMENT
    assert call(p, ptrs=(0, FAKE, FAKE)) == INVALID
    assert call(cb.Problem(1, 80, 80, 16, 16, 65, 3, 1, 1, 1)) == UNSUPPORTED   # filter over 64
    assert call(cb.Problem(0, 8, 8, 16, 16, 3, 3, 1, 1, 1), ptrs=(0, 0, 0)) == OK


def test_grouped_validation():
    L = cb.lib()
    call = lambda prob, groups, dtype=BF16, ptrs=(FAKE, FAKE, FAKE): L.dgrad_grouped(
        ctypes.byref(prob), groups, dtype, *ptrs, None)
    p = cb.Problem(1, 8, 8, 64, 128, 1, 1, 1, 0, 0)
    assert call(p, 3) == INVALID            # 3 divides neither K nor C
    assert call(p, 0) == INVALID
    assert call(p, 4, dtype=F32) == UNSUPPORTED
    assert call(p, 16) == ALIGNMENT         # C/groups = 4 channels: 8-byte rows
    assert call(cb.Problem(0, 8, 8, 64, 128, 3, 3, 1, 1, 1), 4, ptrs=(0, 0, 0)) == OK
    F16 = 2
    # f16 depthwise: validated like bf16 (16-bit rows), refused before any launch
    dw = cb.Problem(1, 8, 8, 12, 12, 3, 3, 1, 1, 1)
    assert L.dgrad_depthwise(ctypes.byref(dw), F16, 0, FAKE, FAKE, FAKE, None) == ALIGNMENT   # 24-byte rows
    dw = cb.Problem(1, 8, 8, 16, 16, 3, 3, 1, 1, 1)
    assert L.dgrad_depthwise(ctypes.byref(dw), F16, 0, FAKE, 0, FAKE, None) == INVALID
    assert L.dgrad_depthwise(ctypes.byref(dw), F16, 0, FAKE + 8, FAKE, FAKE, None) == ALIGNMENT
    dw0 = cb.Problem(0, 8, 8, 16, 16, 7, 7, 2, 3, 3)
    assert L.dgrad_depthwise(ctypes.byref(dw0), F16, 0, 0, 0, 0, None) == OK
    # split-K takes bf16 and f16, not f32; f16 is validated like bf16
    pw = cb.Problem(1, 8, 8, 16, 16, 1, 1, 1, 0, 0)
    assert L.dgrad_pointwise_splitk(ctypes.byref(pw), F32, 0, FAKE, FAKE, FAKE, FAKE, 1 << 30, None) == UNSUPPORTED
    assert L.dgrad_pointwise_splitk(ctypes.byref(pw), F16, 0, FAKE, FAKE, FAKE, 0, 1 << 30, None) == INVALID
    assert L.dgrad_pointwise_splitk(ctypes.byref(pw), F16, 0, FAKE + 8, FAKE, FAKE, FAKE, 1 << 30, None) == ALIGNMENT
    pw0 = cb.Problem(0, 8, 8, 16, 16, 1, 1, 1, 0, 0)
    assert L.dgrad_pointwise_splitk(ctypes.byref(pw0), F16, 0, 0, 0, 0, 0, 0, None) == OK
