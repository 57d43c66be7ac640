"""dgrad_pointwise_splitk_noalloc: split-K pointwise dgrad that allocates nothing.

The entry point has no counterpart on the pages; it runs the split-K kernels of
dgrad_pointwise_splitk with the library's fixed per-device scratch buffer as
their workspace.  The GPU test calls both entry points through the C ABI, the
no-allocation one twice in a row on one stream (two different problems, so the
second call reuses the buffer the first one filled), and compares each result
with dgrad_pointwise_splitk at the same split count, within the bf16 acceptance
bar of the parity tests: max|new - ref| / (max|ref| + 1e-6) <= 1e-2.  The same
kernels with the same split count sum in the same order, so the results are
also expected to be bit-identical.

This file is collected last, so that it runs both after the rest of the suite
and on its own.
"""
import ctypes

import numpy as np
import pytest

import convolution_backward_b200 as cb
from convolution_backward_b200 import synthetic

OK, UNSUPPORTED = 0, 2
BF16 = 1
SCRATCH = cb.SPLITK_SCRATCH_BYTES
FAKE = 0x10000   # 16-byte aligned, never dereferenced (the calls below launch nothing)

P = synthetic.Problem
PROBLEMS = [
    P("na_small_m", "pointwise", "bf16", 2, 14, 14, 512, 2048, seed=121, w_var=1.0 / 2048),
    P("na_ragged", "pointwise", "bf16", 1, 7, 9, 136, 1000, seed=122, w_var=1.0 / 1000),
]
# Automatic split count (3 here) would need 3 * 392 * 2048 * 4 bytes, more than
# the buffer: the call lowers it to 2.
P_LOWERED = P("na_lowered", "pointwise", "bf16", 2, 14, 14, 2048, 2048, seed=123, w_var=1.0 / 2048)


def _prob(p):
    return cb.Problem(p.N, p.H, p.W, p.C, p.K, 1, 1, 1, 0, 0)


def _splits_used(p, splits):
    """The split count the no-allocation call runs with: the requested one, or
    the automatic one lowered until the partial tiles fit the buffer."""
    nbytes, used = cb.splitk_workspace_bytes(p.N, p.H, p.W, p.K, p.C, splits)
    per_split = nbytes // used
    if splits == 0 and nbytes > SCRATCH:
        used = SCRATCH // per_split
    assert 1 <= used and used * per_split <= SCRATCH
    return used


def _device_inputs(p):
    import torch
    inp = synthetic.make_inputs(p)
    dy = torch.from_numpy(inp.dy_bits.view(np.int16)).view(torch.bfloat16).cuda().contiguous()
    w = torch.from_numpy(inp.w_bits.view(np.int16)).view(torch.bfloat16).cuda().contiguous()
    return dy, w


def _normwise(got, ref):
    g = got.float()
    r = ref.float()
    return float((g - r).abs().max()) / (float(r.abs().max()) + 1e-6)


def test_rejects_problems_too_large_for_the_buffer():
    """Host-side refusals: nothing is launched and no device is needed."""
    L = cb.lib()
    # one split of M * C * 4 = 6272 * 512 * 4 bytes (12.8 MB) is over the 8 MiB buffer
    big = cb.Problem(8, 28, 28, 512, 512, 1, 1, 1, 0, 0)
    assert L.dgrad_pointwise_splitk_noalloc(ctypes.byref(big), BF16, 1, FAKE, FAKE, FAKE, None) == UNSUPPORTED
    lowered = _prob(P_LOWERED)
    assert L.dgrad_pointwise_splitk_noalloc(ctypes.byref(lowered), BF16, 3, FAKE, FAKE, FAKE, None) == UNSUPPORTED
    assert L.dgrad_pointwise_splitk_noalloc(ctypes.byref(lowered), BF16, 65, FAKE, FAKE, FAKE, None) == 1
    assert L.dgrad_pointwise_splitk_noalloc(None, BF16, 1, FAKE, FAKE, FAKE, None) == 1
    empty = cb.Problem(0, 14, 14, 64, 256, 1, 1, 1, 0, 0)
    assert L.dgrad_pointwise_splitk_noalloc(ctypes.byref(empty), BF16, 0, 0, 0, 0, None) == OK


@pytest.mark.gpu
@pytest.mark.parametrize("splits", [0, 3])
def test_noalloc_matches_splitk_two_calls_in_a_row(splits):
    import torch
    L = cb.lib()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    cases = []
    for p in PROBLEMS:
        dy, w = _device_inputs(p)
        out = torch.full((p.N, p.H, p.W, p.C), float("nan"), dtype=torch.bfloat16, device="cuda")
        cases.append((p, dy, w, out))
    # the two calls in a row, on one stream
    for p, dy, w, out in cases:
        st = L.dgrad_pointwise_splitk_noalloc(ctypes.byref(_prob(p)), BF16, splits, dy.data_ptr(), w.data_ptr(),
                                              out.data_ptr(), stream)
        assert st == OK, cb.STATUS.get(st, st)
    assert L.dgrad_check_status(stream) == OK
    # the existing entry point with a caller workspace, same split count
    for p, dy, w, out in cases:
        used = _splits_used(p, splits)
        nbytes, _ = cb.splitk_workspace_bytes(p.N, p.H, p.W, p.K, p.C, used)
        ws = torch.empty(nbytes // 4 + 4, dtype=torch.float32, device="cuda")
        ref = torch.empty_like(out)
        st = L.dgrad_pointwise_splitk(ctypes.byref(_prob(p)), BF16, used, dy.data_ptr(), w.data_ptr(),
                                      ref.data_ptr(), ws.data_ptr(), ws.numel() * 4, stream)
        assert st == OK, cb.STATUS.get(st, st)
        assert L.dgrad_check_status(stream) == OK
        assert not torch.isnan(out.float()).any(), p.name
        err = _normwise(out, ref)
        assert err <= 1e-2, f"{p.name} splits={splits}({used}): normwise {err:.3e}"
        assert torch.equal(out, ref), f"{p.name}: same kernels and split count should give identical bits"


@pytest.mark.gpu
def test_noalloc_lowers_automatic_splits_to_fit():
    import torch
    L = cb.lib()
    p = P_LOWERED
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    dy, w = _device_inputs(p)
    used = _splits_used(p, 0)
    _, auto = cb.splitk_workspace_bytes(p.N, p.H, p.W, p.K, p.C, 0)
    assert used < auto
    outs = []
    for _ in range(2):
        out = torch.full((p.N, p.H, p.W, p.C), float("nan"), dtype=torch.bfloat16, device="cuda")
        assert L.dgrad_pointwise_splitk_noalloc(ctypes.byref(_prob(p)), BF16, 0, dy.data_ptr(), w.data_ptr(),
                                                out.data_ptr(), stream) == OK
        outs.append(out)
    ref = cb.pointwise_splitk(dy, w, splits=used)
    assert L.dgrad_check_status(stream) == OK
    for out in outs:
        assert _normwise(out, ref) <= 1e-2
        assert torch.equal(out, ref)


@pytest.mark.gpu
def test_noalloc_automatic_count_refuses_when_one_split_does_not_fit():
    """With splits = 0 the count is lowered until the partial tiles fit; when
    even one split (M * C * 4 bytes) is over the buffer the call is refused and
    nothing is launched, so dX keeps its contents."""
    import torch
    L = cb.lib()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    big = cb.Problem(8, 28, 28, 512, 512, 1, 1, 1, 0, 0)
    dy = torch.zeros((8, 28, 28, 512), dtype=torch.bfloat16, device="cuda")
    w = torch.zeros((512, 512), dtype=torch.bfloat16, device="cuda")
    out = torch.full((8, 28, 28, 512), float("nan"), dtype=torch.bfloat16, device="cuda")
    st = L.dgrad_pointwise_splitk_noalloc(ctypes.byref(big), BF16, 0, dy.data_ptr(), w.data_ptr(), out.data_ptr(),
                                          stream)
    assert st == UNSUPPORTED, cb.STATUS.get(st, st)
    assert L.dgrad_check_status(stream) == OK
    assert torch.isnan(out.float()).all()
