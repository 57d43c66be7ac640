"""convolution_backward_b200 -- B200 (sm_100a) convolution backward-data (dgrad).

A thin ctypes binding over ``libdgrad.so`` (the C ABI in ``include/dgrad.h``).
This module only marshals arguments: it checks tensor shapes, dtypes and
devices, passes raw device pointers and the current CUDA stream, and raises on
a non-OK status.  Every step of the computation runs in the library's CUDA
kernels; there is no CPU or PyTorch fallback.  If the library is missing the
calls raise ``DgradUnavailable``.

    dX = pointwise(dY, W)                          # dY (N,H,W,K), W (K,C) -> (N,H,W,C)
    dX = depthwise(dY, W, H=H, W=W_, stride=1, pad_h=1, pad_w=1)   # W (KH,KW,C)

Tensors are NHWC and contiguous; float32 or bfloat16 (bf16 in, bf16 out,
fp32 accumulate).
"""
from __future__ import annotations

import ctypes
import os
import threading

__all__ = ["pointwise", "pointwise_splitk", "pointwise_splitk_noalloc", "depthwise_tc", "depthwise_tc_workspace_bytes", "dense", "grouped", "splitk_workspace_bytes", "depthwise", "out_dims", "check_status", "DgradError", "DgradUnavailable",
           "Problem", "lib", "library_path", "selftest_timeout", "fma_probe", "STATUS"]

_PKG = os.path.dirname(os.path.abspath(__file__))
# DGRAD_LIBRARY=debug loads libdgrad_debug.so: the same kernels built with index
# checks on every hand-indexed store (a failed check skips the store and makes
# check_status raise with DGRAD_ERR_BOUNDS).
_LIB_PATH = os.path.join(_PKG, "libdgrad_debug.so" if os.environ.get("DGRAD_LIBRARY") == "debug" else "libdgrad.so")
_lock = threading.Lock()
_lib = None

STATUS = {0: "DGRAD_OK", 1: "DGRAD_ERR_INVALID", 2: "DGRAD_ERR_UNSUPPORTED", 3: "DGRAD_ERR_ALIGNMENT",
          4: "DGRAD_ERR_CUDA", 5: "DGRAD_ERR_TIMEOUT", 6: "DGRAD_ERR_BOUNDS"}
DW_MODES = {"auto": 0, "rotated": 1, "rowstream": 2}
DTYPES = {"f32": 0, "bf16": 1, "f16": 2}
SPLITK_SCRATCH_BYTES = 8 << 20   # DGRAD_SPLITK_SCRATCH_BYTES: the fixed per-device split-K buffer


class DgradUnavailable(RuntimeError):
    """libdgrad.so could not be loaded (not built, or built for another platform)."""


class DgradError(RuntimeError):
    def __init__(self, status: int, what: str, cuda_error: int = 0):
        self.status = status
        self.cuda_error = cuda_error
        msg = f"{what}: {STATUS.get(status, status)}"
        if status == 4:
            msg += f" (cudaError {cuda_error})"
        super().__init__(msg)


class Problem(ctypes.Structure):
    """dgrad_problem_t: N, H, W, C, K (int64), KH, KW, stride, pad_h, pad_w (int32)."""
    _fields_ = [("N", ctypes.c_int64), ("H", ctypes.c_int64), ("W", ctypes.c_int64),
                ("C", ctypes.c_int64), ("K", ctypes.c_int64), ("KH", ctypes.c_int32),
                ("KW", ctypes.c_int32), ("stride", ctypes.c_int32), ("pad_h", ctypes.c_int32),
                ("pad_w", ctypes.c_int32)]


def library_path() -> str:
    return _LIB_PATH


def lib():
    """The loaded libdgrad (ctypes.CDLL) with argument types declared."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(_LIB_PATH):
                raise DgradUnavailable(
                    f"{_LIB_PATH} is missing; build it with `python -m convolution_backward_b200._build` "
                    "(nvcc, sm_100a)")
            try:
                L = ctypes.CDLL(_LIB_PATH)
            except OSError as e:
                raise DgradUnavailable(f"cannot load {_LIB_PATH}: {e}") from e
            P = ctypes.POINTER
            vp = ctypes.c_void_p
            L.dgrad_pointwise.argtypes = [P(Problem), ctypes.c_int, vp, vp, vp, vp]
            L.dgrad_pointwise.restype = ctypes.c_int
            L.dgrad_depthwise.argtypes = [P(Problem), ctypes.c_int, ctypes.c_int, vp, vp, vp, vp]
            L.dgrad_depthwise.restype = ctypes.c_int
            L.dgrad_out_dims.argtypes = [P(Problem), P(ctypes.c_int64), P(ctypes.c_int64)]
            L.dgrad_out_dims.restype = ctypes.c_int
            L.dgrad_check_status.argtypes = [vp]
            L.dgrad_check_status.restype = ctypes.c_int
            L.dgrad_status_string.argtypes = [ctypes.c_int]
            L.dgrad_status_string.restype = ctypes.c_char_p
            L.dgrad_last_cuda_error.argtypes = []
            L.dgrad_last_cuda_error.restype = ctypes.c_int
            L.dgrad_selftest_timeout.argtypes = [ctypes.c_longlong, vp]
            L.dgrad_selftest_timeout.restype = ctypes.c_int
            L.dgrad_fma_probe.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, vp, vp]
            L.dgrad_fma_probe.restype = ctypes.c_int
            L.dgrad_pointwise_splitk.argtypes = [P(Problem), ctypes.c_int, ctypes.c_int, vp, vp, vp, vp,
                                                 ctypes.c_size_t, vp]
            L.dgrad_pointwise_splitk.restype = ctypes.c_int
            L.dgrad_pointwise_splitk_workspace.argtypes = [P(Problem), ctypes.c_int, P(ctypes.c_size_t),
                                                           P(ctypes.c_int)]
            L.dgrad_pointwise_splitk_workspace.restype = ctypes.c_int
            L.dgrad_pointwise_splitk_noalloc.argtypes = [P(Problem), ctypes.c_int, ctypes.c_int, vp, vp, vp, vp]
            L.dgrad_pointwise_splitk_noalloc.restype = ctypes.c_int
            L.dgrad_dense.argtypes = [P(Problem), ctypes.c_int, vp, vp, vp, vp]
            L.dgrad_dense.restype = ctypes.c_int
            L.dgrad_grouped.argtypes = [P(Problem), ctypes.c_int64, ctypes.c_int, vp, vp, vp, vp]
            L.dgrad_grouped.restype = ctypes.c_int
            L.dgrad_depthwise_tc.argtypes = [P(Problem), ctypes.c_int, vp, vp, vp, vp, ctypes.c_size_t, vp]
            L.dgrad_depthwise_tc.restype = ctypes.c_int
            L.dgrad_depthwise_tc_workspace.argtypes = [P(Problem), P(ctypes.c_size_t)]
            L.dgrad_depthwise_tc_workspace.restype = ctypes.c_int
            _lib = L
    return _lib


def _check(status: int, what: str) -> None:
    if status != 0:
        raise DgradError(status, what, lib().dgrad_last_cuda_error())


def _stream_ptr(stream, device=None):
    """The raw cudaStream_t of `stream` (default: the current stream of `device`).
    A given stream must belong to `device`."""
    import torch
    if stream is None:
        stream = torch.cuda.current_stream(device)
    elif device is not None and stream.device != device:
        raise ValueError(f"stream is on {stream.device} but the tensors are on {device}")
    return ctypes.c_void_p(stream.cuda_stream)


def _device_of(*ts):
    """The one CUDA device every tensor in `ts` lives on.  The C ABI works on the
    current device, so the wrappers make this device current around each call;
    tensors on different devices are refused."""
    devs = {(t.device.type, t.device.index) for t in ts}
    if len(devs) != 1:
        raise ValueError("all tensors of one call must be on the same CUDA device, got "
                         + ", ".join(sorted(f"{d[0]}:{d[1]}" for d in devs)))
    return ts[0].device


def _call(dev, what, fn, *args, stream=None):
    """Run C entry point `fn` with `dev` current and its stream appended."""
    import torch
    with torch.cuda.device(dev):
        _check(fn(*args, _stream_ptr(stream, dev)), what)


def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.float32:
        return 0
    if t.dtype == torch.bfloat16:
        return 1
    if t.dtype == torch.float16:
        return 2
    raise TypeError(f"unsupported dtype {t.dtype}; use float32, bfloat16 or float16")


def _need_cuda(*ts):
    for t in ts:
        if not t.is_cuda:
            raise ValueError("tensors must be CUDA tensors (no CPU path)")
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous (NHWC)")


def out_dims(H, W, KH, KW, stride=1, pad_h=0, pad_w=-1):
    """(Ho, Wo) of the forward convolution (host-only C call)."""
    prob = Problem(1, H, W, 1, 1, KH, KW, stride, pad_h, pad_w)
    ho, wo = ctypes.c_int64(), ctypes.c_int64()
    _check(lib().dgrad_out_dims(ctypes.byref(prob), ctypes.byref(ho), ctypes.byref(wo)), "dgrad_out_dims")
    return ho.value, wo.value


def pointwise(dY, W, out=None, stream=None):
    """Pointwise dgrad: dX[n,h,w,:] = dY[n,h,w,:] @ W, dY (N,H,W,K), W (K,C).  Calls dgrad_pointwise."""
    import torch
    _need_cuda(dY, W)
    if dY.dim() != 4 or W.dim() != 2 or W.shape[0] != dY.shape[3]:
        raise ValueError("expected dY (N,H,W,K) and W (K,C)")
    if W.dtype != dY.dtype:
        raise TypeError("dY and W must have the same dtype")
    N, H, Wd, K = dY.shape
    C = W.shape[1]
    if out is None:
        out = torch.empty((N, H, Wd, C), dtype=dY.dtype, device=dY.device)
    else:
        _need_cuda(out)
        if tuple(out.shape) != (N, H, Wd, C) or out.dtype != dY.dtype:
            raise ValueError("out has the wrong shape or dtype")
    prob = Problem(N, H, Wd, C, K, 1, 1, 1, 0, 0)
    _call(_device_of(dY, W, out), "dgrad_pointwise", lib().dgrad_pointwise, ctypes.byref(prob), _dtype_code(dY),
          dY.data_ptr(), W.data_ptr(), out.data_ptr(), stream=stream)
    return out


def splitk_workspace_bytes(N, H, W, K, C, splits=0):
    """(bytes, splits) of workspace pointwise_splitk needs (dgrad_pointwise_splitk_workspace)."""
    prob = Problem(N, H, W, C, K, 1, 1, 1, 0, 0)
    nb, used = ctypes.c_size_t(), ctypes.c_int()
    _check(lib().dgrad_pointwise_splitk_workspace(ctypes.byref(prob), int(splits), ctypes.byref(nb),
                                                  ctypes.byref(used)), "dgrad_pointwise_splitk_workspace")
    return nb.value, used.value


def pointwise_splitk(dY, W, splits=0, workspace=None, out=None, stream=None):
    """Split-K pointwise dgrad for small M (bf16; dgrad_pointwise_splitk).

    workspace: a caller-owned CUDA tensor of at least splitk_workspace_bytes(...)
    bytes; allocated here with torch when None."""
    import torch
    _need_cuda(dY, W)
    if dY.dim() != 4 or W.dim() != 2 or W.shape[0] != dY.shape[3]:
        raise ValueError("expected dY (N,H,W,K) and W (K,C)")
    if W.dtype != dY.dtype:
        raise TypeError("dY and W must have the same dtype")
    N, H, Wd, K = dY.shape
    C = W.shape[1]
    nbytes, used = splitk_workspace_bytes(N, H, Wd, K, C, splits)
    if workspace is None:
        workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=dY.device)
    if out is None:
        out = torch.empty((N, H, Wd, C), dtype=dY.dtype, device=dY.device)
    prob = Problem(N, H, Wd, C, K, 1, 1, 1, 0, 0)
    _call(_device_of(dY, W, out, workspace), "dgrad_pointwise_splitk", lib().dgrad_pointwise_splitk,
          ctypes.byref(prob), _dtype_code(dY), int(used), dY.data_ptr(), W.data_ptr(), out.data_ptr(),
          workspace.data_ptr(), workspace.numel() * workspace.element_size(), stream=stream)
    return out


def pointwise_splitk_noalloc(dY, W, out, splits=0, stream=None):
    """Split-K pointwise dgrad that allocates nothing (dgrad_pointwise_splitk_noalloc).

    For callers that must not allocate device memory at call time: the partial
    tiles go to the library's fixed per-device scratch buffer of
    SPLITK_SCRATCH_BYTES, so ``out`` (N,H,W,C, dY's dtype) is required.  Calls
    that overlap in time on one device share that buffer and race; calls ordered
    on one stream do not.  The first call on a device sets the buffer up: make
    it before any stream capture begins.  A problem whose partial tiles do not
    fit the buffer raises DgradError (status 2, unsupported)."""
    _need_cuda(dY, W, out)
    if dY.dim() != 4 or W.dim() != 2 or W.shape[0] != dY.shape[3]:
        raise ValueError("expected dY (N,H,W,K) and W (K,C)")
    if W.dtype != dY.dtype:
        raise TypeError("dY and W must have the same dtype")
    N, H, Wd, K = dY.shape
    C = W.shape[1]
    if tuple(out.shape) != (N, H, Wd, C) or out.dtype != dY.dtype:
        raise ValueError("out must be (N,H,W,C) with dY's dtype")
    prob = Problem(N, H, Wd, C, K, 1, 1, 1, 0, 0)
    _call(_device_of(dY, W, out), "dgrad_pointwise_splitk_noalloc", lib().dgrad_pointwise_splitk_noalloc,
          ctypes.byref(prob), _dtype_code(dY), int(splits), dY.data_ptr(), W.data_ptr(), out.data_ptr(),
          stream=stream)
    return out


def depthwise(dY, W, *, H, W_out=None, stride=1, pad_h=0, pad_w=-1, mode="auto", out=None,
              stream=None, **kw):
    """Depthwise dgrad (groups = C): dY (N,Ho,Wo,C), W (KH,KW,C) -> dX (N,H,W,C).  Calls dgrad_depthwise.

    H and W_out (alias ``Wd``) are dX's spatial extents; pad_w = -1 means pad_h.
    mode: "auto" (rotated-filter at stride 1, row-streaming otherwise),
    "rotated" or "rowstream".
    """
    import torch
    if W_out is None:
        W_out = kw.pop("Wd")
    if kw:
        raise TypeError(f"unexpected arguments {sorted(kw)}")
    _need_cuda(dY, W)
    if dY.dim() != 4 or W.dim() != 3 or W.shape[2] != dY.shape[3]:
        raise ValueError("expected dY (N,Ho,Wo,C) and W (KH,KW,C)")
    if W.dtype != dY.dtype:
        raise TypeError("dY and W must have the same dtype")
    N, Ho, Wo, C = dY.shape
    KH, KW = W.shape[0], W.shape[1]
    prob = Problem(N, H, W_out, C, C, KH, KW, stride, pad_h, pad_w)
    eho, ewo = out_dims(H, W_out, KH, KW, stride, pad_h, pad_w)
    if (eho, ewo) != (Ho, Wo):
        raise ValueError(f"dY spatial extent {(Ho, Wo)} does not match the geometry ({eho}, {ewo})")
    if out is None:
        out = torch.empty((N, H, W_out, C), dtype=dY.dtype, device=dY.device)
    else:
        _need_cuda(out)
        if tuple(out.shape) != (N, H, W_out, C) or out.dtype != dY.dtype:
            raise ValueError("out has the wrong shape or dtype")
    _call(_device_of(dY, W, out), "dgrad_depthwise", lib().dgrad_depthwise, ctypes.byref(prob), _dtype_code(dY),
          DW_MODES[mode], dY.data_ptr(), W.data_ptr(), out.data_ptr(), stream=stream)
    return out


def dense(dY, W, *, H, W_out=None, stride=1, pad_h=0, pad_w=-1, out=None, stream=None, **kw):
    """Dense (ungrouped) dgrad on the tensor cores (bf16 or f16; dgrad_dense): dY (N,Ho,Wo,K),
    W (KH,KW,K,C) -> dX (N,H,W,C).  H and W_out (alias ``Wd``) are dX's spatial extents."""
    import torch
    if W_out is None:
        W_out = kw.pop("Wd")
    if kw:
        raise TypeError(f"unexpected arguments {sorted(kw)}")
    _need_cuda(dY, W)
    if dY.dim() != 4 or W.dim() != 4 or W.shape[2] != dY.shape[3]:
        raise ValueError("expected dY (N,Ho,Wo,K) and W (KH,KW,K,C)")
    if W.dtype != dY.dtype:
        raise TypeError("dY and W must have the same dtype")
    N, Ho, Wo, K = dY.shape
    KH, KW, _, C = W.shape
    eho, ewo = out_dims(H, W_out, KH, KW, stride, pad_h, pad_w)
    if (eho, ewo) != (Ho, Wo):
        raise ValueError(f"dY spatial extent {(Ho, Wo)} does not match the geometry ({eho}, {ewo})")
    if out is None:
        out = torch.empty((N, H, W_out, C), dtype=dY.dtype, device=dY.device)
    else:
        _need_cuda(out)
        if tuple(out.shape) != (N, H, W_out, C) or out.dtype != dY.dtype:
            raise ValueError("out has the wrong shape or dtype")
    prob = Problem(N, H, W_out, C, K, KH, KW, stride, pad_h, pad_w)
    _call(_device_of(dY, W, out), "dgrad_dense", lib().dgrad_dense, ctypes.byref(prob), _dtype_code(dY),
          dY.data_ptr(), W.data_ptr(), out.data_ptr(), stream=stream)
    return out


def grouped(dY, W, groups, *, H, W_out=None, stride=1, pad_h=0, pad_w=-1, out=None, stream=None, **kw):
    """Grouped dgrad on the tensor cores (bf16 or f16; dgrad_grouped): dY (N,Ho,Wo,K),
    W (KH,KW,K,C/groups) -> dX (N,H,W,C).  A 1x1 filter is grouped pointwise dgrad."""
    import torch
    if W_out is None:
        W_out = kw.pop("Wd")
    if kw:
        raise TypeError(f"unexpected arguments {sorted(kw)}")
    _need_cuda(dY, W)
    if dY.dim() != 4 or W.dim() != 4 or W.shape[2] != dY.shape[3]:
        raise ValueError("expected dY (N,Ho,Wo,K) and W (KH,KW,K,C/groups)")
    if W.dtype != dY.dtype:
        raise TypeError("dY and W must have the same dtype")
    N, Ho, Wo, K = dY.shape
    KH, KW, _, Cg = W.shape
    C = Cg * int(groups)
    eho, ewo = out_dims(H, W_out, KH, KW, stride, pad_h, pad_w)
    if (eho, ewo) != (Ho, Wo):
        raise ValueError(f"dY spatial extent {(Ho, Wo)} does not match the geometry ({eho}, {ewo})")
    if out is None:
        out = torch.empty((N, H, W_out, C), dtype=dY.dtype, device=dY.device)
    else:
        _need_cuda(out)
        if tuple(out.shape) != (N, H, W_out, C) or out.dtype != dY.dtype:
            raise ValueError("out has the wrong shape or dtype")
    prob = Problem(N, H, W_out, C, K, KH, KW, stride, pad_h, pad_w)
    _call(_device_of(dY, W, out), "dgrad_grouped", lib().dgrad_grouped, ctypes.byref(prob), int(groups),
          _dtype_code(dY), dY.data_ptr(), W.data_ptr(), out.data_ptr(), stream=stream)
    return out


def depthwise_tc_workspace_bytes(N, H, W, C, KH, KW, pad_h=0, pad_w=-1) -> int:
    """Workspace bytes dgrad_depthwise_tc needs (host only); raises DgradError when unsupported."""
    prob = Problem(N, H, W, C, C, KH, KW, 1, pad_h, pad_w)
    nb = ctypes.c_size_t()
    _check(lib().dgrad_depthwise_tc_workspace(ctypes.byref(prob), ctypes.byref(nb)), "dgrad_depthwise_tc_workspace")
    return nb.value


def depthwise_tc(dY, W, *, H, W_out=None, pad_h=0, pad_w=-1, workspace=None, out=None, stream=None, **kw):
    """Stride-1 depthwise dgrad on the tensor cores (bf16; dgrad_depthwise_tc).

    Same arguments and result as depthwise() at stride 1.  workspace: a CUDA
    tensor of at least depthwise_tc_workspace_bytes(...) bytes, allocated here
    with torch when None."""
    import torch
    if W_out is None:
        W_out = kw.pop("Wd")
    if kw:
        raise TypeError(f"unexpected arguments {sorted(kw)}")
    _need_cuda(dY, W)
    if dY.dim() != 4 or W.dim() != 3 or W.shape[2] != dY.shape[3]:
        raise ValueError("expected dY (N,Ho,Wo,C) and W (KH,KW,C)")
    if W.dtype != dY.dtype:
        raise TypeError("dY and W must have the same dtype")
    N, Ho, Wo, C = dY.shape
    KH, KW = W.shape[0], W.shape[1]
    eho, ewo = out_dims(H, W_out, KH, KW, 1, pad_h, pad_w)
    if (eho, ewo) != (Ho, Wo):
        raise ValueError(f"dY spatial extent {(Ho, Wo)} does not match the geometry ({eho}, {ewo})")
    prob = Problem(N, H, W_out, C, C, KH, KW, 1, pad_h, pad_w)
    nbytes = depthwise_tc_workspace_bytes(N, H, W_out, C, KH, KW, pad_h, pad_w)
    if workspace is None:
        workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=dY.device)
    if out is None:
        out = torch.empty((N, H, W_out, C), dtype=dY.dtype, device=dY.device)
    else:
        _need_cuda(out)
        if tuple(out.shape) != (N, H, W_out, C) or out.dtype != dY.dtype:
            raise ValueError("out has the wrong shape or dtype")
    _call(_device_of(dY, W, out, workspace), "dgrad_depthwise_tc", lib().dgrad_depthwise_tc, ctypes.byref(prob),
          _dtype_code(dY), dY.data_ptr(), W.data_ptr(), out.data_ptr(), workspace.data_ptr(),
          workspace.numel() * workspace.element_size(), stream=stream)
    return out


def check_status(stream=None) -> None:
    """Synchronise the stream and raise if a kernel reported a timeout (dgrad_check_status)."""
    import torch
    dev = stream.device if stream is not None else torch.device("cuda", torch.cuda.current_device())
    with torch.cuda.device(dev):
        _check(lib().dgrad_check_status(_stream_ptr(stream, dev)), "dgrad_check_status")


def selftest_timeout(limit_cycles: int = 20_000_000, stream=None) -> None:
    """Launch the diagnostic kernel whose bounded wait runs out (dgrad_selftest_timeout)."""
    import torch
    dev = stream.device if stream is not None else torch.device("cuda", torch.cuda.current_device())
    with torch.cuda.device(dev):
        _check(lib().dgrad_selftest_timeout(int(limit_cycles), _stream_ptr(stream, dev)), "dgrad_selftest_timeout")


def fma_probe(blocks: int, iters: int, packed: bool, sink, stream=None) -> int:
    """Launch the fp32 FMA-rate probe; returns the FLOP count it performs."""
    _call(_device_of(sink), "dgrad_fma_probe", lib().dgrad_fma_probe, int(blocks), int(iters), 1 if packed else 0,
          sink.data_ptr(), stream=stream)
    return int(blocks) * 256 * int(iters) * 16 * 2
