"""fp64 CPU oracle for convolution backward-data (dgrad).

TEST INFRASTRUCTURE ONLY.  Only the test suite, ``__graft_entry__.smoke()`` and
the benchmark's CPU-baseline / reference leg may import this package.  The CUDA
product path never imports it, and it imports nothing from the product package
(``convolution_backward_b200``); the two share only the seeded input generator,
which holds none of the method's arithmetic.

The arithmetic lives in ``dgrad_oracle.c`` (plain fp64 loops, OpenMP over the
batch).  This module builds it with gcc, loads it with ctypes and marshals numpy
arrays.  Each wrapper names the C routine it calls; the C file cites the
passages each routine follows.  Two whole-array fp64 forms written with numpy
(``pointwise_matmul``, ``depthwise_taps``) serve comparisons of every element of
full-size problems; both are pinned to the C scatter loop.

Layouts (NHWC, channels innermost):
  dY  (N, Ho, Wo, K)           dX (N, H, W, C)
  pointwise W  (K, C)          depthwise W (KH, KW, C)   (groups = C = K)
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dgrad_oracle.c")
_LIB = os.path.join(_HERE, "liboracle_dgrad.so")
_lock = threading.Lock()
_lib = None


class OracleGeom(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int64) for n in
                ("N", "H", "W", "C", "K", "KH", "KW", "S", "ph", "pw", "groups")]


def build(force: bool = False) -> str:
    """Compile dgrad_oracle.c into liboracle_dgrad.so (gcc -O2 -fopenmp)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c99", "-Wall",
               "-o", tmp, _SRC]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            P = ctypes.POINTER
            g = P(OracleGeom)
            d = P(ctypes.c_double)
            i64 = P(ctypes.c_int64)
            lib.oracle_out_dims.argtypes = [g, i64, i64]
            lib.oracle_dgrad.argtypes = [g, d, i64, d, i64, d]
            lib.oracle_dgrad_points.argtypes = [g, d, i64, d, i64, i64, ctypes.c_int64, d]
            lib.oracle_conv_fwd.argtypes = [g, d, d, i64, d]
            lib.oracle_dw_rotated.argtypes = [g, d, d, d]
            lib.oracle_dw_rowstream.argtypes = [g, d, d, d]
            lib.oracle_set_threads.argtypes = [ctypes.c_int]
            lib.oracle_get_threads.restype = ctypes.c_int
            _lib = lib
    return _lib


def set_threads(n: int) -> None:
    """Number of OpenMP threads the oracle uses (0 = OpenMP default)."""
    _load().oracle_set_threads(int(n))


def get_threads() -> int:
    return int(_load().oracle_get_threads())


def _geom(N, H, W, C, K, KH, KW, S, ph, pw, groups) -> OracleGeom:
    return OracleGeom(N, H, W, C, K, KH, KW, S, ph, pw, groups)


def _dptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _i64(vals):
    arr = (ctypes.c_int64 * len(vals))(*[int(v) for v in vals])
    return arr


def out_dims(H, W, KH, KW, S, ph, pw):
    """(Ho, Wo) of the forward convolution, via the C routine oracle_out_dims."""
    g = _geom(1, H, W, 1, 1, KH, KW, S, ph, pw, 1)
    ho, wo = ctypes.c_int64(), ctypes.c_int64()
    if _load().oracle_out_dims(ctypes.byref(g), ctypes.byref(ho), ctypes.byref(wo)):
        raise ValueError("invalid geometry")
    return ho.value, wo.value


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _w_strides(kind: str, KH, KW, C, K, groups):
    """Strides (k, r, s, cg) of Wt(k, r, s, cg) for the filter layouts."""
    if kind == "pointwise":          # W[K][C], 1x1, ungrouped
        return (C, 0, 0, 1)
    if kind == "depthwise":          # W[KH][KW][C], Wt(c, r, s, 0) = W[r][s][c]
        return (1, KW * C, C, 0)
    if kind == "grouped":            # Wt dense [K][KH][KW][C/groups]
        Cg = C // groups
        return (KH * KW * Cg, KW * Cg, Cg, 1)
    raise ValueError(kind)


def dgrad(dy, w, *, kind: str, H: int, W: int, KH: int = 1, KW: int = 1, S: int = 1,
          ph: int = 0, pw: int = 0, groups: int | None = None, C: int | None = None,
          dy_strides=None, dy_shape=None, w_strides=None) -> np.ndarray:
    """dX = dgrad(dY, W) in fp64 by the scatter loop (C: oracle_dgrad).

    kind: "pointwise" (W (K, C)), "depthwise" (W (KH, KW, C)) or "grouped"
    (W (K, KH, KW, C/groups)).  dy_strides / dy_shape read dY as a flat buffer
    with the given element strides (n, ho, wo, k) and logical shape; they exist
    for the planted-mistake tests, as does w_strides (the filter's element
    strides (k, r, s, cg)).
    """
    dy = _f64(dy)
    w = _f64(w)
    if dy_shape is not None:
        N, Ho, Wo, K = dy_shape
        last = sum((d - 1) * st for d, st in zip(dy_shape, dy_strides))
        if last >= dy.size:
            raise ValueError("dY strides reach past the buffer")
    else:
        N, Ho, Wo, K = dy.shape
    if kind == "pointwise":
        C = w.shape[1]
        groups = 1
    elif kind == "depthwise":
        C = w.shape[2]
        groups = C
    else:
        assert C is not None and groups is not None
    g = _geom(N, H, W, C, K, KH, KW, S, ph, pw, groups)
    ys = dy_strides if dy_strides is not None else (Ho * Wo * K, Wo * K, K, 1)
    ws = w_strides if w_strides is not None else _w_strides(kind, KH, KW, C, K, groups)
    dx = np.empty((N, H, W, C), dtype=np.float64)
    rc = _load().oracle_dgrad(ctypes.byref(g), _dptr(dy), _i64(ys), _dptr(w), _i64(ws), _dptr(dx))
    if rc:
        raise ValueError("oracle_dgrad rejected the geometry")
    return dx


def dgrad_points(dy, w, pts, *, kind: str, H: int, W: int, KH: int = 1, KW: int = 1,
                 S: int = 1, ph: int = 0, pw: int = 0, groups: int | None = None,
                 C: int | None = None, N: int | None = None) -> np.ndarray:
    """dX at the (n, h, w, c) rows of pts, one element at a time (C: oracle_dgrad_points).

    dy may be given for a subset of the batch only when pts index within it.
    """
    dy = _f64(dy)
    w = _f64(w)
    Nd, Ho, Wo, K = dy.shape
    if kind == "pointwise":
        C = w.shape[1]
        groups = 1
    elif kind == "depthwise":
        C = w.shape[2]
        groups = C
    g = _geom(Nd if N is None else N, H, W, C, K, KH, KW, S, ph, pw, groups)
    ys = (Ho * Wo * K, Wo * K, K, 1)
    ws = _w_strides(kind, KH, KW, C, K, groups)
    pts = np.ascontiguousarray(np.asarray(pts, dtype=np.int64).reshape(-1, 4))
    out = np.empty(len(pts), dtype=np.float64)
    rc = _load().oracle_dgrad_points(ctypes.byref(g), _dptr(dy), _i64(ys), _dptr(w), _i64(ws),
                                     pts.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)),
                                     len(pts), _dptr(out))
    if rc:
        raise ValueError("oracle_dgrad_points rejected the geometry or a point")
    return out


def conv_fwd(x, w, *, kind: str, K: int | None = None, KH: int = 1, KW: int = 1, S: int = 1,
             ph: int = 0, pw: int = 0, groups: int | None = None) -> np.ndarray:
    """Forward convolution y = conv(x, W) in fp64, gather form (C: oracle_conv_fwd)."""
    x = _f64(x)
    w = _f64(w)
    N, H, W, C = x.shape
    if kind == "pointwise":
        K = w.shape[0]
        groups = 1
    elif kind == "depthwise":
        K = C
        groups = C
    Ho, Wo = out_dims(H, W, KH, KW, S, ph, pw)
    g = _geom(N, H, W, C, K, KH, KW, S, ph, pw, groups)
    ws = _w_strides(kind, KH, KW, C, K, groups)
    y = np.empty((N, Ho, Wo, K), dtype=np.float64)
    if _load().oracle_conv_fwd(ctypes.byref(g), _dptr(x), _dptr(w), _i64(ws), _dptr(y)):
        raise ValueError("oracle_conv_fwd rejected the geometry")
    return y


def dw_rotated(dy, w, *, H: int, W: int, ph: int, pw: int) -> np.ndarray:
    """Stride-1 depthwise dgrad as a correlation with the rotated filter (C: oracle_dw_rotated)."""
    dy = _f64(dy)
    w = _f64(w)
    N, Ho, Wo, C = dy.shape
    KH, KW = w.shape[:2]
    g = _geom(N, H, W, C, C, KH, KW, 1, ph, pw, C)
    dx = np.empty((N, H, W, C), dtype=np.float64)
    if _load().oracle_dw_rotated(ctypes.byref(g), _dptr(dy), _dptr(w), _dptr(dx)):
        raise ValueError("oracle_dw_rotated rejected the geometry")
    return dx


def dw_rowstream(dy, w, *, H: int, W: int, S: int, ph: int, pw: int) -> np.ndarray:
    """Depthwise dgrad by the row-streaming schedule (C: oracle_dw_rowstream)."""
    dy = _f64(dy)
    w = _f64(w)
    N, Ho, Wo, C = dy.shape
    KH, KW = w.shape[:2]
    g = _geom(N, H, W, C, C, KH, KW, S, ph, pw, C)
    dx = np.empty((N, H, W, C), dtype=np.float64)
    if _load().oracle_dw_rowstream(ctypes.byref(g), _dptr(dy), _dptr(w), _dptr(dx)):
        raise ValueError("oracle_dw_rowstream rejected the geometry")
    return dx


# --- Whole-array fp64 forms (numpy), for comparing every element of full-size
# problems in seconds.  Each is the definition written with array slices; each is
# pinned to the scatter loop above on small problems (tests/test_oracle.py).

def pointwise_matmul(dy, w) -> np.ndarray:
    """Pointwise dgrad as the plain product dX[M, C] = dY[M, K] . W[K, C] in fp64,
    M = N*H*W ("add the pointwise fast path dgrad was missing", Technical Details:
    dY offset m*K + k, W offset k*C + c)."""
    dy = np.asarray(dy, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    N, H, W, K = dy.shape
    return (dy.reshape(-1, K) @ w).reshape(N, H, W, w.shape[1])


def depthwise_taps(dy, w, *, H: int, W: int, S: int = 1, ph: int = 0, pw: int = 0) -> np.ndarray:
    """Depthwise dgrad (groups = C) in fp64 as one strided slice update per filter tap.

    The scatter form of the adjoint: dY[n, ho, wo, c] * W[r][s][c] adds into
    dX[n, ho*S - ph + r, wo*S - pw + s, c]; for a fixed tap (r, s) the targets of
    all (ho, wo) form a strided slice of dX, so each tap is one array update.
    Targets outside [0, H) x [0, W) are dropped ("channel-packed and large-filter
    depthwise dgrad", Technical Details: the stride / padding geometry and the
    row-streaming schedule apply exactly these scatter targets)."""
    dy = np.asarray(dy, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    N, Ho, Wo, C = dy.shape
    KH, KW = w.shape[:2]
    dx = np.zeros((N, H, W, C), dtype=np.float64)

    def span(extent_out, extent_in, off):
        # ho values whose target ho*S + off lies in [0, extent_in)
        lo = max(0, -(-(0 - off) // S))
        hi = min(extent_out, (extent_in - 1 - off) // S + 1) if extent_in - 1 - off >= 0 else 0
        return lo, max(lo, hi)

    for r in range(KH):
        h_lo, h_hi = span(Ho, H, r - ph)
        if h_lo >= h_hi:
            continue
        for s in range(KW):
            w_lo, w_hi = span(Wo, W, s - pw)
            if w_lo >= w_hi:
                continue
            h0 = h_lo * S - ph + r
            w0 = w_lo * S - pw + s
            dx[:, h0:h0 + (h_hi - h_lo - 1) * S + 1:S, w0:w0 + (w_hi - w_lo - 1) * S + 1:S, :] += \
                dy[:, h_lo:h_hi, w_lo:w_hi, :] * w[r, s, :]
    return dx
