"""Build libdgrad.so (and libdgrad_debug.so) in-tree with nvcc for sm_100a.

Every .cu file under csrc/ is compiled to an object in _build/ (in parallel),
then linked into convolution_backward_b200/libdgrad.so with the CUDA runtime
linked statically.  ptxas register/spill reports go to _build/ptxas.log.  The
same sources built with -DDGRAD_DEBUG (objects in _build/debug/) give
libdgrad_debug.so, whose kernels check every hand-indexed store against its
output buffer.  Rebuilds only when a source, header or this file is newer than
a library.
"""
from __future__ import annotations

import concurrent.futures as cf
import glob
import os
import shutil
import subprocess

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libdgrad.so")
LIB_DEBUG = os.path.join(PKG, "libdgrad_debug.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
CFLAGS = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xptxas", "-v",
                 "--expt-relaxed-constexpr", "-I", INCLUDE, "-I", CSRC]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _inputs():
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    deps = srcs + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + \
        glob.glob(os.path.join(INCLUDE, "*.h")) + [os.path.abspath(__file__)]
    return srcs, deps


def needs_build() -> bool:
    if not os.path.exists(LIB) or not os.path.exists(LIB_DEBUG):
        return True
    _, deps = _inputs()
    t = min(os.path.getmtime(LIB), os.path.getmtime(LIB_DEBUG))
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not needs_build():
        return LIB
    nvcc = _nvcc()
    os.makedirs(BUILD, exist_ok=True)
    srcs, _ = _inputs()

    debug_dir = os.path.join(BUILD, "debug")
    os.makedirs(debug_dir, exist_ok=True)

    def compile_one(job):
        src, debug = job
        obj = os.path.join(debug_dir if debug else BUILD, os.path.basename(src) + ".o")
        cmd = [nvcc, *CFLAGS, *(["-DDGRAD_DEBUG"] if debug else []), "-c", src, "-o", obj]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed on {src}:\n{r.stdout}\n{r.stderr}")
        return obj, r.stderr

    jobs = [(s, False) for s in srcs] + [(s, True) for s in srcs]
    with cf.ThreadPoolExecutor(max_workers=min(16, os.cpu_count() or 4)) as ex:
        results = list(ex.map(compile_one, jobs))
    release, debug = results[:len(srcs)], results[len(srcs):]
    with open(os.path.join(BUILD, "ptxas.log"), "w") as f:
        for (obj, log), src in zip(release, srcs):
            f.write(f"==== {os.path.basename(src)}\n{log}\n")
    for lib, objs in ((LIB, release), (LIB_DEBUG, debug)):
        tmp = lib + f".tmp{os.getpid()}"
        cmd = [nvcc, *ARCH, "-shared", "-cudart", "static", "-o", tmp, *[o for o, _ in objs],
               "-ldl", "-lpthread", "-lrt"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
        os.replace(tmp, lib)
    if verbose:
        print(f"built {LIB}")
    return LIB


if __name__ == "__main__":
    build(force=True, verbose=True)
