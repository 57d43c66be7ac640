"""Benchmark: dgrad effective TFLOP/s and HBM GB/s on B200, % of roofline.

One step = one pass of the whole dgrad hot path over the benchmark suite: the
pointwise fp32 problem, depthwise 3x3, pointwise bf16 (tcgen05), depthwise
31x31, and the non-square / strided set (51x5, 5x51, 7x7 stride 2), each one
kernel launch through the C ABI on inputs already resident in HBM.  Inputs
rotate through several copies per problem so that every launch reads data that
is not in L2 (each problem's copies together exceed twice the L2 size).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload suite|<problem>] [--impl ours|reference]

--impl reference times the fp64 CPU oracle on the host cores (a bounded sample
of the same workload each step).  Under torchrun every rank runs its own replica
(no collective: dgrad of independent batches shares nothing); rank 0 prints one
JSON line with the job total and the max-over-ranks time.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import shutil
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from convolution_backward_b200 import synthetic  # noqa: E402

METRIC = "dgrad effective TFLOP/s and HBM GB/s on 1 B200, % of roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                  "sm_max_mhz": 1965.0}
FP32_LANES_PER_SM = 128
KERN_REPS = 10   # separately timed replays per kernel graph; the median is reported


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def workload_problems(name: str):
    if name == "suite":
        return synthetic.all_problems()
    if name in synthetic.WORKLOADS:
        return synthetic.WORKLOADS[name]
    if name in synthetic.EXTRA_WORKLOADS:
        return synthetic.EXTRA_WORKLOADS[name]
    return [synthetic.problem(name)]


# ------------------------------------------------------------------ distributed

def dist_init():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        import torch
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(world, value: float, device=None) -> float:
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(flops_per_rank: float, world: int, step_ms_max: float) -> float:
    """Whole-job TFLOP/s: every rank's work over the slowest rank's step time."""
    return flops_per_rank * world / (step_ms_max * 1e-3) / 1e12


# ----------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi sampling of SM clock and throttle reasons while the timed region runs."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        exe = shutil.which("nvidia-smi")
        if not exe:
            return
        self.proc = subprocess.Popen([exe, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                      "-i", str(self.gpu), "-lms", "100"], stdout=subprocess.PIPE,
                                     stderr=subprocess.DEVNULL, text=True)
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if not self.proc:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=2)
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------ CPU oracle

def _sample_call(p, inp, n, c):
    """Oracle arguments for a bounded sample of problem p and the nominal FLOPs it covers.

    Depthwise: the first n images and first c channels (channels of a depthwise
    dgrad are independent).  Dense: the first n images and the first c dX
    channels (each dX channel reads only its own filter slice).  Pointwise: the
    first n*c rows of dY[M, K] as n pseudo-images of c rows (rows of a pointwise
    dgrad are independent)."""
    if p.kind == "dense":
        dy = inp.dy[:n]
        w = np.ascontiguousarray(inp.w[:, :, :, :c].transpose(2, 0, 1, 3))   # (K, KH, KW, c): grouped layout
        kw = dict(kind="grouped", groups=1, C=c, H=p.H, W=p.W, KH=p.KH, KW=p.KW, S=p.stride, ph=p.pad_h,
                  pw=p.pad_w)
        return dy, w, kw, p.nominal_flops() * n * c // (p.N * p.C)
    if p.kind == "pointwise":
        rows = n * c
        dy = inp.dy.reshape(-1, p.K)[:rows].reshape(n, 1, c, p.K)
        kw = dict(kind="pointwise", H=1, W=c)
        return dy, inp.w, kw, p.nominal_flops() * rows // (p.N * p.H * p.W)
    dy = inp.dy[:n, :, :, :c]
    w = inp.w[:, :, :c]
    kw = dict(kind="depthwise", H=p.H, W=p.W, KH=p.KH, KW=p.KW, S=p.stride, ph=p.pad_h, pw=p.pad_w)
    return dy, w, kw, p.nominal_flops() * n * c // (p.N * p.C)


def oracle_sample_plan(problems, inputs, budget_s: float):
    """Per problem a sample (n, c) sized so the whole suite takes about budget_s
    of oracle time on this host: n = min(batch, threads) so every thread works,
    c calibrated from one small timed call."""
    import oracle
    threads = oracle.get_threads()
    per = budget_s / max(1, len(problems))
    plan = []
    for p in problems:
        inp = inputs[p.name]
        per_image = p.kind in ("depthwise", "dense")
        n = min(p.N, threads) if per_image else threads
        full_c = p.C if per_image else (p.N * p.H * p.W) // n
        c = min(full_c, 8 if per_image else 64)
        dy, w, kw, _ = _sample_call(p, inp, n, c)
        t0 = time.perf_counter()
        oracle.dgrad(dy, w, **kw)
        dt = max(time.perf_counter() - t0, 1e-4)
        c = int(max(1, min(full_c, c * per / dt)))
        if per_image and c >= 8:
            c -= c % 8
        plan.append((p, n, c))
    return plan, threads


def run_oracle_sample(plan, inputs):
    import oracle
    flops = 0
    secs = 0.0
    for p, n, c in plan:
        dy, w, kw, fl = _sample_call(p, inputs[p.name], n, c)
        t0 = time.perf_counter()
        oracle.dgrad(dy, w, **kw)
        secs += time.perf_counter() - t0
        flops += fl
    return flops, secs


def describe_plan(plan):
    out = []
    for p, n, c in plan:
        if p.kind == "pointwise":
            out.append(f"{p.name}: {n * c}/{p.N * p.H * p.W} rows")
        else:
            out.append(f"{p.name}: {n}/{p.N} images x {c}/{p.C} channels")
    return "; ".join(out)


def cpu_baseline(problems, inputs, budget_s=15.0):
    """The oracle on the host cores over a bounded sample: the suite rate, the
    rate of each problem, and (on a smaller sample) the rate of one thread."""
    import oracle
    plan, threads = oracle_sample_plan(problems, inputs, budget_s)
    flops, secs = 0, 0.0
    per_problem = []
    for item in plan:
        f, t = run_oracle_sample([item], inputs)
        flops += f
        secs += t
        per_problem.append({"problem": item[0].name, "tflops": round(f / t / 1e12, 6), "seconds": round(t, 3)})
    # one thread: the same problems on a sample `threads` times smaller (one image, or 1/threads of the rows)
    small = []
    for p, n, c in plan:
        if p.kind == "pointwise":
            small.append((p, n, max(1, c // threads)))
        else:
            small.append((p, 1, c))
    oracle.set_threads(1)
    try:
        f1, t1 = run_oracle_sample(small, inputs)
    finally:
        oracle.set_threads(threads)
    return {"value": flops / secs / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
            "sample": describe_plan(plan), "seconds": round(secs, 3), "flops": flops,
            "per_problem": per_problem,
            "single_thread": {"value": round(f1 / t1 / 1e12, 6), "unit": "TFLOP/s", "cores": 1,
                              "sample": describe_plan(small), "seconds": round(t1, 3)}}


# ---------------------------------------------------------------------- ours

def inbounds_flops(p) -> int:
    """FLOPs of the taps that land inside dX (zero padding skipped): the nominal
    count is 2*N*Ho*Wo*K*(C/groups)*KH*KW, padded taps included; here each of the
    two spatial axes counts only the (output, tap) pairs whose dX position
    ho*S - pad + r lies in [0, H) (and likewise for columns)."""
    rows = sum(1 for ho in range(p.Ho) for r in range(p.KH) if 0 <= ho * p.stride - p.pad_h + r < p.H)
    cols = sum(1 for wo in range(p.Wo) for s in range(p.KW) if 0 <= wo * p.stride - p.pad_w + s < p.W)
    return 2 * p.N * rows * cols * p.K * (p.C // p.groups)


def traffic_record():
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(path):
        return {}
    with open(path) as f:
        return json.load(f)


def source_digest(relpath: str) -> str:
    h = hashlib.sha256()
    with open(os.path.join(ROOT, relpath), "rb") as f:
        h.update(f.read())
    return h.hexdigest()[:16]


KERNEL_SOURCE = {"pointwise": {"bf16": "convolution_backward_b200/csrc/pointwise_tc.cu",
                               "f32": "convolution_backward_b200/csrc/pointwise_f32.cu"},
                 "rotated": "convolution_backward_b200/csrc/dw_rotated.cu",
                 "rowstream": "convolution_backward_b200/csrc/dw_rowstream.cu",
                 "rowstream_fast": "convolution_backward_b200/csrc/dw_rowstream_fast.cu",
                 "tile": "convolution_backward_b200/csrc/dw_tile.cu",
                 "toeplitz": "convolution_backward_b200/csrc/dw_toeplitz.cu",
                 "dense": "convolution_backward_b200/csrc/dense_tc.cu"}


def kernel_of(p):
    if p.variant == "splitk":
        return "pw_tc_splitk_kernel", KERNEL_SOURCE["pointwise"]["bf16"]
    if p.variant == "tc":
        return "dw_toeplitz_kernel", KERNEL_SOURCE["toeplitz"]
    if p.kind == "dense":
        return "dense_tc_kernel", KERNEL_SOURCE["dense"]
    if p.variant == "rotated" and p.KH * p.KW > 49:
        return "dw_rot_kernel", KERNEL_SOURCE["rotated"]
    if p.kind == "pointwise":
        return ("pw_tc_pair_kernel" if p.dtype == "bf16" else "pw_f32_kernel"), KERNEL_SOURCE["pointwise"][p.dtype]
    if p.stride == 1 and p.dtype == "bf16" and p.KH <= 7 and p.KW <= 7 and p.KH == p.KW and p.KH % 2 == 1 \
            and p.KH >= 3:
        return "dw_tile_kernel", KERNEL_SOURCE["tile"]
    if p.stride == 1:
        return "dw_rot_kernel", KERNEL_SOURCE["rotated"]
    if p.dtype == "bf16" and (p.KH, p.KW, p.stride) in ((7, 7, 2), (5, 5, 2), (3, 3, 2)):
        return "dw_rs_reg_kernel", KERNEL_SOURCE["rowstream_fast"]
    return "dw_rowstream_kernel", KERNEL_SOURCE["rowstream"]


def run_ours(args, world, rank, local):
    import torch
    import convolution_backward_b200 as cb

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    peaks, peak_src = load_peaks()
    problems = workload_problems(args.workload)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    sms = torch.cuda.get_device_properties(dev).multi_processor_count

    inputs = {p.name: synthetic.make_inputs(p) for p in problems}
    sets = {}
    workspaces = {}
    for p in problems:
        inp = inputs[p.name]
        if p.dtype == "bf16":
            dy = torch.from_numpy(inp.dy_bits.view(np.int16)).view(torch.bfloat16).to(dev)
            w = torch.from_numpy(inp.w_bits.view(np.int16)).view(torch.bfloat16).to(dev)
        else:
            dy = torch.from_numpy(inp.dy).to(dev)
            w = torch.from_numpy(inp.w).to(dev)
        copies = max(2, math.ceil(2 * l2 / p.algorithmic_bytes()) + 1)
        sets[p.name] = [(dy.clone(), w.clone(), torch.empty(p.dx_shape, dtype=dy.dtype, device=dev))
                        for _ in range(copies)]
        if p.variant == "splitk":
            nb, _ = cb.splitk_workspace_bytes(p.N, p.H, p.W, p.K, p.C, 0)
            workspaces[p.name] = torch.empty(max(nb, 16), dtype=torch.uint8, device=dev)
        if p.variant == "tc":
            nb = cb.depthwise_tc_workspace_bytes(p.N, p.H, p.W, p.C, p.KH, p.KW, p.pad_h, p.pad_w)
            workspaces[p.name] = torch.empty(max(nb, 16), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def call(p, dy, w, out):
        if p.variant == "splitk":
            cb.pointwise_splitk(dy, w, splits=0, workspace=workspaces[p.name], out=out)
        elif p.variant == "tc":
            cb.depthwise_tc(dy, w, H=p.H, Wd=p.W, pad_h=p.pad_h, pad_w=p.pad_w, workspace=workspaces[p.name],
                            out=out)
        elif p.kind == "pointwise":
            cb.pointwise(dy, w, out=out)
        elif p.kind == "dense":
            cb.dense(dy, w, H=p.H, Wd=p.W, stride=p.stride, pad_h=p.pad_h, pad_w=p.pad_w, out=out)
        else:
            cb.depthwise(dy, w, H=p.H, Wd=p.W, stride=p.stride, pad_h=p.pad_h, pad_w=p.pad_w, out=out,
                         mode="rotated" if p.variant == "rotated" else "auto")

    def step(i, evs=None):
        for j, p in enumerate(problems):
            s = sets[p.name]
            dy, w, out = s[i % len(s)]
            if evs is not None:
                evs[j][0].record(stream)
            call(p, dy, w, out)
            if evs is not None:
                evs[j][1].record(stream)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    cb.check_status()

    # CUDA graphs: the timed step is one graph holding `steps` whole steps (every
    # problem once per step, copies rotating), and each problem also gets a graph
    # of back-to-back launches for its per-kernel duration.  Graph replay removes
    # host launch latency from the device timeline.
    g_steps = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_steps):
        for i in range(args.steps):
            step(args.warmup + i)
    reps = {}
    g_kern = []
    g_warm = []   # the same buffers every launch: a warm-L2 figure, reported separately
    for j, p in enumerate(problems):
        r = max(8, len(sets[p.name]))
        reps[j] = r
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(r):
                dy, w, out = sets[p.name][i % len(sets[p.name])]
                call(p, dy, w, out)
        g_kern.append(g)
        gw = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gw):
            for i in range(r):
                call(p, *sets[p.name][0])
        g_warm.append(gw)
    for _ in range(2):
        g_steps.replay()
        for g in g_kern + g_warm:
            g.replay()
    torch.cuda.synchronize()
    cb.check_status()

    # --- timed region
    barrier(world)
    torch.cuda.synchronize()
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    g_steps.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    step_ms = e0.elapsed_time(e1) / args.steps
    # per kernel: KERN_REPS separately timed replays of its graph, median (and min)
    kern_ms, kern_min_ms, warm_ms = [], [], []

    def timed_replays(g, r):
        out = []
        for _ in range(KERN_REPS):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            g.replay()
            b.record(stream)
            torch.cuda.synchronize()
            out.append(a.elapsed_time(b) / r)
        return out

    for j in range(len(problems)):
        t = timed_replays(g_kern[j], reps[j])
        kern_ms.append(statistics.median(t))
        kern_min_ms.append(min(t))
        warm_ms.append(statistics.median(timed_replays(g_warm[j], reps[j])))
    kern_iters = KERN_REPS
    clocks = sampler.stop()
    barrier(world)
    cb.check_status()
    # kernels one call launches: the tensor-core depthwise call runs the dY transpose (whose extra
    # CTAs pack the filter), the MMA kernel and the dX transpose; split-K runs the GEMM and the
    # reduction; every other call is one kernel
    per_call = [3 if p.variant == "tc" else 2 if p.variant == "splitk" else 1 for p in problems]
    n_launches = sum((args.steps + 2 * kern_iters * reps[j]) * per_call[j] for j in range(len(problems)))

    step_ms_max = max_over_ranks(world, step_ms, dev)
    flops_step = sum(p.nominal_flops() for p in problems)
    bytes_step = sum(p.algorithmic_bytes() for p in problems)
    value = job_throughput(flops_step, world, step_ms_max)

    # --- per-kernel rooflines
    sm_max = clocks.get("sm_max_mhz") or peaks.get("sm_max_mhz", 1965.0)
    fp32_peak = sms * FP32_LANES_PER_SM * 2 * sm_max * 1e6 / 1e12
    hbm = peaks["hbm_gbs"]
    bf16_peak = peaks["bf16_tflops"]
    traffic = traffic_record()
    per_kernel = []
    for p, ms, ms_min, ms_warm in zip(problems, kern_ms, kern_min_ms, warm_ms):
        fl = p.nominal_flops()
        fl_in = inbounds_flops(p)
        by = p.algorithmic_bytes()
        tf = fl / (ms * 1e-3) / 1e12
        gbs = by / (ms * 1e-3) / 1e9
        t_bytes = by / (hbm * 1e9)
        if (p.kind in ("pointwise", "dense") and p.dtype == "bf16") or p.variant == "tc":
            # tensor-core paths: nominal FLOPs against the bf16 tensor peak (the banded-Toeplitz
            # depthwise issues about 3x its nominal FLOPs as MMAs; the fraction stays nominal)
            t_flop = fl / (bf16_peak * 1e12)
            bound = "tensor"
        else:
            t_flop = fl / (fp32_peak * 1e12)
            bound = "alu"
        frac = max(t_bytes, t_flop) / (ms * 1e-3)
        kname, src = kernel_of(p)
        rec = traffic.get(p.name)
        tr = None
        if rec and rec.get("source_sha") == source_digest(src):
            tr = rec.get("bytes_per_launch")
        per_kernel.append({
            "problem": p.name, "kernel": kname, "us": round(ms * 1e3, 3), "tflops": round(tf, 3),
            "gbs": round(gbs, 1), "roofline_frac": round(frac, 4),
            "binding": "hbm" if t_bytes >= t_flop else bound,
            "floor_us": round(max(t_bytes, t_flop) * 1e6, 3),
            "frac_of_tensor_peak": round(tf / bf16_peak, 4) if bound == "tensor" else None,
            "frac_of_hbm": round(gbs / hbm, 4),
            "fp32_floor_us": round(fl / (fp32_peak * 1e12) * 1e6, 3) if p.kind == "depthwise" else None,
            # the depthwise roofline as the benchmark's target defines it (bytes at HBM
            # bandwidth against nominal FMAs at the FP32 peak), for every depthwise kernel,
            # tensor-core ones included
            "frac_hbm_fp32_roofline": (round(max(t_bytes, fl / (fp32_peak * 1e12)) / (ms * 1e-3), 4)
                                       if p.kind == "depthwise" else None),
            "inbounds_flop": fl_in, "nominal_flop": fl, "inbounds_tflops": round(fl_in / (ms * 1e-3) / 1e12, 3),
            "us_min": round(ms_min * 1e3, 3), "replays": KERN_REPS,
            "warm_l2_us": round(ms_warm * 1e3, 3),
            "warm_l2_tflops": round(fl / (ms_warm * 1e-3) / 1e12, 3),
            "dram_bytes_per_launch": tr})
    dom = max(range(len(problems)), key=lambda j: kern_ms[j])
    dp = problems[dom]
    dk = per_kernel[dom]
    if (dp.kind in ("pointwise", "dense") and dp.dtype == "bf16") or dp.variant == "tc":
        roof = {"bound": "tensor", "achieved": dk["tflops"], "peak": bf16_peak, "unit": "TFLOP/s",
                "frac": round(dk["tflops"] / bf16_peak, 4), "traffic": dk["dram_bytes_per_launch"]}
    elif dk["binding"] == "hbm":
        roof = {"bound": "hbm", "achieved": dk["gbs"], "peak": hbm, "unit": "GB/s",
                "frac": round(dk["gbs"] / hbm, 4), "traffic": dk["dram_bytes_per_launch"]}
    else:
        roof = {"bound": "alu", "achieved": dk["tflops"], "peak": round(fp32_peak, 2), "unit": "TFLOP/s",
                "frac": round(dk["tflops"] / fp32_peak, 4), "traffic": dk["dram_bytes_per_launch"]}
    if dp.variant == "tc":
        roof["basis"] = ("nominal FLOPs against the bf16 tensor peak (the kernel runs on the tensor cores); "
                         "frac_hbm_fp32_roofline is the depthwise roofline of the benchmark's target: "
                         "max(bytes / HBM, nominal FLOPs / FP32 peak) / time")
        roof["frac_hbm_fp32_roofline"] = dk["frac_hbm_fp32_roofline"]
    roof.update({"kernel": dk["kernel"], "problem": dp.name,
                 "peak_source": (f"{peak_src} (MEASURED_PEAKS.json)" if roof["bound"] != "alu" else
                                 f"derived: {sms} SMs x {FP32_LANES_PER_SM} FMA/clk x 2 x {sm_max:.0f} MHz")})

    # --- FMA-rate probe (measured fp32 FMA throughput at this run's clocks)
    probe = {}
    sink = torch.zeros(sms * 8, device=dev)
    for packed in (0, 1):
        cb.fma_probe(sms * 8, 64, bool(packed), sink)
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fl = cb.fma_probe(sms * 8, 20000, bool(packed), sink)
        b.record(stream)
        torch.cuda.synchronize()
        probe["ffma2" if packed else "ffma"] = round(fl / (a.elapsed_time(b) * 1e-3) / 1e12, 2)

    # --- end to end through the public API from pinned host buffers
    host = {}
    h2d = d2h = 0
    for p in problems:
        dy, w, out = sets[p.name][0]
        host[p.name] = (dy.cpu().pin_memory(), w.cpu().pin_memory(),
                        torch.empty(p.dx_shape, dtype=dy.dtype).pin_memory())
        h2d += dy.numel() * dy.element_size() + w.numel() * w.element_size()
        d2h += out.numel() * out.element_size()
    e2e_steps = max(3, min(args.steps, 10))
    # Copies in on one stream, copies out on another, the calls on the launching stream, so the
    # two PCIe directions and the kernels overlap across problems and steps.  Input and output
    # buffers rotate over the same copies as the device-timed step; events keep every buffer's
    # uses in order (its H2D after the last call that read it, its call after the last D2H of
    # its output).
    s_in = torch.cuda.Stream(dev)
    s_out = torch.cuda.Stream(dev)
    comp_done, d2h_done = {}, {}

    def e2e_step(i, start=None):
        for p in problems:
            hdy, hw, hout = host[p.name]
            k = i % len(sets[p.name])
            dy, w, out = sets[p.name][k]
            key = (p.name, k)
            with torch.cuda.stream(s_in):
                if start is not None:
                    s_in.wait_event(start)
                if key in comp_done:
                    s_in.wait_event(comp_done[key])
                dy.copy_(hdy, non_blocking=True)
                w.copy_(hw, non_blocking=True)
                ev_in = torch.cuda.Event()
                ev_in.record(s_in)
            stream.wait_event(ev_in)
            if key in d2h_done:
                stream.wait_event(d2h_done[key])
            call(p, dy, w, out)
            ev_c = torch.cuda.Event()
            ev_c.record(stream)
            comp_done[key] = ev_c
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_c)
                hout.copy_(out, non_blocking=True)
                ev_o = torch.cuda.Event()
                ev_o.record(s_out)
                d2h_done[key] = ev_o

    e2e_step(0)
    torch.cuda.synchronize()
    barrier(world)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for i in range(e2e_steps):
        e2e_step(i + 1, start=a if i == 0 else None)
    stream.wait_stream(s_out)
    b.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(world, a.elapsed_time(b) / e2e_steps, dev)
    cb.check_status()

    out = {
        "metric": METRIC, "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(step_ms_max, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16+f32",
        "data": "synthetic (seeded numpy draws of the named shapes and distributions)",
        "config": {"workload": args.workload if args.workload != "suite" else
                   "dgrad suite: " + ", ".join(p.name for p in problems),
                   "problems": [p.name for p in problems],
                   "l2": f"each problem rotates over input copies totalling > 2x L2 ({l2 >> 20} MiB)",
                   "parallelism": f"replicas x{world}"},
        "hbm_gbs_effective": round(bytes_step * world / (step_ms_max * 1e-3) / 1e9, 1),
        "roofline": roof,
        "per_kernel": per_kernel,
        "fp32_fma_probe_tflops": probe,
        "clocks": clocks,
        "e2e": {"value": round(flops_step * world / (e2e_ms * 1e-3) / 1e12, 3), "unit": "TFLOP/s",
                "ms_per_step": round(e2e_ms, 4), "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": n_launches,
        "timing": ("CUDA graphs replayed on the launching stream, CUDA events around the replay; the step "
                   "is one graph of `steps` steps; per_kernel us = median of 10 separately timed replays of "
                   "a graph of back-to-back launches over rotating cold copies (warm_l2_us: the same buffers "
                   "every launch, so inputs that fit stay in L2)"),
        "peaks": {"source": peak_src, "hbm_gbs": hbm, "bf16_tflops": bf16_peak,
                  "fp32_tflops_at_max_clock": round(fp32_peak, 2)},
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(problems, inputs, budget_s=args.cpu_budget)
    return out


def run_reference(args, world, rank):
    problems = workload_problems(args.workload)
    inputs = {p.name: synthetic.make_inputs(p) for p in problems}
    budget = args.cpu_budget / max(1, args.steps + args.warmup)
    plan, threads = oracle_sample_plan(problems, inputs, budget)
    for _ in range(args.warmup):
        run_oracle_sample(plan, inputs)
    tot_flops, tot_s = 0, 0.0
    for _ in range(args.steps):
        f, s = run_oracle_sample(plan, inputs)
        tot_flops += f
        tot_s += s
    value = tot_flops / tot_s / 1e12
    sample = describe_plan(plan)
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": tot_s / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded numpy draws of the named shapes and distributions)",
        "config": {"workload": args.workload if args.workload != "suite" else
                   "dgrad suite: " + ", ".join(p.name for p in problems),
                   "problems": [p.name for p in problems], "parallelism": "host cores (OpenMP)"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="suite")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-budget", type=float, default=15.0,
                    help="seconds of oracle time (cpu_baseline; for --impl reference, the whole run)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        # The oracle runs on the host cores of rank 0 alone; other ranks exit at once.
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        if rank == 0:
            print(json.dumps(run_reference(args, world, rank)), flush=True)
        return
    world, rank, local = dist_init()
    out = run_ours(args, world, rank, local)
    if rank == 0:
        print(json.dumps(out), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
