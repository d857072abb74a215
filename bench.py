#!/usr/bin/env python
"""Benchmark of the tile-hybrid (dense | 2:4) decode GEMV on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl hyb|reference]
                    [--workload NAME] [--sweep]

One step = one hyb_spmv call (the whole hot path: stream the packed values and
masks, decode, fp32 FMA, reduce, store) on the headline workload:

    ffn_down_4096x14336_f0.5_b1 -- the Llama-shaped FFN down projection
    (n=4096 outputs, k=14336 inputs), bf16 N(0, 0.02) with 1 % x20 outliers,
    128x128 tiles of which half are 2:4 (seeded shuffle), batch 1.

Inputs are larger than L2: each step uses the next of 16 packed copies of the
matrix (1.47 GB in total), so every step streams from HBM.  The printed value
is achieved GB/s over the algorithmic bytes (packed values + masks + tile map +
x + y).  With N > 1 (torchrun) every rank runs its own replica (the product is
not sharded; weak scaling) and the time is the max over ranks.

--impl reference times the CPU oracle on a bounded row sample of the same
workload (rank 0 only).
"""
import argparse
import ctypes
import hashlib
import json
import os
import re
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from sparse_weight_b200 import hyb, inputs  # noqa: E402

FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0
ROTATE = 16

WORKLOADS = {
    # name: (n, k, b1, b2, frac, batch, std, outliers)
    "ffn_down_4096x14336_f0.5_b1": (4096, 14336, 128, 128, 0.5, 1, 0.02, 0.01),
    "ffn_up_14336x4096_f0.5_b1": (14336, 4096, 128, 128, 0.5, 1, 0.02, 0.01),
    "attn_4096x4096_bern0.5_b1": (4096, 4096, 128, 128, None, 1, 0.02, 0.0),
    "ffn_down_4096x14336_f0.5_b4": (4096, 14336, 128, 128, 0.5, 4, 0.02, 0.01),
    "ffn_down_4096x14336_f0.5_b8": (4096, 14336, 128, 128, 0.5, 8, 0.02, 0.01),
    "ffn_down_4096x14336_f0.5_b16": (4096, 14336, 128, 128, 0.5, 16, 0.02, 0.01),
    "ffn_down_4096x14336_f0.0_b1": (4096, 14336, 128, 128, 0.0, 1, 0.02, 0.01),
    "ffn_down_4096x14336_f1.0_b1": (4096, 14336, 128, 128, 1.0, 1, 0.02, 0.01),
    "ffn_down_4096x14336_f1.0_b4": (4096, 14336, 128, 128, 1.0, 4, 0.02, 0.01),
    "ffn_down_4096x14336_f1.0_b16": (4096, 14336, 128, 128, 1.0, 16, 0.02, 0.01),
    "ffn_down_4096x14336_f0.0_b16": (4096, 14336, 128, 128, 0.0, 16, 0.02, 0.01),
    # Llama-3.3-70B FFN matrices, all 2:4, with a low-rank term (rank below)
    "llama70b_down_8192x28672_lr128_b1": (8192, 28672, 128, 128, 1.0, 1, 0.015, 0.0),
    "llama70b_gate_28672x8192_lr128_b1": (28672, 8192, 128, 128, 1.0, 1, 0.015, 0.0),
    "llama70b_down_8192x28672_lr64_b1": (8192, 28672, 128, 128, 1.0, 1, 0.015, 0.0),
    "llama70b_down_8192x28672_lr128_b4": (8192, 28672, 128, 128, 1.0, 4, 0.015, 0.0),
}
# workloads with a low-rank term y += U (V^T x): name -> (rank, std of U and V)
LOWRANK = {
    "llama70b_down_8192x28672_lr128_b1": (128, 0.01),
    "llama70b_gate_28672x8192_lr128_b1": (128, 0.01),
    "llama70b_down_8192x28672_lr64_b1": (64, 0.01),
    "llama70b_down_8192x28672_lr128_b4": (128, 0.01),
}


# ---------------------------------------------------------------------------
# environment helpers
# ---------------------------------------------------------------------------

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            d = json.load(fh)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# Sources the streaming kernels (hybrid_tma_kernel, dense_gemv_kernel) are
# compiled from: a profile taken on them stays valid while these are unchanged.
PROFILED_SOURCES = ("hyb_internal.cuh", "hyb_spmv.cu")


def csrc_digest():
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "sparse_weight_b200", "csrc")
    for name in PROFILED_SOURCES:
        with open(os.path.join(csrc, name), "rb") as fh:
            h.update(name.encode())
            h.update(fh.read())
    return h.hexdigest()[:16]


def kernel_of(P):
    """Streaming kernel the product runs for P: the TMA-ring kernel when the
    library made a split for it (plan with CTAs), else the generic one."""
    return "hybrid_tma_kernel" if P.plan is not None and P.plan_ctas > 0 else "hybrid_rowwarp_kernel"


def profiled_traffic(workload, kernel):
    """DRAM bytes per launch from the committed ncu summary of this workload,
    if it was taken on the current kernel sources; else None."""
    path = os.path.join(ROOT, "profiles", f"{kernel}_{workload}.md")
    try:
        txt = open(path).read()
    except OSError:
        return None
    src = re.search(r"csrc_sha:\s*([0-9a-f]+)", txt)
    tr = re.search(r"dram_bytes_per_launch:\s*([0-9]+)", txt)
    if not src or not tr or src.group(1) != csrc_digest():
        return None
    return int(tr.group(1))


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4,
        "hw_slowdown": 0x8, "sync_boost": 0x10, "sw_thermal_slowdown": 0x20,
        "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80,
        "display_clock_setting": 0x100,
    }

    def __init__(self, index, period=0.005):
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self.ok = False
        self.period = period
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.nv = None

    def _sample(self):
        mhz = self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)
        bits = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        self.samples.append(mhz)
        for name, b in self.REASONS.items():
            if bits & b and name != "gpu_idle":
                self.reasons.add(name)

    def _run(self):
        while not self._stop.is_set():
            try:
                self._sample()
            except Exception:
                return
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *exc):
        if self.ok:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": len(self.samples)}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ---------------------------------------------------------------------------
# workload
# ---------------------------------------------------------------------------

def make_matrix(name):
    n, k, b1, b2, frac, batch, std, outliers = WORKLOADS[name]
    T = (n // b1) * (k // b2)
    if frac is None:
        tmap = inputs.tile_map_bernoulli(T, 0.5, inputs.seed_of(name, "map"))
    else:
        tmap = inputs.tile_map_fraction(T, frac, inputs.seed_of(name, "map"))
    W = inputs.weight(n, k, std, inputs.seed_of(name, "W"), outliers=outliers)
    return W, tmap


class Workload:
    def __init__(self, name, device, rotate=ROTATE):
        self.name = name
        n, k, b1, b2, frac, batch, std, outliers = WORKLOADS[name]
        self.n, self.k, self.b1, self.b2, self.batch = n, k, b1, b2, batch
        W, tmap = make_matrix(name)
        self.W_host, self.tmap = W, tmap
        Wd = W.to(device)
        base = hyb.pack(Wd, tmap, b1, b2)
        self.frac_real = float(tmap.mean())
        rotate = rotation(name, tmap, rotate)
        self.mats = [base] + [base.clone() for _ in range(rotate - 1)]
        self.dense = [Wd] + [Wd.clone() for _ in range(rotate - 1)]
        # the same W packed with every tile dense, streamed by the same kernel:
        # the dense reference that differs from the product only in the format
        dpk = hyb.pack(Wd, np.zeros_like(tmap), b1, b2)
        self.dense_packed = [dpk] + [dpk.clone() for _ in range(rotate - 1)]
        self.X = [inputs.activations(batch, k, inputs.seed_of(name, "X", i)).to(device)
                  for i in range(rotate)]
        self.Y = [torch.empty(batch, n, dtype=torch.float32, device=device)
                  for _ in range(rotate)]
        self.rank, lr_std = LOWRANK.get(name, (0, 0.0))
        self.U_host = self.V_host = None
        self.lr = None
        if self.rank:
            self.U_host, self.V_host = inputs.lowrank(n, k, self.rank, lr_std,
                                                      inputs.seed_of(name, "LR"))
            self.U, self.V = self.U_host.to(device), self.V_host.to(device)
            self.lr = hyb.HybLowrank(self.rank, hyb._bits(self.U).data_ptr(), self.rank,
                                     hyb._bits(self.V).data_ptr(), self.rank)
        self.ws = hyb.new_workspace(hyb.workspace_bytes(base, batch, self.rank), device)
        self.dws = hyb.new_workspace(hyb.dense_workspace_bytes(n, k, batch), device)
        # pre-marshalled C-ABI arguments (the timed loop only calls into C)
        L = hyb.lib()
        self.fn = L.hyb_spmm_skinny_ex
        self.dfn = L.hyb_gemv_dense_ex
        self.flags = 0  # launch options of every call (hyb_*_ex)
        self.structs = [m.struct() for m in self.mats]
        self.dstructs = [m.struct() for m in self.dense_packed]
        self.stream = torch.cuda.current_stream(device)
        self.set_stream(self.stream)
        # algorithmic bytes of one product: packed values + masks, tile map, x, y
        # (and U, V for a low-rank term)
        self.bytes_step = (base.nbytes() + base.num_tiles + 2 * batch * k + 4 * batch * n
                           + 2 * self.rank * (n + k))
        self.dense_bytes_step = 2 * n * k + 2 * batch * k + 4 * batch * n

    def set_stream(self, stream):
        """Marshal every call's arguments for launches on `stream`."""
        s = ctypes.c_void_p(stream.cuda_stream)
        n, k, batch = self.n, self.k, self.batch
        rotate = len(self.mats)
        f = self.flags
        lr = ctypes.byref(self.lr) if self.lr is not None else None
        self.args = [(ctypes.byref(self.structs[i]), batch, ctypes.c_void_p(self.X[i].data_ptr()),
                      k, ctypes.c_void_p(self.Y[i].data_ptr()), n, hyb.HYB_F32, lr, f,
                      ctypes.c_void_p(self.ws.data_ptr()), self.ws.numel(), s)
                     for i in range(rotate)]
        self.pargs = [(ctypes.byref(self.dstructs[i]), batch,
                       ctypes.c_void_p(self.X[i].data_ptr()), k,
                       ctypes.c_void_p(self.Y[i].data_ptr()), n, hyb.HYB_F32, None, f,
                       ctypes.c_void_p(self.ws.data_ptr()), self.ws.numel(), s)
                      for i in range(rotate)]
        self.dargs = [(n, k, batch, ctypes.c_void_p(self.dense[i].data_ptr()), k,
                       ctypes.c_void_p(self.X[i].data_ptr()), k,
                       ctypes.c_void_p(self.Y[i].data_ptr()), n, hyb.HYB_F32, f,
                       ctypes.c_void_p(self.dws.data_ptr()), self.dws.numel(), s)
                      for i in range(rotate)]

    def step(self, i):
        rc = self.fn(*self.args[i % len(self.args)])
        if rc != 0:
            raise hyb.HybError("hyb_spmm_skinny", rc)

    def check(self):
        """Raise if a kernel of the legs run so far flagged its workspace."""
        hyb.check_status(self.ws, self.stream)
        hyb.check_status(self.dws, self.stream)

    def dense_step(self, i):
        rc = self.dfn(*self.dargs[i % len(self.dargs)])
        if rc != 0:
            raise hyb.HybError("hyb_gemv_dense", rc)

    def dense_packed_step(self, i):
        rc = self.fn(*self.pargs[i % len(self.pargs)])
        if rc != 0:
            raise hyb.HybError("hyb_spmm_skinny", rc)


def max_over_ranks(ms, device, world):
    """The slowest rank's time (every rank calls this, in the same order)."""
    if world <= 1:
        return ms
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def aggregate_gbs(bytes_per_step, steps, ms, world):
    """Whole-job throughput: every rank streams its own replica."""
    return world * bytes_per_step * steps / (ms * 1e-3) / 1e9


def timed(fn, steps, warmup, stream, world=1):
    """Device time of `steps` calls (CUDA events on the launching stream),
    barrier + synchronize on both sides, max over ranks."""
    for i in range(warmup):
        fn(i)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(steps):
        fn(warmup + i)
    e1.record(stream)
    e1.synchronize()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    if world > 1:
        ms = max_over_ranks(ms, torch.device("cuda", torch.cuda.current_device()), world)
        torch.distributed.barrier()
    return ms


def graph_timed(wl, fn, steps, warmup, world=1, flags=0):
    """Device time of `steps` calls captured in one CUDA graph and replayed
    (the launch path of a decode engine): warm-up calls run eagerly first;
    CUDA events on the replay stream, barrier + synchronize on both sides, max
    over ranks.  `flags`: the calls' launch options (HYB_LAUNCH_OVERLAP_PREV:
    each call a programmatic dependent of the one before it)."""
    wl.flags = flags
    side = torch.cuda.Stream()
    with torch.cuda.stream(side):
        wl.set_stream(side)
        for i in range(warmup):
            fn(i)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        wl.set_stream(torch.cuda.current_stream())
        for i in range(steps):
            fn(warmup + i)
    wl.set_stream(wl.stream)
    torch.cuda.synchronize()
    g.replay()  # one untimed replay: first-launch costs of the graph
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(side):
        e0.record(side)
        g.replay()
        e1.record(side)
    e1.synchronize()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    if world > 1:
        ms = max_over_ranks(ms, torch.device("cuda", torch.cuda.current_device()), world)
        torch.distributed.barrier()
    del g
    wl.flags = 0
    wl.set_stream(wl.stream)
    return ms


def e2e_timed(wl, steps, warmup, stream, world=1):
    """Same metric through the public C ABI with host buffers: per step the
    pinned host x is copied in, the product runs, and y is copied back."""
    xh = [wl.X[i].cpu().pin_memory() for i in range(len(wl.X))]
    yh = torch.empty(wl.batch, wl.n, dtype=torch.float32).pin_memory()

    def one(i):
        j = i % len(wl.X)
        wl.X[j].copy_(xh[j], non_blocking=True)
        wl.step(j)
        yh.copy_(wl.Y[j], non_blocking=True)

    ms = timed(one, steps, warmup, stream, world)
    h2d = xh[0].numel() * xh[0].element_size()
    d2h = yh.numel() * yh.element_size()
    return ms, h2d, d2h


# ---------------------------------------------------------------------------
# CPU oracle timing (reported baseline)
# ---------------------------------------------------------------------------

def oracle_sample(wl_name, W_host, tmap, rows_per_step=256, threads=1, U=None, V=None):
    """A bounded sample of the workload for the CPU oracle: the fp64 hybrid
    product of `rows_per_step` output rows (selection applied on the fly),
    split over `threads` host threads (the oracle's C routine runs without the
    GIL, each thread on its own rows)."""
    import concurrent.futures as cf

    import oracle
    o = oracle.Oracle()
    n, k, b1, b2, frac, batch, std, outliers = WORKLOADS[wl_name]
    Wb = inputs.bits(W_host)
    Ub = inputs.bits(U) if U is not None else None
    Vb = inputs.bits(V) if V is not None else None
    rank = 0 if U is None else U.shape[1]
    X = inputs.bits(inputs.activations(batch, k, inputs.seed_of(wl_name, "X", 0)))
    rng = np.random.default_rng(0)
    sparse_frac = float(np.mean(tmap))
    bytes_per_row = k * (2 * (1 - sparse_frac) + 1.125 * sparse_frac)
    pool = cf.ThreadPoolExecutor(max_workers=threads) if threads > 1 else None

    def step(i):
        rows = np.sort(rng.choice(n, rows_per_step, replace=False)).astype(np.int64)
        if pool is None:
            o.rows(Wb, b1, b2, tmap, X, rows, U=Ub, V=Vb)
            return
        parts = np.array_split(rows, threads)
        list(pool.map(lambda r: o.rows(Wb, b1, b2, tmap, X, r, U=Ub, V=Vb), parts))
    # (each sampled step recomputes V^T x: its V bytes count once per step)
    return step, (bytes_per_row + 2 * rank) * rows_per_step + 2 * batch * k \
        + 4 * batch * rows_per_step + 2 * rank * k


def host_cores():
    """Host threads the CPU legs may use (this process's CPU affinity)."""
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def _cpu_leg(wl, threads, budget_s):
    rows = 256 * threads
    step, nbytes = oracle_sample(wl.name, wl.W_host, wl.tmap, rows_per_step=rows,
                                 threads=threads, U=wl.U_host, V=wl.V_host)
    step(0)
    t0 = time.perf_counter()
    reps = 0
    while time.perf_counter() - t0 < budget_s:
        step(reps)
        reps += 1
    dt = time.perf_counter() - t0
    return round(nbytes * reps / dt / 1e9, 4), rows, reps, dt


def cpu_baseline(wl, budget_s=10.0):
    """The oracle timed on the host cores: every core (the reported value) and
    one thread."""
    cores = host_cores()
    v_all, rows_all, reps_all, dt_all = _cpu_leg(wl, cores, budget_s)
    v_one, rows_one, reps_one, dt_one = _cpu_leg(wl, 1, budget_s)
    return {"value": v_all, "unit": "GB/s", "cores": cores, "kind": "oracle",
            "sample": f"oracle_rows_f64 (fp64) on {rows_all} random output rows of {wl.name} "
                      f"per repetition split over {cores} threads, {reps_all} repetitions in "
                      f"{dt_all:.1f} s",
            "single_thread": {"value": v_one, "unit": "GB/s", "cores": 1,
                              "sample": f"{rows_one} rows per repetition, {reps_one} "
                                        f"repetitions in {dt_one:.1f} s"}}


def run_reference(args, world, rank):
    if rank != 0:
        return 0
    name = args.workload
    W, tmap = make_matrix(name)
    cores = host_cores()
    rows = 256 * cores
    rank, lr_std = LOWRANK.get(name, (0, 0.0))
    U = V = None
    if rank:
        n, k = WORKLOADS[name][:2]
        U, V = inputs.lowrank(n, k, rank, lr_std, inputs.seed_of(name, "LR"))
    step, nbytes = oracle_sample(name, W, tmap, rows_per_step=rows, threads=cores, U=U, V=V)
    for i in range(args.warmup):
        step(i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        step(args.warmup + i)
    dt = time.perf_counter() - t0
    value = nbytes * args.steps / dt / 1e9
    n, k, b1, b2, frac, batch, std, outliers = WORKLOADS[name]
    line = {
        "impl": "reference", "metric": "hybrid 2:4 GEMV achieved HBM GB/s (algorithmic bytes)",
        "value": round(value, 4), "unit": "GB/s", "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(dt * 1e3 / args.steps, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": workload_config(name, float(np.mean(tmap)), rotation(name, tmap),
                                  packed_bytes(name, tmap)),
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": cores,
                         "kind": "oracle",
                         "sample": f"oracle_rows_f64 (fp64) on {rows} random output rows of "
                                   f"{name} per step, split over {cores} threads"},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# --sweep: the other measurements (one JSON line each, not the headline)
# ---------------------------------------------------------------------------



class Calls:
    """A rotation of pre-marshalled calls of a hyb_*_ex entry point (for
    graph_timed).  make_args gives each call's arguments without the launch
    options, which go in front of the trailing (ws, ws_bytes, stream)."""

    def __init__(self, fn, make_args, count, name, with_flags=True):
        self.fn, self.make_args, self.count, self.name = fn, make_args, count, name
        self.with_flags = with_flags  # False: an entry point without launch options
        self.flags = 0
        self.stream = torch.cuda.current_stream()
        self.set_stream(self.stream)

    def set_stream(self, stream):
        sp = ctypes.c_void_p(stream.cuda_stream)
        self.args = []
        for i in range(self.count):
            a = list(self.make_args(i, sp))
            if self.with_flags:
                a.insert(len(a) - 3, self.flags)
            self.args.append(tuple(a))

    def step(self, i):
        rc = self.fn(*self.args[i % self.count])
        if rc != 0:
            raise hyb.HybError(self.name, rc)


def _tensor_roofline(n, k, us):
    """Batch >= 4 products run on the tensor cores (bf16 m16n8k16, batch
    padded to 16 rows, 2:4 tiles expanded to dense): issued tensor FLOPs per
    second against the measured dense bf16 peak.  A small fraction means the
    product is not bound by tensor throughput."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as fh:
            peak, kind = float(json.load(fh)["bf16_tflops"]), "measured"
    except Exception:
        peak, kind = 1590.0, "fallback"
    achieved = 2 * 16 * n * k / (us * 1e-6) / 1e12
    return {"bound": "tensor", "achieved": round(achieved, 2), "peak": peak, "unit": "TFLOP/s",
            "frac": round(achieved / peak, 4), "peak_kind": f"{kind} cuBLAS bf16 (burst)",
            "issued": "2 x 16 x n x k per product (mma.sync m16n8k16 bf16 -> fp32)"}


def sweep(device, steps=200, warmup=10):
    """Hybrid vs dense on the FFN shapes across 2:4-tile fractions and batches,
    the 4096x4096 attention matrix, the 32-layer Llama-3.1-8B chain (224
    matrices, one CUDA graph), the Llama-3.3-70B FFN with a rank-128 (and
    rank-64) low-rank term, and prefill on the tensor cores."""
    peak, peak_kind = measured_peak()
    L = hyb.lib()
    OV = hyb.LAUNCH_OVERLAP_PREV
    l2 = 126 << 20
    sm_mhz = 1965.0

    def rot_count(nbytes):
        return max(2, int(np.ceil(3 * l2 / nbytes)))

    def emit(d):
        print(json.dumps(d), flush=True)

    # ---- FFN shapes x fraction x batch, and the attention matrix ----
    shapes = [("ffn_up", 14336, 4096, [0.0, 0.25, 0.5, 0.75, 1.0]),
              ("ffn_down", 4096, 14336, [0.0, 0.25, 0.5, 0.75, 1.0]),
              ("attn", 4096, 4096, ["bern0.5"])]
    for role, n, k, fracs in shapes:
        W = inputs.weight(n, k, 0.02, inputs.seed_of("ffn_sweep", n, k, "W"),
                          outliers=0.01 if role != "attn" else 0.0)
        Wd = W.to(device)
        nrot_d = rot_count(2 * n * k)
        dense = [Wd] + [Wd.clone() for _ in range(nrot_d - 1)]
        Xs = {b: [inputs.activations(b, k, inputs.seed_of("sweep", n, k, b, i)).to(device)
                  for i in range(max(nrot_d, 16))] for b in (1, 4, 8, 16)}
        Ys = {b: [torch.empty(b, n, dtype=torch.float32, device=device)
                  for _ in range(max(nrot_d, 16))] for b in (1, 4, 8, 16)}
        dense_us, dense_plain_us = {}, {}
        for b in ((1,) if role == "attn" else (1, 4, 8, 16)):
            dws = hyb.new_workspace(hyb.dense_workspace_bytes(n, k, b), device)
            c = Calls(L.hyb_gemv_dense_ex, lambda i, sp, b=b, dws=dws: (
                n, k, b, ctypes.c_void_p(dense[i].data_ptr()), k,
                ctypes.c_void_p(Xs[b][i].data_ptr()), k, ctypes.c_void_p(Ys[b][i].data_ptr()), n,
                hyb.HYB_F32, ctypes.c_void_p(dws.data_ptr()), dws.numel(), sp), nrot_d, "dense")
            dense_us[b] = graph_timed(c, c.step, steps, warmup, flags=OV) / steps * 1e3
            dense_plain_us[b] = graph_timed(c, c.step, steps, warmup) / steps * 1e3
            hyb.check_status(dws)
        del dense
        for f in fracs:
            T = (n // 128) * (k // 128)
            if f == "bern0.5":
                tmap = inputs.attn_map(T)
            else:
                tmap = inputs.tile_map_fraction(T, f, inputs.seed_of("ffn_sweep", n, k, f))
            base = hyb.pack(Wd, tmap, 128, 128)
            nrot = rot_count(base.nbytes())
            mats = [base] + [base.clone() for _ in range(nrot - 1)]
            structs = [m.struct() for m in mats]
            for b in ((1,) if role == "attn" else (1, 4, 8, 16)):
                ws = hyb.new_workspace(hyb.workspace_bytes(base, b), device)
                xs, ys = Xs[b], Ys[b]
                c = Calls(L.hyb_spmm_skinny_ex, lambda i, sp, b=b, ws=ws, xs=xs, ys=ys: (
                    ctypes.byref(structs[i]), b, ctypes.c_void_p(xs[i % len(xs)].data_ptr()), k,
                    ctypes.c_void_p(ys[i % len(ys)].data_ptr()), n, hyb.HYB_F32, None,
                    ctypes.c_void_p(ws.data_ptr()), ws.numel(), sp), nrot, "hybrid")
                us = graph_timed(c, c.step, steps, warmup, flags=OV) / steps * 1e3
                us_plain = graph_timed(c, c.step, steps, warmup) / steps * 1e3
                hyb.check_status(ws)
                nbytes = base.nbytes() + base.num_tiles + 2 * b * k + 4 * b * n
                gbs = nbytes / (us * 1e-6) / 1e9
                kept = base.n_vals  # kept entries = packed values
                line = {"sweep": "ffn" if role != "attn" else "attn", "shape": f"{n}x{k}",
                        "tile": "128x128", "sparse_tile_frac": float(np.mean(tmap)), "batch": b,
                        "us": round(us, 3), "GBps": round(gbs, 1),
                        "frac_of_measured_hbm": round(gbs / peak, 4),
                        "frac_of_8tbs": round(gbs / NOMINAL_HBM_GBS, 4),
                        "dense_us": round(dense_us[b], 3),
                        "speedup_vs_dense": round(dense_us[b] / us, 4),
                        "format_bound_speedup": round((2 * n * k) / base.nbytes(), 4),
                        "plain_launch": {"us": round(us_plain, 3),
                                         "dense_us": round(dense_plain_us[b], 3)}}
                if b >= 4:
                    line["tensor_roofline"] = _tensor_roofline(n, k, us)
                emit(line)
                del ws
            del mats, structs, base
        del Wd, Xs, Ys
        torch.cuda.empty_cache()

    # ---- 32-layer Llama-3.1-8B chain, 224 matrices in one CUDA graph ----
    W_role = {role: inputs.weight(n, k, 0.02, inputs.seed_of("llama8b_chain", role, "W")).to(device)
              for role, n, k in inputs.LLAMA8B_LAYER}
    mats, shapes8 = [], []
    for layer in range(32):
        f = inputs.chain_fraction(layer)
        for role, n, k in inputs.LLAMA8B_LAYER:
            T = (n // 128) * (k // 64)
            tmap = inputs.tile_map_fraction(T, f, inputs.seed_of("llama8b_chain", layer, role, "map"))
            mats.append(hyb.pack(W_role[role], tmap, 128, 64))
            shapes8.append((n, k))
    xs = [inputs.activations(1, k, inputs.seed_of("chain", i)).to(device) for i, (n, k) in enumerate(shapes8)]
    ys = [torch.empty(1, n, dtype=torch.float32, device=device) for n, k in shapes8]
    ws = hyb.new_workspace(max(hyb.workspace_bytes(m, 1) for m in mats), device)
    structs = [m.struct() for m in mats]
    chain = Calls(L.hyb_spmm_skinny_ex, lambda i, sp: (
        ctypes.byref(structs[i]), 1, ctypes.c_void_p(xs[i].data_ptr()), shapes8[i][1],
        ctypes.c_void_p(ys[i].data_ptr()), shapes8[i][0], hyb.HYB_F32, None,
        ctypes.c_void_p(ws.data_ptr()), ws.numel(), sp), len(mats), "chain")
    reps = 4
    ms = graph_timed(chain, chain.step, reps * len(mats), len(mats), flags=OV)
    ms_plain = graph_timed(chain, chain.step, reps * len(mats), len(mats))
    hyb.check_status(ws)
    packed = sum(m.nbytes() + m.num_tiles for m in mats)
    nbytes = packed + sum(2 * k + 4 * n for n, k in shapes8)
    dws = hyb.new_workspace(max(hyb.dense_workspace_bytes(n, k, 1) for n, k in shapes8), device)
    roles8 = [r for _ in range(32) for r, _, _ in inputs.LLAMA8B_LAYER]
    dchain = Calls(L.hyb_gemv_dense_ex, lambda i, sp: (
        shapes8[i][0], shapes8[i][1], 1, ctypes.c_void_p(W_role[roles8[i]].data_ptr()), shapes8[i][1],
        ctypes.c_void_p(xs[i].data_ptr()), shapes8[i][1], ctypes.c_void_p(ys[i].data_ptr()),
        shapes8[i][0], hyb.HYB_F32, ctypes.c_void_p(dws.data_ptr()), dws.numel(), sp),
        len(mats), "dense chain")
    dms = graph_timed(dchain, dchain.step, reps * len(mats), len(mats), flags=OV)
    dms_plain = graph_timed(dchain, dchain.step, reps * len(mats), len(mats))
    hyb.check_status(dws)
    us_chain = ms / reps * 1e3
    emit({"sweep": "llama8b_chain", "matrices": len(mats), "tile": "128x64", "batch": 1,
          "us_per_chain": round(us_chain, 2), "us_per_matrix": round(us_chain / len(mats), 3),
          "GBps": round(nbytes / (us_chain * 1e-6) / 1e9, 1), "packed_GB": round(packed / 1e9, 3),
          "dense_us_per_chain": round(dms / reps * 1e3, 2),
          "speedup_vs_dense": round(dms / ms, 4),
          "plain_launch": {"us_per_chain": round(ms_plain / reps * 1e3, 2),
                           "dense_us_per_chain": round(dms_plain / reps * 1e3, 2)},
          "note": "one weight draw per role; tile maps drawn per layer (f_l ~ U[0.2,1])"})
    del mats, structs, W_role, xs, ys, ws, dws
    torch.cuda.empty_cache()

    # ---- Llama-3.3-70B FFN, all 2:4, rank-128 low-rank term, 8 layers ----
    mats70, sh70 = [], []
    for role, n, k in inputs.LLAMA70B_FFN:
        T = (n // 128) * (k // 128)
        W = inputs.weight(n, k, 0.015, inputs.seed_of("llama70b", role, "W")).to(device)
        base = hyb.pack(W, np.ones(T, np.uint8), 128, 128)
        del W
        for layer in range(8):
            mats70.append(base if layer == 0 else base.clone())
            sh70.append((n, k))
    mats70 = [mats70[(i % 3) * 8 + i // 3] for i in range(24)]
    sh70 = [sh70[(i % 3) * 8 + i // 3] for i in range(24)]
    structs = [m.struct() for m in mats70]
    for rank, batches in ((128, (1, 4, 8, 16)), (64, (1,))):
        lr_by_role = {}
        for role, n, k in inputs.LLAMA70B_FFN:
            U, V = inputs.lowrank(n, k, rank, 0.01, inputs.seed_of("llama70b", role, "LR", rank))
            lr_by_role[(n, k)] = (U.to(device), V.to(device))
        lrs = [lr_by_role[sh] for sh in sh70]
        lrstructs = [hyb.HybLowrank(rank, hyb._bits(U).data_ptr(), rank,
                                    hyb._bits(V).data_ptr(), rank) for U, V in lrs]
        _sweep_70b(L, structs, lrstructs, mats70, sh70, rank, batches, device, peak, emit, sm_mhz)
        del lrs, lrstructs, lr_by_role
    del mats70, structs
    torch.cuda.empty_cache()
    _sweep_prefill(device, emit)
    return 0


def _sweep_prefill(device, emit, steps=20, warmup=3):
    """Prefill on the tensor cores (hyb_spmm_prefill): the FFN shapes at 512,
    1024, 2048 and 4096 tokens, every CTA shape and three 2:4-tile fractions,
    against torch.matmul (cuBLAS
    bf16, the dense weight) on the same inputs.  Tokens x weight bytes exceed
    L2, so back-to-back calls are timed (CUDA events, mean of `steps`)."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as fh:
            peak = float(json.load(fh)["bf16_tflops"])
    except Exception:
        peak = 1590.0
    for n, k in ((4096, 14336), (14336, 4096)):
        W = inputs.weight(n, k, 0.02, inputs.seed_of("prefill_sweep", n, k)).to(device)
        T = (n // 128) * (k // 128)
        for m in (512, 1024, 2048, 4096):
            X = inputs.activations(m, k, inputs.seed_of("prefill_sweep", "X", m, k)).to(device)
            Y = torch.empty(m, n, dtype=torch.float32, device=device)
            stream = torch.cuda.current_stream(device)
            cub_ms = timed(lambda i: torch.matmul(X, W.t()), steps, warmup, stream)
            cub_us = cub_ms / steps * 1e3
            chosen = hyb.prefill_block_shape(n, m)
            for f, blk in ((f, blk) for f in (0.0, 0.5, 1.0) for blk in hyb.PREFILL_SHAPES):
                tmap = inputs.tile_map_fraction(T, f, inputs.seed_of("prefill_sweep", f))
                P = hyb.pack(W, tmap, 128, 128)
                ws = hyb.new_workspace(hyb.lib().hyb_prefill_workspace_bytes(), device)
                ms = timed(lambda i: hyb.spmm_prefill(P, X, Y=Y, ws=ws, block=blk),
                           steps, warmup, stream)
                hyb.check_status(ws)
                us = ms / steps * 1e3
                flops = 2 * m * n * k
                emit({"sweep": "prefill", "shape": f"{n}x{k}", "tokens": m, "tile": "128x128",
                      "block_rows": blk[0], "block_tokens": blk[1],
                      "chosen_by_hyb_spmm_prefill": tuple(blk) == tuple(chosen),
                      "sparse_tile_frac": float(np.mean(tmap)), "us": round(us, 2),
                      "tensor_roofline": {"bound": "tensor",
                                          "achieved": round(flops / (us * 1e-6) / 1e12, 1),
                                          "peak": peak, "unit": "TFLOP/s",
                                          "frac": round(flops / (us * 1e-6) / 1e12 / peak, 4),
                                          "flops": "2 m n k counted dense (2:4 tiles run "
                                                   "the sparse MMA: half the work)"},
                      "cublas_bf16_dense_us": round(cub_us, 2),
                      "speedup_vs_cublas_dense": round(cub_us / us, 4),
                      "kernel": "hybrid_prefill_kernel (tcgen05.mma kind::f16, TMEM accumulator)"})
                del P, ws
        del W
    torch.cuda.empty_cache()


def _sweep_70b(L, structs, lrstructs, mats70, sh70, rank, batches, device, peak, emit, sm_mhz):
    OV = hyb.LAUNCH_OVERLAP_PREV
    for b in batches:
        xs = [inputs.activations(b, k, inputs.seed_of("l70", i, b)).to(device) for i, (n, k) in enumerate(sh70)]
        ys = [torch.empty(b, n, dtype=torch.float32, device=device) for n, k in sh70]
        ws = hyb.new_workspace(max(hyb.workspace_bytes(m, b, rank) for m in mats70), device)
        c = Calls(L.hyb_spmm_skinny_ex, lambda i, sp, b=b, ws=ws, xs=xs, ys=ys: (
            ctypes.byref(structs[i]), b, ctypes.c_void_p(xs[i].data_ptr()), sh70[i][1],
            ctypes.c_void_p(ys[i].data_ptr()), sh70[i][0], hyb.HYB_F32, ctypes.byref(lrstructs[i]),
            ctypes.c_void_p(ws.data_ptr()), ws.numel(), sp), 24, "70b")
        ms = graph_timed(c, c.step, 48, 24, flags=OV)
        us = ms / 2 * 1e3
        us_plain = graph_timed(c, c.step, 48, 24) / 2 * 1e3
        hyb.check_status(ws)
        nbytes = sum(m.nbytes() + m.num_tiles + 2 * b * k + 4 * b * n + 2 * rank * (n + k)
                     for m, (n, k) in zip(mats70, sh70))
        gbs = nbytes / (us * 1e-6) / 1e9
        line = {"sweep": "llama70b_ffn_lowrank", "matrices": 24, "batch": b, "rank": rank,
                "lowrank_path": "fused into the streaming kernel" if b <= 4
                                else "three kernels (V^T x, U t, product)",
                "us_per_8_layers": round(us, 2), "us_per_matrix": round(us / 24, 3),
                "GBps": round(gbs, 1), "frac_of_measured_hbm": round(gbs / peak, 4),
                "plain_launch": {"us_per_8_layers": round(us_plain, 2)}}
        if b >= 4:
            line["tensor_roofline"] = _tensor_roofline(sum(n * k for n, k in sh70), 1, us)
        emit(line)
        del ws, xs, ys


def sweep_nm(device, steps=200, warmup=10):
    """General N:M tiles (hyb_spmm_skinny_nm; 4:8 runs in the streaming
    kernel): the 4096x14336 down projection with 4:8 tiles at three
    fractions, batch 1 and 8, graph replay of rotating copies (larger than
    L2)."""
    peak, _ = measured_peak()
    L = hyb.lib()
    n, k, b1, b2, nk, m = 4096, 14336, 128, 128, 4, 8
    W = inputs.weight(n, k, 0.02, inputs.seed_of("nm_sweep", "W"), outliers=0.01).to(device)
    T = (n // b1) * (k // b2)
    for f in (0.0, 0.5, 1.0):
        tmap = inputs.tile_map_fraction(T, f, inputs.seed_of("nm_sweep", f))
        base = hyb.pack_nm(W, tmap, b1, b2, nk, m)
        nrot = max(2, int(np.ceil(3 * (126 << 20) / base.nbytes())))
        mats = [base] + [base.clone() for _ in range(nrot - 1)]
        structs = [x.struct() for x in mats]
        ws = hyb.new_workspace(max(hyb.workspace_bytes(base, 8), hyb.pack_workspace_bytes()),
                               device)
        for b in (1, 8):
            xs = [inputs.activations(b, k, inputs.seed_of("nm_sweep", b, i)).to(device)
                  for i in range(nrot)]
            ys = [torch.empty(b, n, dtype=torch.float32, device=device) for _ in range(nrot)]
            c = Calls(L.hyb_spmm_skinny_nm, lambda i, sp, b=b, xs=xs, ys=ys: (
                ctypes.byref(structs[i]), nk, m, b, ctypes.c_void_p(xs[i].data_ptr()), k,
                ctypes.c_void_p(ys[i].data_ptr()), n, hyb.HYB_F32,
                ctypes.c_void_p(ws.data_ptr()), ws.numel(), sp), nrot, "nm", with_flags=False)
            us = graph_timed(c, c.step, steps, warmup) / steps * 1e3
            nbytes = base.nbytes() + base.num_tiles + 2 * b * k + 4 * b * n
            gbs = nbytes / (us * 1e-6) / 1e9
            print(json.dumps({"sweep": "nm", "pattern": f"{nk}:{m}", "shape": f"{n}x{k}",
                              "tile": f"{b1}x{b2}", "sparse_tile_frac": float(np.mean(tmap)),
                              "batch": b, "us": round(us, 3), "GBps": round(gbs, 1),
                              "frac_of_measured_hbm": round(gbs / peak, 4),
                              "kernel": "hybrid_tma_kernel (4:8 tiles: mask-byte PRMT "
                                        "selectors, scalar fp32 FMAs)"}), flush=True)
        hyb.check_status(ws)
        del mats, structs, base
        torch.cuda.empty_cache()
    return 0


def packed_bytes(name, tmap):
    """Packed values + masks of the workload's matrix (the format's closed form)."""
    n, k, b1, b2 = WORKLOADS[name][:4]
    s = int(np.sum(tmap == 1))
    return (len(tmap) - s) * 2 * b1 * b2 + s * (b1 * b2 + b1 * b2 // 8)


def rotation(name, tmap, rotate=ROTATE):
    """Packed copies cycled through: a matrix larger than L2 needs only a few
    to stay cold."""
    nb = packed_bytes(name, tmap)
    if nb > (126 << 20):
        rotate = min(rotate, max(2, int(np.ceil(3 * (126 << 20) / nb))))
    return rotate


def workload_config(name, frac_real, rot, nbytes):
    n, k, b1, b2, frac, batch, std, outliers = WORKLOADS[name]
    cfg = {"workload": name, "n": n, "k": k, "tile": f"{b1}x{b2}",
           "sparse_tile_frac": round(frac_real, 4), "batch": batch,
           "weights": f"bf16 N(0,{std})" + (f" with {outliers:.0%} x20 outliers" if outliers else ""),
           "l2": f"inputs larger than L2: {rot} rotating packed copies ({rot * nbytes / 1e9:.2f} GB)",
           "parallelism": "replicas"}
    rank = LOWRANK.get(name, (0, 0.0))[0]
    if rank:
        cfg["lowrank"] = {"rank": rank, "U": f"bf16 [{n}][{rank}]", "V": f"bf16 [{k}][{rank}]"}
    return cfg


# ---------------------------------------------------------------------------

def run_tp(args, device, world, rank):
    """Row-sharded decode: every rank applies its bands of the workload's
    matrix (hyb_shard_bands) to the full X, then one all-gather assembles Y on
    every rank.  Eager steps between CUDA events, max over ranks; value = the
    whole matrix's algorithmic bytes per step / time (strong scaling)."""
    from sparse_weight_b200 import tp
    W, tmap = make_matrix(args.workload)
    n, k, b1, b2, frac, batch, std, outliers = WORKLOADS[args.workload]
    P = hyb.pack(W.to(device), tmap, b1, b2)
    # rotating copies (larger than L2 in all), each sharded the same way
    rot = rotation(args.workload, tmap, args.rotate)
    shards = [tp.RowShard(m, rank, world) for m in [P] + [P.clone() for _ in range(rot - 1)]]
    X = inputs.activations(batch, k, inputs.seed_of(args.workload, "X", 0)).to(device)
    local = shards[0].local
    ws = (hyb.new_workspace(hyb.workspace_bytes(local, batch), device)
          if local is not None else None)
    stream = torch.cuda.current_stream(device)
    ms = timed(lambda i: shards[i % rot].apply(X, ws=ws), args.steps, args.warmup, stream,
               world)
    if ws is not None:
        hyb.check_status(ws)
    nbytes = P.nbytes() + P.num_tiles + 2 * batch * k + 4 * batch * n
    value = nbytes * args.steps / (ms * 1e-3) / 1e9
    if world > 1:
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps({
            "metric": "hybrid 2:4 GEMV achieved HBM GB/s (algorithmic bytes)",
            "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms / args.steps, 6),
            "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": dict(workload_config(args.workload, float(np.mean(tmap)), rot, P.nbytes()),
                           parallelism=f"tp{world} (row shards, NCCL all-gather of Y)",
                           rows_per_rank=[hi - lo for lo, hi in shards[0].rows],
                           launch="eager steps (the shard product, the all-gather and the "
                                  "row reassembly)"),
            "gpu_launches": args.steps}), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", default="hyb", choices=["hyb", "reference"])
    ap.add_argument("--workload", default="ffn_down_4096x14336_f0.5_b1", choices=list(WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--rotate", type=int, default=ROTATE,
                    help="packed copies cycled through (their total must exceed L2)")
    ap.add_argument("--sweep", action="store_true",
                    help="print the fraction / batch sweep, the 224-matrix chain and the 70B "
                         "low-rank lines instead of the headline line")
    ap.add_argument("--nm", action="store_true",
                    help="print the general N:M (4:8) lines instead of the headline line")
    ap.add_argument("--tp", action="store_true",
                    help="row-sharded (tensor-parallel) decode of the workload's matrix over the "
                         "ranks: each rank its bands, one NCCL all-gather of Y per step "
                         "(strong scaling; the default is one replica per rank)")
    ap.add_argument("--prefill-profile", action="store_true",
                    help="prefill case for a profiler: hyb_spmm_prefill on 4096x14336, "
                         "f = 0.5, 2048 tokens (two bands x 240 tokens: 144 CTAs), --steps eager calls")
    ap.add_argument("--dense", action="store_true",
                    help="with --profile: run the row-major dense baseline leg instead")
    ap.add_argument("--profile", action="store_true",
                    help="small case for a profiler: 2 rotating copies (184 MB > L2), "
                         "hybrid product only, no dense / end-to-end / CPU legs")
    args = ap.parse_args()
    if args.profile:
        args.rotate = 2
        args.no_cpu_baseline = True
    world, rank, local = dist_env()
    if args.impl == "reference":
        return run_reference(args, world, rank)

    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=device)
    if args.prefill_profile:
        n, k, m = 4096, 14336, 2048
        W = inputs.weight(n, k, 0.02, inputs.seed_of("prefill_profile", n, k)).to(device)
        T = (n // 128) * (k // 128)
        P = hyb.pack(W, inputs.tile_map_fraction(T, 0.5, inputs.seed_of("prefill_profile", "map")),
                     128, 128)
        X = inputs.activations(m, k, inputs.seed_of("prefill_profile", "X")).to(device)
        Y = torch.empty(m, n, dtype=torch.float32, device=device)
        ws = hyb.new_workspace(hyb.lib().hyb_prefill_workspace_bytes(), device)
        ms = timed(lambda i: hyb.spmm_prefill(P, X, Y=Y, ws=ws), args.steps, args.warmup,
                   torch.cuda.current_stream(device))
        hyb.check_status(ws)
        if rank == 0:
            print(json.dumps({"profile_run": "prefill 4096x14336 f0.5 m2048", "ms": ms,
                              "steps": args.steps}))
        return 0
    if args.tp:
        return run_tp(args, device, world, rank)
    if args.sweep:
        return sweep(device)
    if args.nm:
        return sweep_nm(device)
    wl = Workload(args.workload, device, rotate=args.rotate)
    stream = wl.stream

    if args.profile:
        fn = wl.dense_step if args.dense else wl.step
        ms = timed(fn, args.steps, args.warmup, stream, world)
        wl.check()
        if rank == 0:
            print(json.dumps({"profile_run": args.workload + (" dense" if args.dense else ""),
                              "ms": ms, "steps": args.steps}))
        return 0
    # Every leg runs as a decode engine would run a chain of layers: K calls
    # captured in one CUDA graph, each launched as a programmatic dependent of
    # the one before (HYB_LAUNCH_OVERLAP_PREV); the same legs launched plainly
    # (each product starts after the previous one has drained) are reported
    # beside them.
    ov = hyb.LAUNCH_OVERLAP_PREV
    # after every leg the workspaces' status words are read: a bounded wait
    # that ran out inside a kernel leaves outputs incomplete, and then no
    # number is printed (hyb.check_status raises)
    with ClockSampler(local) as clocks:
        ms = graph_timed(wl, wl.step, args.steps, args.warmup, world, flags=ov)
    wl.check()
    plain_ms = graph_timed(wl, wl.step, args.steps, args.warmup, world)
    wl.check()
    eager_ms = timed(wl.step, args.steps, args.warmup, stream, world)
    wl.check()
    dense_ms = graph_timed(wl, wl.dense_step, args.steps, args.warmup, world, flags=ov)
    wl.check()
    dense_plain_ms = graph_timed(wl, wl.dense_step, args.steps, args.warmup, world)
    wl.check()
    dpk_ms = graph_timed(wl, wl.dense_packed_step, args.steps, args.warmup, world, flags=ov)
    wl.check()
    dpk_plain_ms = graph_timed(wl, wl.dense_packed_step, args.steps, args.warmup, world)
    wl.check()
    e2e_ms, h2d, d2h = e2e_timed(wl, args.steps, args.warmup, stream, world)
    wl.check()

    per_step_ms = ms / args.steps
    value = aggregate_gbs(wl.bytes_step, args.steps, ms, world)
    achieved = wl.bytes_step / (per_step_ms * 1e-3) / 1e9
    peak, peak_kind = measured_peak()
    dense_us = dense_ms / args.steps * 1e3
    kernel = kernel_of(wl.mats[0])
    line = {
        "metric": "hybrid 2:4 GEMV achieved HBM GB/s (algorithmic bytes)",
        "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(per_step_ms, 6), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": workload_config(wl.name, wl.frac_real, len(wl.mats), wl.mats[0].nbytes()),
        "us_per_matrix": round(per_step_ms * 1e3, 3),
        "launch": "CUDA graph of the K steps, each a programmatic dependent of the one "
                  "before (HYB_LAUNCH_OVERLAP_PREV)",
        "plain_launch_us_per_matrix": {
            "graph": round(plain_ms / args.steps * 1e3, 3),
            "eager": round(eager_ms / args.steps * 1e3, 3),
            "dense": round(dense_plain_ms / args.steps * 1e3, 3),
            "dense_packed": round(dpk_plain_ms / args.steps * 1e3, 3)},
        "dense_us_per_matrix": round(dense_us, 3),
        "speedup_vs_dense": round(dense_us / (per_step_ms * 1e3), 4),
        "dense_packed_us_per_matrix": round(dpk_ms / args.steps * 1e3, 3),
        "speedup_vs_dense_packed": round(dpk_ms / ms, 4),
        "format_bound_speedup": round((2 * wl.n * wl.k) / wl.mats[0].nbytes(), 4),
        "frac_of_nominal_8tbs": round(achieved / NOMINAL_HBM_GBS, 4),
        "roofline": {"bound": "hbm", "achieved": round(achieved, 2), "peak": peak,
                     "unit": "GB/s", "frac": round(achieved / peak, 4),
                     "traffic": profiled_traffic(args.workload, kernel),
                     "peak_kind": peak_kind, "kernel": kernel,
                     "bytes_per_launch": wl.bytes_step},
        "e2e": {"value": round(aggregate_gbs(wl.bytes_step, args.steps, e2e_ms, world), 2),
                "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "consumer": ("tensor cores (bf16 m16n8k16, batch padded to 16, fp32 accumulate)"
                     if wl.batch >= 4 else "scalar fp32 FMAs (PRMT-selected x pairs)"),
        "lowrank_path": (None if not wl.rank else "fused into the streaming kernel"
                         if wl.batch <= 4 else "three kernels (V^T x, U t, product)"),
        "gpu_launches": args.steps * (1 if wl.rank == 0 or wl.batch <= 4 else 3),
        "clocks": clocks.summary(),
    }
    if wl.batch >= 4:
        line["tensor_roofline"] = _tensor_roofline(wl.n, wl.k, per_step_ms * 1e3)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl)
    if world > 1:
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
