"""Benchmark of the Avey-B ranker + neural-processor hot path on B200.

One step = one full encoder forward of the long-context workload (batch 1,
N = 98304 tokens, S = 64, d = 768, m = 1536 (768/768), k = 7, four layers
S,D,S,D): avey_rank (normalise, MaxSim, top-k) -> avey_compress -> 4 x
avey_layer_forward, through the C ABI, on inputs already resident in HBM.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

N > 1 is launched with torchrun: every rank encodes its own sequence (weak
scaling, no data-path collective; NCCL carries only the barrier and the
max-over-ranks of the timings).  Rank 0 prints one JSON line.

--impl reference times the fp64 CPU oracle (the only reference this build
has) on the host cores, on a bounded sample of target splits of the same
workload per step.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synthetic as sy  # noqa: E402

WORKLOAD = "long_bf16"
METRIC = "encoder tokens/sec at N=96K d=768 (1 B200); MaxSim % tensor peak, mix % HBM BW"
UNIT = "tokens/s"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
THROTTLE_BAD = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown")
REASONS = ("gpu_idle", "applications_clocks_setting", "sw_power_cap", "hw_slowdown",
           "hw_thermal_slowdown", "hw_power_brake_slowdown", "sw_thermal_slowdown", "sync_boost")


# ------------------------------------------------------------- utilities ---

def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return PEAKS_FALLBACK, "fallback"


def workload_desc(wl) -> str:
    kinds = ",".join("S" if k == sy.STATIC else "D" for k in wl.pattern)
    return (f"{wl.name}: B={wl.B} N={wl.N} S={wl.S} d={wl.d} m={wl.m} ({wl.m_h}/{wl.m_t}) "
            f"k={wl.k} layers={kinds} prenorm={int(wl.prenorm)}")


def maxsim_flops(wl) -> float:
    """Algorithmic MaxSim work per forward: 2 * (n S)^2 * d per sequence."""
    R = wl.n * wl.S
    return 2.0 * wl.B * R * R * wl.d


def maxsim_executed_flops(wl) -> float:
    """MMA work the MaxSim kernel executes: for S >= 32, the 256x256 tiles on or
    right of the diagonal of 256-row blocks (the mirrored scores come from the
    same tile); for S = 16, every 128x256 tile of the (nS) x (nS) product."""
    R = wl.n * wl.S
    kpad = -(-wl.d // 64) * 64
    if wl.S >= 32:
        t = -(-R // 256)
        return 2.0 * wl.B * (t * (t + 1) // 2) * 256 * 256 * kpad
    return 2.0 * wl.B * (-(-R // 128)) * (-(-R // 256)) * 128 * 256 * kpad


def compress_bytes(wl) -> float:
    """Algorithmic HBM bytes of the forward's compression call: the k+1
    gathered bf16 blocks in; out, ahead of at least one layer, only the split
    pair (4 bytes per element), else fp32 as well (8 bytes per element)."""
    return (wl.k + 1) * wl.T * wl.d * 2.0 + wl.T * wl.d * (4.0 if wl.layers else 8.0)


def layer_flops(wl) -> float:
    """Enricher + fuser GEMMs, 2 T d m each, per layer."""
    return wl.layers * 2 * (2.0 * wl.T * wl.d * wl.m)


class ClockSampler:
    """Samples nvidia-smi clocks and throttle reasons while running."""

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.path = os.path.join("/tmp", f"avey_clocks_{os.getpid()}.csv")

    def __enter__(self):
        q = "clocks.sm,clocks.max.sm," + ",".join(f"clocks_event_reasons.{r}" for r in REASONS)
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), f"--query-gpu={q}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=self.fh, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.fh.close()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sm, smax, active = [], [], set()
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 2 + len(REASONS):
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
            except ValueError:
                continue
            for r, v in zip(REASONS, parts[2:]):
                if v.lower().startswith("active"):
                    active.add(r)
        # samples taken while the GPU idled at the edges are not "under load"
        busy = [s for s in sm if smax and s > 0.3 * max(smax)] or sm
        return {"sm_mhz": statistics.median(busy) if busy else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(active - {"gpu_idle"}), "samples": len(sm)}


def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init_dist(backend: str, world: int):
    import datetime
    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return dist


def max_over_ranks(value: float, device=None) -> float:
    """Max of a per-rank float over all ranks (identity when not distributed)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seed(rank: int) -> int:
    """Embedding seed of the sequence a rank encodes (rank 0 = the parity seed)."""
    return rank


def traffic_from_profile(kernel_src: str, workload: str):
    """DRAM bytes per MaxSim launch from the committed ncu summary, or None when
    the kernel source changed since that capture or the capture was taken on
    another workload."""
    path = os.path.join(ROOT, "profiles", "maxsim_long_bf16.md")
    if not os.path.exists(path):
        return None
    txt = open(path).read()
    m1 = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", txt)
    m2 = re.search(r"source_sha256:\s*([0-9a-f]{64})", txt)
    m3 = re.search(r"traffic_workload:\s*(\S+)", txt)
    if not (m1 and m2 and m3) or m3.group(1) != workload:
        return None
    sha = hashlib.sha256(open(kernel_src, "rb").read()).hexdigest()
    return float(m1.group(1)) if sha == m2.group(1) else None


def l2_note(wl) -> str:
    """How the timed steps stand to the 126 MB L2 (inputs larger than L2, or not)."""
    x_mb = wl.B * wl.N * wl.d * 2 / 1e6
    if x_mb > 126:
        return f"inputs larger than L2 (X is {x_mb:.0f} MB bf16, 126 MB L2); no flush"
    return f"X is {x_mb:.0f} MB bf16 and fits the 126 MB L2; no flush (a parity-size workload, not a bench line)"


# ----------------------------------------------------------- CPU baseline ---

def cpu_baseline(wl, E, W, budget_s: float = 15.0, max_splits: int = 64):
    """The fp64 oracle as it stands, on this host's cores, on a bounded sample
    of target splits of the same workload (rank, compression, every layer)."""
    import oracle as orc
    X64 = E.X.astype(np.float64)
    one = sy.sample_targets(wl, 1, seed=100)[:1]
    t0 = time.perf_counter()
    orc.forward(X64, W, wl, sel=one)
    t_one = time.perf_counter() - t0
    count = int(max(1, min(max_splits, budget_s / max(t_one, 1e-3))))
    sel = sy.sample_targets(wl, count, seed=101)[:count]
    t0 = time.perf_counter()
    orc.forward(X64, W, wl, sel=sel)
    el = time.perf_counter() - t0
    toks = sel.shape[0] * wl.S
    # the same oracle on one core, on the one-split sample
    cores = orc.threads()
    orc.set_threads(1)
    try:
        t0 = time.perf_counter()
        orc.forward(X64, W, wl, sel=one)
        el1 = time.perf_counter() - t0
    finally:
        orc.set_threads(cores)
    return {"value": toks / el, "unit": UNIT, "cores": cores, "kind": "oracle",
            "cpu_model": cpu_model(), "value_1core": wl.S / el1,
            "sample": f"{sel.shape[0]} seeded target splits x {wl.S} tokens of {wl.name} "
                      f"(full rank row, compression, {wl.layers} layers each), {el:.1f} s; "
                      f"1 core: 1 split, {el1:.1f} s"}


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


# -------------------------------------------------------------- our arm ---

def run_ours(args):
    import torch
    import attention_free_long_b200 as av
    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = init_dist("nccl", world)
    barrier = (lambda: dist.barrier(device_ids=[local])) if world > 1 else (lambda: None)

    wl = sy.WORKLOADS[args.workload]
    E = sy.gen_embeddings(wl, seed=rank_seed(rank))
    W = sy.gen_weights(wl)
    dt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    x = torch.from_numpy(E.X).to(dev, dt)
    P = torch.from_numpy(W.P).to(dev, dt)
    layers = av.device_layers(W, dt, dev)
    ws = av.make_workspace(wl.B, wl.N, wl.d, wl.S, wl.k, wl.m, dt, wl.prenorm, dev)

    def step(marks=None):
        return av.encoder_forward(x, P, layers, wl.S, wl.k, wl.m_h, wl.eps, wl.prenorm, ws, marks)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    st = av.device_status()
    if st != 0:
        raise RuntimeError(f"device status {av.STATUS.get(st, st)} after warm-up")

    # ---- device-timed region: inputs resident in HBM (X is 151 MB > L2) ----
    n_marks = 2 + wl.layers
    marks = [[torch.cuda.Event(enable_timing=True) for _ in range(n_marks + 1)] for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    l0 = av.kernel_launches()
    with ClockSampler(local) as clk:
        start.record()
        for s in range(args.steps):
            step(marks[s])
        end.record()
        torch.cuda.synchronize()
    launches = av.kernel_launches() - l0
    barrier()
    torch.cuda.synchronize()
    ms = start.elapsed_time(end) / args.steps
    ms_max = max_over_ranks(ms, dev)
    stage = np.array([[marks[s][i].elapsed_time(marks[s][i + 1]) for i in range(n_marks)]
                      for s in range(args.steps)]).mean(axis=0)
    rank_ms, compress_ms, layer_ms = float(stage[0]), float(stage[1]), stage[2:].tolist()
    st = av.device_status()
    if st != 0:
        raise RuntimeError(f"device status {av.STATUS.get(st, st)} after the timed region")

    # ---- dynamic mix alone at the layer's shape (HBM-bound kernel) ----
    T, mt = wl.T, wl.m_t
    zpair = torch.rand((2, T, wl.m), device=dev).to(torch.bfloat16)
    zt = zpair[:, :, wl.m_h:]
    L = av.lib()
    import ctypes
    mix_call = lambda: L.avey_dynamic_mix(ctypes.c_void_p(zt.data_ptr()), wl.m, av.AVEY_BF16X2,
                                          T // wl.S, wl.S, mt, wl.eps,
                                          ctypes.c_void_p(zt.data_ptr()), wl.m, av._stream())
    for _ in range(3):
        assert mix_call() == 0
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    reps = max(10, args.steps)
    e0.record()
    for _ in range(reps):
        mix_call()
    e1.record()
    torch.cuda.synchronize()
    mix_ms = e0.elapsed_time(e1) / reps

    def time_alone(call, reps_):
        for _ in range(3):
            assert call() == 0
        e0.record()
        for _ in range(reps_):
            call()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / reps_

    # ---- static mix alone at the layer's shape (V of the first static layer) ----
    smix_ms = None
    vstat = next((l_.V for l_ in layers if l_.kind == av.AVEY_STATIC), None)
    if vstat is not None:
        smix_ms = time_alone(lambda: L.avey_static_mix(
            ctypes.c_void_p(vstat.data_ptr()), ctypes.c_void_p(zt.data_ptr()), wl.m, av.AVEY_BF16X2,
            T // wl.S, wl.S, mt, ctypes.c_void_p(zt.data_ptr()), wl.m, av._stream()), reps)
    del zpair, zt

    # ---- top-k alone: at the workload's shape, and on a larger sweep where
    # the score matrix (5.4 GB) is far past L2 and launch latency ----
    def topk_time(B_, n_, reps_):
        # timed as a captured CUDA graph of reps_ launches, so that host-side
        # call overhead does not hide the kernel at small sizes
        sc = torch.rand((B_, n_, n_), device=dev)
        ti = torch.empty((B_, n_, wl.k), dtype=torch.int32, device=dev)
        tw = torch.empty((B_, n_, wl.k), dtype=torch.float32, device=dev)
        call = lambda: L.avey_topk(ctypes.c_void_p(sc.data_ptr()), B_, n_, wl.k, 0,
                                   ctypes.c_void_p(ti.data_ptr()), ctypes.c_void_p(tw.data_ptr()),
                                   av._stream())
        for _ in range(3):
            assert call() == 0
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for _ in range(reps_):
                call()
        g.replay()
        torch.cuda.synchronize()
        e0.record()
        g.replay()
        e1.record()
        torch.cuda.synchronize()
        ms_ = e0.elapsed_time(e1) / reps_
        del g, sc, ti, tw
        by = B_ * n_ * n_ * 4.0 + B_ * n_ * wl.k * 8.0
        return ms_, by

    topk_ms, topk_bytes = topk_time(wl.B, wl.n, reps)
    sweep_B, sweep_n = 9, 12288
    sweep_ms, sweep_bytes = topk_time(sweep_B, sweep_n, 5)
    torch.cuda.empty_cache()

    # ---- end to end through the public API with host buffers ----
    # Every step copies its input embeddings host -> device (pinned) and its
    # fp32 output device -> host.  Double-buffered: the copies of steps i+1 and
    # i-1 run on their own streams while step i computes.
    xh = torch.from_numpy(E.X).to(dt).pin_memory()
    outh = [torch.empty((wl.B, wl.n * wl.S, wl.d), dtype=torch.float32).pin_memory() for _ in range(2)]
    xd = [torch.empty_like(x) for _ in range(2)]
    wss = [ws, av.make_workspace(wl.B, wl.N, wl.d, wl.S, wl.k, wl.m, dt, wl.prenorm, dev)]
    comp = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()
    h2d_done, comp_done, d2h_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]
    started = [False, False]

    def e2e_step(i):
        j = i & 1
        with torch.cuda.stream(s_in):
            if started[j]:
                s_in.wait_event(comp_done[j])  # the compute that read xd[j] is done
            xd[j].copy_(xh, non_blocking=True)
            h2d_done[j].record(s_in)
        comp.wait_event(h2d_done[j])
        if started[j]:
            comp.wait_event(d2h_done[j])  # the output in wss[j] has been copied out
        out = av.encoder_forward(xd[j], P, layers, wl.S, wl.k, wl.m_h, wl.eps, wl.prenorm, wss[j])
        comp_done[j].record(comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(comp_done[j])
            outh[j].copy_(out, non_blocking=True)
            d2h_done[j].record(s_out)
        started[j] = True

    for i in range(2):
        e2e_step(i)
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    start.record()
    for st_ in (s_in, s_out):
        st_.wait_event(start)
    for i in range(args.steps):
        e2e_step(i)
    for st_ in (s_in, s_out):
        e_ = ev()
        e_.record(st_)
        comp.wait_event(e_)
    end.record()
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(start.elapsed_time(end) / args.steps, dev)
    st = av.device_status()
    if st != 0:
        raise RuntimeError(f"device status {av.STATUS.get(st, st)} after the e2e region")
    h2d_bytes = int(xh.numel() * xh.element_size())
    d2h_bytes = int(outh[0].numel() * outh[0].element_size())
    del wss, xd, outh, xh
    torch.cuda.empty_cache()

    # ---- the processor without neural compression, same workload ----
    # Every split's (k+1)S-token context goes through the layers as one block
    # (Avey-B paperlayer summary §4.3); the pages report compression as a
    # 4.37x throughput gain over this.
    unc = None
    if not args.no_uncompressed:
        Wu = sy.gen_weights(wl, block=(wl.k + 1) * wl.S)
        layers_u = av.device_layers(Wu, dt, dev)
        ws_u = av.make_workspace(wl.B, wl.N, wl.d, wl.S, wl.k, wl.m, dt, wl.prenorm, dev,
                                 uncompressed=True)

        def step_u(m=None):
            return av.encoder_forward_uncompressed(x, layers_u, wl.S, wl.k, wl.m_h, wl.eps,
                                                   wl.prenorm, ws_u, m)

        for _ in range(2):
            step_u()
        torch.cuda.synchronize()
        st = av.device_status()
        if st != 0:
            raise RuntimeError(f"device status {av.STATUS.get(st, st)} in the uncompressed run")
        reps_u = max(3, min(10, args.steps))
        marks_u = [[torch.cuda.Event(enable_timing=True) for _ in range(n_marks + 1)]
                   for _ in range(reps_u)]
        barrier()
        torch.cuda.synchronize()
        start.record()
        for r_ in range(reps_u):
            step_u(marks_u[r_])
        end.record()
        torch.cuda.synchronize()
        ms_u = max_over_ranks(start.elapsed_time(end) / reps_u, dev)
        st_u = np.array([[marks_u[r_][i].elapsed_time(marks_u[r_][i + 1]) for i in range(n_marks)]
                         for r_ in range(reps_u)]).mean(axis=0)
        unc = {"ms_per_step": ms_u, "value": wl.B * wl.N * world / (ms_u * 1e-3), "unit": UNIT,
               "steps": reps_u, "compression_speedup": ms_u / ms_max, "pages_speedup": 4.37,
               "kernels_ms": {"rank": float(st_u[0]), "context": float(st_u[1]),
                              "layers": st_u[2:].tolist()},
               "note": ("each split's (k+1)S-token context through every layer as one block; "
                        "compression_speedup = uncompressed / compressed ms per step on this GPU; "
                        "pages_speedup is the pages' figure (their hardware and code)")}
        del ws_u, layers_u
        torch.cuda.empty_cache()

    tokens = wl.B * wl.N * world
    peaks, peak_kind = load_peaks()
    sustained = peaks.get("bf16_tflops_sustained", PEAKS_FALLBACK["bf16_tflops_sustained"])
    hbm = peaks.get("hbm_gbs", PEAKS_FALLBACK["hbm_gbs"])
    achieved = maxsim_flops(wl) / (rank_ms * 1e-3) / 1e12
    mix_bytes = 2.0 * T * mt * 4  # read Z_t pair, write c pair
    comp_bytes = compress_bytes(wl)
    kernel_src = os.path.join(ROOT, "attention_free_long_b200", "csrc", "avey_maxsim2.cu")
    result = {
        "metric": METRIC, "value": tokens / (ms_max * 1e-3), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded Gaussian mixture, random N(0,1/fan_in) weights)",
        "config": {"workload": workload_desc(wl), "global_batch": wl.B * world, "seq_len": wl.N,
                   "parallelism": f"dp{world} (one sequence per GPU, no collective)",
                   "l2": l2_note(wl)},
        "roofline": {"bound": "tensor", "kernel": "maxsim (avey_rank call)",
                     "achieved": achieved, "peak": sustained, "unit": "TFLOP/s",
                     "frac": achieved / sustained,
                     "peak_kind": f"{peak_kind} bf16 sustained (kernel inside a long step)",
                     "algorithmic_flop_per_launch": maxsim_flops(wl),
                     "executed_flop_per_launch": maxsim_executed_flops(wl),
                     "executed_achieved": maxsim_executed_flops(wl) / (rank_ms * 1e-3) / 1e12,
                     "executed_frac": maxsim_executed_flops(wl) / (rank_ms * 1e-3) / 1e12 / sustained,
                     "traffic": traffic_from_profile(kernel_src, wl.name),
                     "note": ("duration is the whole avey_rank call (norms + MaxSim + top-k); "
                              "achieved counts the definition's 2(nS)^2 d FLOP, the kernel executes "
                              "about half of them (each tile yields the scores of a split pair in "
                              "both directions), executed_* count the MMA work actually issued")},
        "kernels_ms": {"rank": rank_ms, "compress": compress_ms, "layers": layer_ms},
        "hbm": {"dynamic_mix": {"ms": mix_ms, "gbs": mix_bytes / (mix_ms * 1e-3) / 1e9,
                                "frac": mix_bytes / (mix_ms * 1e-3) / 1e9 / hbm,
                                "peak": hbm, "bytes": mix_bytes},
                "compress": {"ms": compress_ms, "gbs": comp_bytes / (compress_ms * 1e-3) / 1e9,
                             "frac": comp_bytes / (compress_ms * 1e-3) / 1e9 / hbm,
                             "bytes": comp_bytes},
                "static_mix": None if smix_ms is None else {
                    "ms": smix_ms, "gbs": mix_bytes / (smix_ms * 1e-3) / 1e9,
                    "frac": mix_bytes / (smix_ms * 1e-3) / 1e9 / hbm, "bytes": mix_bytes},
                "topk": {"ms": topk_ms, "gbs": topk_bytes / (topk_ms * 1e-3) / 1e9,
                         "frac": topk_bytes / (topk_ms * 1e-3) / 1e9 / hbm, "bytes": topk_bytes,
                         "note": f"{topk_bytes / 1e6:.1f} MB of scores: latency-bound at this size"},
                "topk_sweep": {"B": sweep_B, "n": sweep_n, "k": wl.k, "ms": sweep_ms,
                               "gbs": sweep_bytes / (sweep_ms * 1e-3) / 1e9,
                               "frac": sweep_bytes / (sweep_ms * 1e-3) / 1e9 / hbm,
                               "bytes": sweep_bytes}},
        "e2e": {"value": tokens / (e2e_ms * 1e-3), "unit": UNIT,
                "h2d_bytes_per_step": h2d_bytes,
                "d2h_bytes_per_step": d2h_bytes,
                "note": "copies of neighbouring steps overlap compute (two buffers, copy streams)"},
        "gpu_launches": int(launches),
        "clocks": clk.summary(),
    }
    if unc is not None:
        result["uncompressed"] = unc
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(wl, E, W)
    if world > 1:
        dist.barrier(device_ids=[local])
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(result), flush=True)


# ----------------------------------------------- one sequence, N GPUs ---

def run_sharded(args):
    """--shard sequence: the workload's sequence split across the ranks (strong
    scaling).  Every rank holds the whole input; MaxSim tiles are dealt
    round-robin, the score partials are summed by one NCCL all-reduce, and
    top-k, compression and the layers run on each rank's target splits."""
    import torch
    import attention_free_long_b200 as av
    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = init_dist("nccl", world)
    barrier = (lambda: dist.barrier(device_ids=[local])) if world > 1 else (lambda: None)
    allreduce = (lambda buf: dist.all_reduce(buf)) if world > 1 else (lambda buf: None)

    wl = sy.WORKLOADS[args.workload]
    E = sy.gen_embeddings(wl, seed=rank_seed(0))  # the same sequence on every rank
    W = sy.gen_weights(wl)
    x = torch.from_numpy(E.X).to(dev, torch.bfloat16)
    P = torch.from_numpy(W.P).to(dev, torch.bfloat16)
    layers = av.device_layers(W, torch.bfloat16, dev)
    ws = av.make_shard_workspace(wl.B, wl.N, wl.d, wl.S, wl.k, wl.m, torch.bfloat16, wl.prenorm,
                                 rank, world, dev)

    def step(marks=None):
        return av.encoder_forward_sharded(x, P, layers, wl.S, wl.k, wl.m_h, wl.eps, wl.prenorm,
                                          rank, world, allreduce, ws, marks)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    st = av.device_status()
    if st != 0:
        raise RuntimeError(f"device status {av.STATUS.get(st, st)} after warm-up")
    n_marks = 2 + wl.layers
    marks = [[torch.cuda.Event(enable_timing=True) for _ in range(n_marks + 1)] for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    l0 = av.kernel_launches()
    with ClockSampler(local) as clk:
        start.record()
        for s_ in range(args.steps):
            step(marks[s_])
        end.record()
        torch.cuda.synchronize()
    launches = av.kernel_launches() - l0
    barrier()
    torch.cuda.synchronize()
    ms_max = max_over_ranks(start.elapsed_time(end) / args.steps, dev)
    stage = np.array([[marks[s_][i].elapsed_time(marks[s_][i + 1]) for i in range(n_marks)]
                      for s_ in range(args.steps)]).mean(axis=0)
    st = av.device_status()
    if st != 0:
        raise RuntimeError(f"device status {av.STATUS.get(st, st)} after the timed region")

    # end to end: every step copies the whole input in and this rank's rows out
    xh = torch.from_numpy(E.X).to(torch.bfloat16).pin_memory()
    T_r = wl.B * (ws.t1 - ws.t0) * wl.S
    outh = torch.empty((max(T_r, 1), wl.d), dtype=torch.float32).pin_memory()
    xd = torch.empty_like(x)
    for _ in range(2):
        xd.copy_(xh, non_blocking=True)
        o = step()
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    start.record()
    for _ in range(args.steps):
        xd.copy_(xh, non_blocking=True)
        o = av.encoder_forward_sharded(xd, P, layers, wl.S, wl.k, wl.m_h, wl.eps, wl.prenorm, rank,
                                       world, allreduce, ws)
        outh[:T_r].copy_(o.reshape(T_r, wl.d), non_blocking=True)
    end.record()
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(start.elapsed_time(end) / args.steps, dev)

    tokens = wl.B * wl.N
    peaks, peak_kind = load_peaks()
    sustained = peaks.get("bf16_tflops_sustained", PEAKS_FALLBACK["bf16_tflops_sustained"])
    part_ms = float(stage[0])
    result = {
        "metric": METRIC, "value": tokens / (ms_max * 1e-3), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max,
        "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded Gaussian mixture, random N(0,1/fan_in) weights)",
        "config": {"workload": workload_desc(wl), "global_batch": wl.B, "seq_len": wl.N,
                   "parallelism": (f"sp{world}: one sequence across {world} GPU(s); MaxSim tiles "
                                   "round-robin, score partials summed by one all-reduce of "
                                   f"{wl.B * wl.n * wl.n * 4 / 1e6:.1f} MB, then each rank's "
                                   "target splits"),
                   "l2": l2_note(wl)},
        "roofline": {"bound": "tensor", "kernel": "maxsim part + all-reduce (rank 0)",
                     "achieved": maxsim_executed_flops(wl) / world / (part_ms * 1e-3) / 1e12,
                     "peak": sustained, "unit": "TFLOP/s",
                     "frac": maxsim_executed_flops(wl) / world / (part_ms * 1e-3) / 1e12 / sustained,
                     "peak_kind": f"{peak_kind} bf16 sustained", "traffic": None,
                     "note": "executed MMA work of this rank's 1/N of the triangular tiles over "
                             "the duration of its MaxSim part plus the all-reduce"},
        "kernels_ms": {"maxsim_part_and_allreduce": part_ms, "topk_and_compress": float(stage[1]),
                       "layers": stage[2:].tolist()},
        "e2e": {"value": tokens / (e2e_ms * 1e-3), "unit": UNIT,
                "h2d_bytes_per_step": int(xh.numel() * xh.element_size()),
                "d2h_bytes_per_step": int(T_r * wl.d * 4),
                "note": "every rank copies the whole input in and its own rows out"},
        "gpu_launches": int(launches),
        "clocks": clk.summary(),
    }
    if world > 1:
        dist.barrier(device_ids=[local])
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(result), flush=True)


# -------------------------------------------------------- reference arm ---

def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return
    import oracle as orc
    wl = sy.WORKLOADS[args.workload]
    E, W = sy.gen_embeddings(wl, seed=0), sy.gen_weights(wl)
    X64 = E.X.astype(np.float64)
    t0 = time.perf_counter()
    orc.forward(X64, W, wl, sel=sy.sample_targets(wl, 1, seed=200)[:1])
    t_one = time.perf_counter() - t0
    budget = 150.0
    per_step = int(max(1, min(16, budget / max(1, args.steps + args.warmup) / max(t_one, 1e-3))))
    for i in range(args.warmup):
        orc.forward(X64, W, wl, sel=sy.sample_targets(wl, per_step, seed=300 + i)[:per_step])
    el = 0.0
    for i in range(args.steps):
        sel = sy.sample_targets(wl, per_step, seed=400 + i)[:per_step]
        t0 = time.perf_counter()
        orc.forward(X64, W, wl, sel=sel)
        el += time.perf_counter() - t0
    toks = args.steps * per_step * wl.S
    value = toks / el
    sample = (f"{per_step} seeded target splits x {wl.S} tokens of {wl.name} per step "
              f"(full rank row, compression, {wl.layers} layers each)")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": el / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded Gaussian mixture, random N(0,1/fan_in) weights)",
        "config": {"workload": workload_desc(wl), "global_batch": wl.B, "seq_len": wl.N,
                   "parallelism": "host cores (OpenMP)"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": orc.threads(), "kind": "oracle",
                         "cpu_model": cpu_model(), "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawTextHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=WORKLOAD, choices=sorted(sy.WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-uncompressed", action="store_true",
                    help="skip the measurement of the processor without compression")
    ap.add_argument("--shard", choices=["replicas", "sequence"], default="replicas",
                    help="replicas: one sequence per GPU (weak scaling, no collective); "
                         "sequence: the workload's sequence split across the GPUs (strong scaling)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    _, world, _ = dist_env()
    if world != args.gpus:
        if args.gpus > 1:
            ap.error(f"--gpus {args.gpus} needs torchrun with {args.gpus} ranks (WORLD_SIZE={world})")
    if args.impl == "reference":
        run_reference(args)
    elif args.shard == "sequence":
        run_sharded(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
