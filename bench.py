"""Benchmark of the Avey-B ranker + neural-processor hot path on B200.

One step = one full encoder forward of the long-context workload (batch 1,
N = 98304 tokens, S = 64, d = 768, m = 1536 (768/768), k = 7, four layers
S,D,S,D): avey_rank (normalise, MaxSim, top-k) -> avey_compress -> 4 x
avey_layer_forward, through the C ABI, on inputs already resident in HBM.
The timed region records one CUDA event after every kernel launch (the
library's kernel trace), which gives the per-kernel times and the MaxSim
roofline.  After it, the same line reports the HBM-bound kernels alone, the
processor without compression, and a second workload (default: batch 4,
N = 32768, S = 128, d = 1024, m = 2048, k = 15, 12 layers) with its own
per-kernel breakdown and end-to-end figure.

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
import json
import math
import os
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


def l2_note(wl) -> str:
    """How the timed steps stand to the 126 MB L2 (inputs larger than L2, or not)."""
    x_mb = wl.B * wl.N * wl.d * 2 / 1e6
    if x_mb > 126:
        return f"inputs larger than L2 (X is {x_mb:.0f} MB bf16, 126 MB L2); no flush"
    return f"X is {x_mb:.0f} MB bf16 and fits the 126 MB L2; no flush (a parity-size workload, not a bench line)"


# ----------------------------------------------------------- CPU baseline ---

def cpu_baseline(wl, E, W, budget_s: float = 12.0, max_splits: int = 256):
    """The fp64 oracle as it stands, on this host's cores, on a bounded sample
    of target splits of the same workload (rank, compression, every layer),
    sized to about budget_s of wall time from a batch of 8 splits run the
    same way."""
    import oracle as orc
    X64 = E.X.astype(np.float64)
    one = sy.sample_targets(wl, 1, seed=100)[:1]
    cal = sy.sample_targets(wl, 8, seed=99)[:8]
    t0 = time.perf_counter()
    orc.forward(X64, W, wl, sel=cal)
    per = (time.perf_counter() - t0) / cal.shape[0]
    count = int(max(1, min(max_splits, budget_s / max(per, 1e-3))))
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

def _time_alone(call, reps, e0, e1):
    """Mean device ms of ``call`` (returns an avey status) over ``reps`` calls."""
    import torch
    for _ in range(3):
        assert call() == 0
    torch.cuda.synchronize()
    e0.record()
    for _ in range(reps):
        call()
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / reps


def mixes_alone(av, wl, layers, dev, reps):
    """The split-size static and dynamic mixes timed alone at the layer's shape
    (in place on Z's tail columns, as inside a layer).  Returns
    (static_ms or None, dynamic_ms, bytes): the bytes are the algorithmic read
    of the Z_t pair plus the write of the c pair."""
    import ctypes
    import torch
    T, mt = wl.T, wl.m_t
    zpair = torch.rand((2, T, wl.m), device=dev).to(torch.bfloat16)
    zt = zpair[:, :, wl.m_h:]
    L = av.lib()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    zp = ctypes.c_void_p(zt.data_ptr())
    dyn = _time_alone(lambda: L.avey_dynamic_mix(zp, wl.m, av.AVEY_BF16X2, T // wl.S, wl.S, mt,
                                                 wl.eps, zp, wl.m, av._stream()), reps, e0, e1)
    stat = None
    vstat = next((l_.V for l_ in layers if l_.kind == av.AVEY_STATIC), None)
    if vstat is not None:
        vp = ctypes.c_void_p(vstat.data_ptr())
        stat = _time_alone(lambda: L.avey_static_mix(vp, zp, wl.m, av.AVEY_BF16X2, T // wl.S, wl.S,
                                                     mt, zp, wl.m, av._stream()), reps, e0, e1)
    del zpair, zt
    torch.cuda.empty_cache()
    return stat, dyn, 2.0 * T * mt * 4


def compress_alone(av, wl, E, W, dev, reps):
    """avey_compress timed alone at the workload's shape, writing the split
    pair only (as inside the forward), on the GPU ranker's selection."""
    import ctypes
    import torch
    dt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    x = torch.from_numpy(E.X).to(dev, dt)
    P = torch.from_numpy(W.P).to(dev, dt)
    idx, w = av.avey_rank(x, wl.S, wl.k)
    pair = torch.empty((2, wl.B * wl.n * wl.S, wl.d), dtype=torch.bfloat16, device=dev)
    L = av.lib()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ms = _time_alone(lambda: L.avey_compress(av._ptr(x), av._dt(x), wl.B, wl.N, wl.d, wl.S, wl.k,
                                             av._ptr(idx), av._ptr(w), av._ptr(P), None,
                                             av._ptr(pair), av._stream()), reps, e0, e1)
    del x, P, idx, w, pair
    torch.cuda.empty_cache()
    return ms


def forward_leg(av, wl, dev, args, rank, world, local, barrier, e2e=True, sample_clocks=True):
    """One workload through encoder_forward: warm-up, the device-timed region
    (inputs resident in HBM; per-call events and a kernel trace recorded
    live), then the same forward end to end with host buffers."""
    import torch
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
        raise RuntimeError(f"device status {av.STATUS.get(st, st)} after warm-up ({wl.name})")

    # ---- device-timed region ----
    n_marks = 2 + wl.layers
    marks = [[torch.cuda.Event(enable_timing=True) for _ in range(n_marks + 1)]
             for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    per_step = 4 + 4 * wl.layers  # upper bound of launches per forward (prenorm adds one per layer)
    trace = av.KernelTrace(capacity=args.steps * per_step + 8)
    barrier()
    torch.cuda.synchronize()
    l0 = av.kernel_launches()
    clk = ClockSampler(local) if sample_clocks else None
    if clk is not None:
        clk.__enter__()
    try:
        with trace:
            start.record()
            for s_ in range(args.steps):
                step(marks[s_])
            end.record()
        torch.cuda.synchronize()
    finally:
        if clk is not None:
            clk.__exit__(None, None, None)
    launches = av.kernel_launches() - l0
    barrier()
    torch.cuda.synchronize()
    ms = start.elapsed_time(end) / args.steps
    ms_max = max_over_ranks(ms, dev)
    stage = np.array([[marks[s_][i].elapsed_time(marks[s_][i + 1]) for i in range(n_marks)]
                      for s_ in range(args.steps)]).mean(axis=0)
    st = av.device_status()
    if st != 0:
        raise RuntimeError(f"device status {av.STATUS.get(st, st)} after the timed region ({wl.name})")
    # the first interval runs from the trace's opening event, recorded before
    # the host had enqueued the first kernel, so it holds the host's lead-in:
    # it counts as a launch but is left out of the per-launch time
    kern, count, lead = {}, {}, {}
    for i, (name, kms) in enumerate(trace.kernels()):
        count[name] = count.get(name, 0) + 1
        kern.setdefault(name, [])
        if i > 0:
            kern[name].append(kms)
        else:
            lead[name] = kms
    kernels = {}
    for name, v in kern.items():
        per = float(np.mean(v)) if v else float(lead[name])  # one launch only: keep it
        kernels[name] = {"ms_per_launch": per, "launches_per_step": count[name] / args.steps,
                         "ms_per_step": per * count[name] / args.steps}
    out = {"wl": wl, "ms": ms_max, "value": wl.B * wl.N * world / (ms_max * 1e-3),
           "kernels_ms": {"rank": float(stage[0]), "compress": float(stage[1]),
                          "layers": stage[2:].tolist()},
           "kernels": kernels, "launches": int(launches),
           "clocks": clk.summary() if clk is not None else None,
           "layers": layers, "E": E, "W": W}
    if not e2e:
        del ws, x, P
        torch.cuda.empty_cache()
        return out

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
        o = av.encoder_forward(xd[j], P, layers, wl.S, wl.k, wl.m_h, wl.eps, wl.prenorm, wss[j])
        comp_done[j].record(comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(comp_done[j])
            outh[j].copy_(o, non_blocking=True)
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
        raise RuntimeError(f"device status {av.STATUS.get(st, st)} after the e2e region ({wl.name})")
    out["e2e"] = {"value": wl.B * wl.N * world / (e2e_ms * 1e-3), "unit": UNIT,
                  "h2d_bytes_per_step": int(xh.numel() * xh.element_size()),
                  "d2h_bytes_per_step": int(outh[0].numel() * outh[0].element_size()),
                  "note": "copies of neighbouring steps overlap compute (two buffers, copy streams)"}
    del wss, xd, outh, xh, ws, x, P
    torch.cuda.empty_cache()
    return out


def maxsim_roofline(wl, leg, peaks, peak_kind):
    """MaxSim's tensor roofline from its launches inside the timed region."""
    name = "maxsim_pair" if wl.S >= 32 else "maxsim_tc"
    k = leg["kernels"].get(name)
    if k is None:
        return None
    kms = k["ms_per_launch"]
    burst = peaks.get("bf16_tflops", PEAKS_FALLBACK["bf16_tflops"])
    sustained = peaks.get("bf16_tflops_sustained", PEAKS_FALLBACK["bf16_tflops_sustained"])
    executed = maxsim_executed_flops(wl)
    achieved = executed / (kms * 1e-3) / 1e12
    return {"bound": "tensor", "kernel": name, "achieved": achieved, "peak": burst,
            "unit": "TFLOP/s", "frac": achieved / burst,
            "peak_kind": f"{peak_kind} bf16 burst (cuBLAS)",
            "frac_of_sustained": achieved / sustained, "peak_sustained": sustained,
            "kernel_ms": kms, "executed_flop_per_launch": executed,
            "definition_flop_per_launch": maxsim_flops(wl),
            "traffic": None,
            "note": ("achieved = the MMA work the kernel issues (the 256x256 tiles on or right of the "
                     "diagonal; each yields the scores of a split pair in both directions) / its "
                     "mean launch time inside the timed region (kernel trace events on the launch "
                     "stream); definition_flop_per_launch counts 2 (nS)^2 d, both directions in "
                     "full; traffic is null: DRAM bytes come from an ncu capture, not this run")}


def _hbm(ms, nbytes, peak):
    if ms is None:
        return None
    gbs = nbytes / (ms * 1e-3) / 1e9
    return {"ms": ms, "gbs": gbs, "frac": gbs / peak, "bytes": nbytes}


def run_ours(args):
    import torch
    import attention_free_long_b200 as av
    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = init_dist("nccl", world)
    barrier = (lambda: dist.barrier(device_ids=[local])) if world > 1 else (lambda: None)
    peaks, peak_kind = load_peaks()
    hbm = peaks.get("hbm_gbs", PEAKS_FALLBACK["hbm_gbs"])

    wl = sy.WORKLOADS[args.workload]
    leg = forward_leg(av, wl, dev, args, rank, world, local, barrier)
    layers, E, W = leg["layers"], leg["E"], leg["W"]
    reps = max(10, args.steps)

    # ---- HBM-bound kernels: the mixes and compression alone at the
    # workload's shape and inside the forward (kernel trace) ----
    smix_ms, mix_ms, mix_bytes = mixes_alone(av, wl, layers, dev, reps)
    kin = leg["kernels"]
    dyn_in = kin.get("dynamic_mix_tc", {}).get("ms_per_launch")
    stat_in = kin.get("static_mix_tc", {}).get("ms_per_launch")
    comp_in = (kin.get("compress_tc") or kin.get("compress_bf16") or {}).get("ms_per_launch")
    comp_ms = compress_alone(av, wl, E, W, dev, reps) if wl.dtype == "bf16" else None
    comp_bytes = compress_bytes(wl)

    # ---- top-k alone: at the workload's shape, and on a larger sweep where
    # the score matrix (5.4 GB) is far past L2 and launch latency ----
    import ctypes
    L = av.lib()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

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
    norms_ms = kin.get("inv_norms", {}).get("ms_per_launch")
    norms_bytes = wl.B * wl.N * wl.d * 2.0 + wl.B * wl.n * wl.S * 4.0

    # ---- the processor without neural compression, same workload ----
    # Every split's (k+1)S-token context goes through the layers as one block
    # (Avey-B paperlayer summary §4.3); the pages report compression as a
    # 4.37x throughput gain over this.
    unc = None
    n_marks = 2 + wl.layers
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if not args.no_uncompressed:
        dt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
        x = torch.from_numpy(E.X).to(dev, dt)
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
               "steps": reps_u, "compression_speedup": ms_u / leg["ms"], "pages_speedup": 4.37,
               "kernels_ms": {"rank": float(st_u[0]), "context": float(st_u[1]),
                              "layers": st_u[2:].tolist()},
               "note": ("each split's (k+1)S-token context through every layer as one block; "
                        "compression_speedup = uncompressed / compressed ms per step on this GPU; "
                        "pages_speedup is the pages' figure (their hardware and code)")}
        del ws_u, layers_u, x
        torch.cuda.empty_cache()

    # ---- the large workload (batch 4, N = 32768, S = 128, d = 1024,
    # m = 2048, k = 15, 12 layers): per-kernel breakdown and end to end ----
    large = None
    if args.large_workload != "none":
        wl5 = sy.WORKLOADS[args.large_workload]
        leg5 = forward_leg(av, wl5, dev, args, rank, world, local, barrier)
        s5, d5, b5 = mixes_alone(av, wl5, leg5["layers"], dev, reps)
        k5 = leg5["kernels"]
        ksum = sum(v["ms_per_step"] for v in k5.values())
        large = {"config": {"workload": workload_desc(wl5), "global_batch": wl5.B * world,
                            "seq_len": wl5.N, "l2": l2_note(wl5)},
                 "value": leg5["value"], "unit": UNIT, "ms_per_step": leg5["ms"],
                 "steps": args.steps, "kernels_ms": leg5["kernels_ms"], "kernels": k5,
                 "kernel_sum_ms": ksum, "e2e": leg5["e2e"],
                 "roofline": maxsim_roofline(wl5, leg5, peaks, peak_kind),
                 "layers_executed_tflops": layer_flops(wl5) * 2 / (sum(leg5["kernels_ms"]["layers"]) * 1e-3) / 1e12,
                 "mixes_alone": {"static": _hbm(s5, b5, hbm), "dynamic": _hbm(d5, b5, hbm)},
                 "clocks": leg5["clocks"], "gpu_launches": leg5["launches"]}
        del leg5
        torch.cuda.empty_cache()

    tokens = wl.B * wl.N * world
    ksum = sum(v["ms_per_step"] for v in kin.values())
    result = {
        "metric": METRIC, "value": leg["value"], "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": leg["ms"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded Gaussian mixture, random N(0,1/fan_in) weights)",
        "config": {"workload": workload_desc(wl), "global_batch": wl.B * world, "seq_len": wl.N,
                   "parallelism": f"dp{world} (one sequence per GPU, no collective)",
                   "l2": l2_note(wl)},
        "roofline": maxsim_roofline(wl, leg, peaks, peak_kind),
        "kernels_ms": leg["kernels_ms"], "kernels": kin, "kernel_sum_ms": ksum,
        "hbm": {"peak": hbm, "peak_kind": f"{peak_kind} HBM copy bandwidth",
                "dynamic_mix": dict(_hbm(mix_ms, mix_bytes, hbm), in_forward=_hbm(dyn_in, mix_bytes, hbm)),
                "static_mix": None if smix_ms is None else dict(
                    _hbm(smix_ms, mix_bytes, hbm), in_forward=_hbm(stat_in, mix_bytes, hbm)),
                "compress": dict(_hbm(comp_ms, comp_bytes, hbm) or {},
                                 in_forward=_hbm(comp_in, comp_bytes, hbm)),
                "inv_norms": _hbm(norms_ms, norms_bytes, hbm),
                "topk": dict(_hbm(topk_ms, topk_bytes, hbm),
                             note=f"{topk_bytes / 1e6:.1f} MB of scores: latency-bound at this size"),
                "topk_sweep": dict(_hbm(sweep_ms, sweep_bytes, hbm), B=sweep_B, n=sweep_n, k=wl.k),
                "note": ("mixes and compression: alone at the workload's shape, and in_forward from "
                         "the kernel trace (inside the forward they run at the clock the power cap "
                         "leaves after MaxSim or a layer GEMM); inverse norms from the kernel "
                         "trace; top-k alone")},
        "e2e": leg["e2e"],
        "gpu_launches": leg["launches"],
        "clocks": leg["clocks"],
    }
    if unc is not None:
        result["uncompressed"] = unc
    if large is not None:
        result["large"] = large
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
    ap.add_argument("--large-workload", default="large_bf16",
                    choices=["none"] + sorted(sy.WORKLOADS),
                    help="second workload measured after the first (per-kernel breakdown and "
                         "end to end); none skips it")
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
