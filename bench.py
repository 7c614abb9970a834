#!/usr/bin/env python
"""Benchmark of the MoE expert layer: fwd+bwd tokens/s and grouped-GEMM
TFLOP/s on B200, one process per GPU.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

N > 1 runs under torchrun as independent replicas (the layer keeps all
experts on one GPU and has no exchange step): every rank runs the same
workload on its own tokens, the timing is the max over ranks and `value`
is the tokens of all ranks over that time (weak scaling).

Timed region: W untimed warm-up steps (eager), then exactly K steps, each
one replay of a CUDA graph captured from the step's library calls and
bracketed by CUDA events on the stream the library launches on; between
steps (and outside the events) a 512 MiB buffer is written to flush the
126 MB L2, then a second 512 MiB buffer is read, so that the flush's own
dirty lines are written back before the step starts.
Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE layer fwd+bwd tokens/s and grouped-GEMM TFLOP/s (% of B200 peak), 1 GPU"
UNIT = "tokens/s"
DEFAULT_WORKLOAD = "e8"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--no-ratio", action="store_true", help="skip the E=128 vs E=8 measurement")
    ap.add_argument("--no-mxfp8", action="store_true", help="skip the MXFP8 workload measurement")
    ap.add_argument("--no-skew", action="store_true",
                    help="skip the skewed-routing workload measurement")
    ap.add_argument("--api-trace", metavar="JSON",
                    help="instead of timing: trace --steps eager steps of the workload with the "
                         "CUDA profiler (CUPTI, through torch.profiler) and write the per-step "
                         "counts of kernels, copies and synchronising API calls to JSON")
    ap.add_argument("--no-variants", action="store_true",
                    help="skip the layer variants (load-balancing loss, ...) on the main workload")
    ap.add_argument("--dtype", choices=["bf16", "mxfp8"], default="bf16",
                    help="expert GEMM operands of the main workload")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="target CPU time of the oracle sample")
    return ap.parse_args()


def dist_env():
    from mixture_experts_layer_39_b200.replicas import world
    return world()


# dense datasheet figures (B200): bf16 2.25 PFLOP/s, fp8 twice that
DATASHEET_BF16_TFLOPS = 2250.0
FP8_OVER_BF16 = 2.0


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            d = json.load(fh)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------------ clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.dev = device_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(self.dev), "-lms", "100"], stdout=self.fh, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.fh.close()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), float(parts[3]), parts[5:9]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return None
        loaded = [r for r in rows if r[2] > 250.0] or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in loaded for i, v in enumerate(r[3])
                          if v.lower().startswith("active")})
        return {"sm_mhz": statistics.median(r[0] for r in loaded),
                "sm_max_mhz": max(r[1] for r in loaded), "reasons": reasons,
                "samples": len(loaded), "power_w_max": max(r[2] for r in loaded)}


# ------------------------------------------------------------------ oracle timing
def _oracle_step(x, w_r, w_gu, w_d, dy, k, bias, route):
    from oracle import moe_ref as R
    fwd = R.layer_fwd(x, w_r, w_gu, w_d, k, bias=bias, route=route)
    R.layer_bwd(fwd, dy, x, w_r, w_gu, w_d)


def _oracle_inputs(cfg, T_s):
    import torch
    from mixture_experts_layer_39_b200.inputs import make_inputs
    inp = make_inputs(cfg, seed=0, device="cuda" if torch.cuda.is_available() else "cpu")
    f64 = lambda t: t.detach().to("cpu").double().numpy()
    return (f64(inp["x"][:T_s]), f64(inp["w_r"]), f64(inp["w_gu"]), f64(inp["w_d"]),
            f64(inp["dy"][:T_s]), None if inp["bias"] is None else f64(inp["bias"]),
            None if inp["route"] is None else inp["route"][:T_s].cpu().numpy())


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return max(n)
    except Exception:
        pass
    return os.cpu_count() or 1


def _oracle_seconds(cfg, T_s):
    args = _oracle_inputs(cfg, T_s)
    t0 = time.perf_counter()
    _oracle_step(*args[:4], args[4], cfg.k, args[5], args[6])
    return max(time.perf_counter() - t0, 1e-3)


def size_oracle_sample(cfg, seconds):
    """Tokens per oracle step so that one step costs about `seconds`.  A step
    has a fixed part (every expert's full weights are rounded and their
    gradients formed whatever the token count) and a part linear in the
    tokens, so two probe sizes fit t = a + b T and the sample solves it."""
    T1 = min(128, cfg.T)
    T2 = min(4 * T1, cfg.T)
    _oracle_seconds(cfg, T1)  # first touch of the weights and BLAS threads, not timed
    t1 = _oracle_seconds(cfg, T1)
    if T2 == T1:
        return T1
    t2 = _oracle_seconds(cfg, T2)
    b = (t2 - t1) / (T2 - T1)
    if b <= 0:
        b = t2 / T2
    a = max(t1 - b * T1, 0.0)
    T_fit = int(max(seconds - a, 0.0) / b)
    return max(T1, min(cfg.T, T_fit // 64 * 64 if T_fit >= 64 else T_fit))


def cpu_baseline(cfg, seconds):
    T_s = size_oracle_sample(cfg, seconds)
    args = _oracle_inputs(cfg, T_s)
    t0 = time.perf_counter()
    _oracle_step(*args[:4], args[4], cfg.k, args[5], args[6])
    dt = time.perf_counter() - t0
    return {"value": T_s / dt, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
            "sample": (f"oracle fwd+bwd (NumPy float64, bf16 storage rounding) on the first "
                       f"{T_s} of {cfg.T} tokens of workload {cfg.name} with all {cfg.E} experts' "
                       f"full weights; one pass, {dt:.1f} s"),
            "seconds": dt, "tokens": T_s}


# ------------------------------------------------------------------ our arm
def gini(counts):
    """Gini coefficient of the per-expert routed-row counts: 0 when every
    expert gets the same load, (E - 1) / E when one expert gets all of it.
    With the counts sorted ascending, c_1 <= ... <= c_E,
    G = 2 * sum_i i * c_i / (E * sum_i c_i) - (E + 1) / E."""
    c = np.sort(np.asarray(counts, dtype=np.float64).ravel())
    E, total = c.size, c.sum()
    if E == 0 or total <= 0:
        return 0.0
    i = np.arange(1, E + 1, dtype=np.float64)
    return float(2.0 * np.dot(i, c) / (E * total) - (E + 1.0) / E)


def load_report(counts):
    """Per-expert load of one step's routing, read from the device counts
    after the timed region: the real load, not a balance score."""
    c = np.asarray(counts, dtype=np.int64).ravel()
    return {"max_over_mean_load": float(c.max() / c.mean()), "max_count": int(c.max()),
            "min_count": int(c.min()), "mean_count": float(c.mean()),
            "zero_experts": int((c == 0).sum()), "gini": gini(c)}


def gemm_traffic(cfg_name):
    """DRAM bytes per step of the grouped-GEMM launches from the committed ncu
    summary, only while the kernel sources are the ones it was taken on."""
    p = os.path.join(ROOT, "profiles", "grouped_gemm_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as fh:
        d = json.load(fh)
    h = hashlib.sha256()
    for rel in ("mixture_experts_layer_39_b200/csrc/tc_gemm.cuh",
                "mixture_experts_layer_39_b200/csrc/gemm.cu"):
        with open(os.path.join(ROOT, rel), "rb") as fh:
            h.update(fh.read())
    if d.get("source_sha256") != h.hexdigest() or d.get("workload") != cfg_name:
        return None
    return d.get("dram_bytes_per_step")


class L2Flush:
    """Empties the 126 MB L2 of the layer's data between timed steps: writes
    a 512 MiB buffer, then reads another one, so that the step starts with
    no line of its own data cached and no dirty line of the flush left to
    write back (that write-back is the flush's cost, not the step's)."""

    def __init__(self, dev):
        import torch
        self.w = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
        self.r = torch.zeros(512 << 20, dtype=torch.uint8, device=dev)

    def __call__(self, value):
        self.w.fill_(value)
        self.r.max()


def measure(L, g, steps, warmup, flush, dev, with_gemm_events=True):
    """Times `steps` steps of the layer.  After `warmup` eager steps the step
    (every library call of MoELayer.forward/.backward, in order) is captured
    once as a CUDA graph and replayed: the library launches on the caller's
    stream and allocates nothing, so the captured graph holds exactly the
    step's kernels.  Events around the expert GEMMs are captured as external
    event nodes; the step events are recorded on the stream around each
    replay, and the L2 flush runs between steps outside them."""
    import torch

    def one_step(ev=None):
        stream = torch.cuda.current_stream()
        L.router(g["x"], g["w_r"], g["bias"], g["route"])
        L.permute(g["x"])
        if L.aux_alpha > 0:
            L.load_stats()
            L.balance_loss()
        if ev: ev[0].record(stream)
        if L.fuse_combine:  # the shared expert first; the combine runs in the down GEMM
            if L.shared_ff > 0:
                L.shared_fwd(g["x"], g["w_gu_s"], g["w_d_s"])
            L.experts_fwd(g["w_gu"], g["w_d"])
        else:
            L.experts_fwd(g["w_gu"], g["w_d"])
            if L.shared_ff > 0:
                L.shared_fwd(g["x"], g["w_gu_s"], g["w_d_s"])
        if ev: ev[1].record(stream)
        if not L.fuse_combine:
            L.combine()
        L.combine_bwd(g["dy"])
        L.router_bwd(g["x"], g["w_r"])
        if ev: ev[2].record(stream)
        L.experts_bwd(g["w_gu"], g["w_d"])
        if L.shared_ff > 0:
            L.shared_bwd(g["dy"], g["x"], g["w_gu_s"], g["w_d_s"])
        if ev: ev[3].record(stream)
        L.permute_bwd(g["w_r"])

    for _ in range(warmup):
        flush(1)
        one_step()
    torch.cuda.synchronize(dev)
    gev = ([torch.cuda.Event(enable_timing=True, external=True) for _ in range(4)]
           if with_gemm_events else None)
    graph = torch.cuda.CUDAGraph()
    n0 = L.handle.launch_count()
    with torch.cuda.graph(graph):
        one_step(gev)
    per_step = L.handle.launch_count() - n0  # kernels in the graph
    stream = torch.cuda.current_stream()
    for _ in range(2):  # first replays upload the graph
        flush(1)
        graph.replay()
    torch.cuda.synchronize(dev)
    mk = lambda: torch.cuda.Event(enable_timing=True)
    step_ev = [(mk(), mk()) for _ in range(steps)]
    gemm_ms = [] if gev else None
    for i in range(steps):
        flush(i & 0xFF)
        step_ev[i][0].record(stream)
        graph.replay()
        step_ev[i][1].record(stream)
        if gev:  # the graph's events are re-recorded by the next replay
            step_ev[i][1].synchronize()
            gemm_ms.append(gev[0].elapsed_time(gev[1]) + gev[2].elapsed_time(gev[3]))
    torch.cuda.synchronize(dev)
    step_ms = [a.elapsed_time(b) for a, b in step_ev]
    del graph
    return step_ms, gemm_ms, per_step * steps


def measure_memory_bound(L, g, flush, reps=10):
    """HBM-bound calls of the step, each timed alone with CUDA events after an
    L2 flush (median of `reps`), against its algorithmic bytes: useful rows
    only, no pad rows, metadata and router outputs counted where they are
    written.  The layer holds a completed step, so every call sees the inputs
    it has in the step."""
    import torch
    T, d, k, E = L.T, L.d, L.k, L.E
    rows = T * k * d * 2  # the T*k routed bf16 rows
    tok = T * d * 2       # one bf16 row per token
    fused = L.fuse_router_dx
    calls = {
        "router": (lambda: L.router(g["x"], g["w_r"], g["bias"], g["route"]),
                   tok + T * E * 4 + T * k * 8, "read x; write probs, ids, gate weights"),
        "permute": (lambda: L.permute(g["x"]), tok + rows,
                    "routing metadata + read x, write the T*k routed rows"),
        "combine": (lambda: L.combine(), rows + tok, "read the routed rows, write y"),
        "combine_bwd": (lambda: L.combine_bwd(g["dy"]), tok + 2 * rows,
                        "read dY and the routed rows of O, write dO"),
        "permute_bwd": (lambda: L.permute_bwd(g["w_r"]),
                        rows + tok + (0 if fused else T * d * 4),
                        "read dX_perm" + ("" if fused else " and dX_router (fp32)") + ", write dX"
                        + (" (router input gradient formed in the same pass)" if fused else "")),
    }
    stream = torch.cuda.current_stream()
    out = {}
    for name, (fn, nbytes, what) in calls.items():
        fn()  # warm
        ts = []
        for _ in range(reps):
            flush(3)
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            b.synchronize()
            ts.append(a.elapsed_time(b))
        ts.sort()
        ms = ts[len(ts) // 2]
        out[name] = {"ms": ms, "bytes": nbytes, "gb_s": nbytes / (ms / 1e3) / 1e9, "what": what}
    return out


def measure_e2e(L, g, steps, warmup, dev):
    """The same step through the public API with host buffers: every step's
    inputs (x, dY and, in random-routing mode, the expert ids) are copied in
    from pinned host memory and its results (y, dX) copied back, inside the
    timed region.  HostStepper overlaps step i's kernels with the copy-in of
    step i+1 and the copy-out of step i's results."""
    import torch
    from mixture_experts_layer_39_b200.pipeline import HostStepper

    stepper = HostStepper(L, with_route=g["route"] is not None)
    pin = lambda t: t.detach().cpu().pin_memory()
    xs = [pin(g["x"]), pin(g["x"].flip(0))]
    dys = [pin(g["dy"]), pin(g["dy"].flip(0))]
    routes = [pin(g["route"]), pin(g["route"].flip(0))] if g["route"] is not None else [None, None]
    ys = [torch.empty(L.y.shape, dtype=L.y.dtype, pin_memory=True) for _ in range(2)]
    dxs = [torch.empty(L.dx.shape, dtype=L.dx.dtype, pin_memory=True) for _ in range(2)]

    def plan(n):
        out = []
        for i in range(n):
            st = {"x": xs[i & 1], "dy": dys[i & 1], "y": ys[i & 1], "dx": dxs[i & 1]}
            if routes[0] is not None:
                st["route"] = routes[i & 1]
            out.append(st)
        return out

    h2d = sum(t.numel() * t.element_size() for t in (xs[0], dys[0]))
    if routes[0] is not None:
        h2d += routes[0].numel() * routes[0].element_size()
    d2h = ys[0].numel() * ys[0].element_size() + dxs[0].numel() * dxs[0].element_size()
    stepper.run(plan(warmup), g["w_r"], g["w_gu"], g["w_d"], g["bias"])
    torch.cuda.synchronize(dev)
    start = torch.cuda.Event(enable_timing=True)
    start.record(stepper.compute)
    stepper.run(plan(steps), g["w_r"], g["w_gu"], g["w_d"], g["bias"], after=start)
    end = stepper.done_event()
    torch.cuda.synchronize(dev)
    e2e_ms = start.elapsed_time(end)
    # the host link alone: the same per-step copies, both directions at once, no kernels
    start = torch.cuda.Event(enable_timing=True)
    start.record(stepper.compute)
    stepper.copy_in.wait_event(start)
    stepper.copy_out.wait_event(start)
    for i in range(steps):
        with torch.cuda.stream(stepper.copy_in):
            stepper.x[i & 1].copy_(xs[i & 1], non_blocking=True)
            stepper.dy[i & 1].copy_(dys[i & 1], non_blocking=True)
            if routes[0] is not None:
                stepper.route[i & 1].copy_(routes[i & 1], non_blocking=True)
        with torch.cuda.stream(stepper.copy_out):
            ys[i & 1].copy_(stepper.y[i & 1], non_blocking=True)
            dxs[i & 1].copy_(stepper.dx[i & 1], non_blocking=True)
    end = stepper.done_event()
    torch.cuda.synchronize(dev)
    return e2e_ms, h2d, d2h, start.elapsed_time(end)


def run_ours(args):
    import torch
    import torch.distributed as dist
    from mixture_experts_layer_39_b200.inputs import CONFIGS, make_inputs
    from mixture_experts_layer_39_b200.layer import MoELayer

    ws, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if ws > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    def max_over_ranks(v):
        from mixture_experts_layer_39_b200.replicas import max_over_ranks as mor
        return mor(v, dev)

    def barrier():
        if ws > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)

    cfg = CONFIGS[args.workload]
    flush = L2Flush(dev)
    sampler = ClockSampler(local)

    def bench_cfg(c, steps, warmup, with_e2e, dtype="bf16", **layer_kw):
        g = make_inputs(c, seed=rank, device=dev)
        L = MoELayer(c.T, c.d, c.f, c.E, c.k, device=dev, dtype=dtype, **layer_kw)
        barrier()
        step_ms, gemm_ms, launches = measure(L, g, steps, warmup, flush, dev)
        barrier()
        out = {"total_ms": max_over_ranks(sum(step_ms)), "step_ms": step_ms,
               "gemm_ms": gemm_ms, "launches": launches, "counts": L.counts.cpu().numpy()}
        if with_e2e:
            out["memory_bound"] = measure_memory_bound(L, g, flush)
            barrier()
            e2e_ms, h2d, d2h, link_ms = measure_e2e(L, g, steps, min(warmup, 3), dev)
            barrier()
            out.update({"e2e_total_ms": max_over_ranks(e2e_ms), "h2d": h2d, "d2h": d2h,
                        "link_total_ms": max_over_ranks(link_ms)})
        st = L.handle.get_status()
        if st != 0:
            raise RuntimeError(f"device status {st} after the benchmark")
        del L, g
        torch.cuda.empty_cache()
        return out

    sampler.start()
    main = bench_cfg(cfg, args.steps, args.warmup, True, dtype=args.dtype)
    # variants right after the main workload, on the same warm GPU
    variants = {}
    if not args.no_variants and args.dtype == "bf16":
        variants["aux_loss"] = bench_cfg(cfg, args.steps, args.warmup, False, aux_alpha=0.01)
        variants["recompute"] = bench_cfg(cfg, args.steps, args.warmup, False, recompute=True)
        variants["gather"] = bench_cfg(cfg, args.steps, args.warmup, False, gather=True)
        variants["fused_combine"] = bench_cfg(cfg, args.steps, args.warmup, False,
                                              fuse_combine=True)
        if cfg.name == "e8":
            variants["shared_expert"] = bench_cfg(CONFIGS["e8_shared"], args.steps, args.warmup,
                                                  False, shared_ff=CONFIGS["e8_shared"].shared_ff)
    ratio = None
    if not args.no_ratio and cfg.name == "e8":
        ratio = bench_cfg(CONFIGS["e128"], args.steps, args.warmup, False)
    skew = None
    if not args.no_skew and cfg.name == "e8":
        skew = bench_cfg(CONFIGS["skew"], args.steps, args.warmup, False)
    mx = mx_bf16 = None
    if not args.no_mxfp8 and cfg.name == "e8":
        mx = bench_cfg(CONFIGS["mxfp8"], args.steps, args.warmup, False, dtype="mxfp8")
        # the same workload with bf16 expert GEMMs, for the MXFP8-vs-BF16 comparison
        mx_bf16 = bench_cfg(CONFIGS["mxfp8"], args.steps, args.warmup, False, dtype="bf16")
    clocks = sampler.stop()

    K = args.steps
    tokens = cfg.T * K * ws
    value = tokens / (main["total_ms"] / 1e3)
    e2e_value = tokens / (main["e2e_total_ms"] / 1e3)
    peaks, peak_kind = load_peaks()
    gemm_flops = cfg.gemm_flops_fwd_bwd()
    gemm_ms = statistics.mean(main["gemm_ms"])
    achieved = gemm_flops / (gemm_ms / 1e3) / 1e12
    traffic = gemm_traffic(cfg.name)
    counts = main["counts"]
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": K,
        "warmup": args.warmup, "ms_per_step": main["total_ms"] / K, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if args.dtype == "bf16" else "mxfp8 (e4m3 + e8m0/32)",
        "data": "synthetic (seeded N(0,1) activations, N(0,1/d) weights, learned-style routing)",
        "config": {"workload": f"{cfg.name}: T={cfg.T} d_model={cfg.d} d_ff={cfg.f} E={cfg.E} "
                               f"top_k={cfg.k}"
                               + (f" ({cfg.T // 4096}x4096 tokens)" if cfg.T % 4096 == 0 else ""),
                   "global_batch": cfg.T * ws, "parallelism": f"replicas{ws}" if ws > 1 else "1 GPU",
                   "l2": "flushed between timed steps outside the step events (512 MiB write, "
                         "then a 512 MiB read of another buffer)"},
        "roofline": {"bound": "tensor", "kernel": "grouped_gemm_kernel: every expert GEMM launch of a step "
                               "(events around the two expert calls)",
                     "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": achieved / peaks["bf16_tflops"], "traffic": traffic,
                     "peak_source": f"{peak_kind} bf16 burst",
                     "datasheet_peak": DATASHEET_BF16_TFLOPS,
                     "frac_of_datasheet": achieved / DATASHEET_BF16_TFLOPS},
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": main["h2d"],
                "d2h_bytes_per_step": main["d2h"],
                "how": "HostStepper: pinned-host x/dY in, y/dX out every step; copies of "
                       "neighbouring steps overlap the kernels on two copy streams",
                "copy_only_ms_per_step": main["link_total_ms"] / K,
                "of_copy_bound": main["link_total_ms"] / main["e2e_total_ms"],
                "copy_only_note": "the same copies with no kernels, both directions at once: "
                                  "the host link's bound on this number"},
        "gpu_launches": main["launches"],
        "grouped_gemm": {"tflops": achieved, "ms_per_step": gemm_ms,
                         "share_of_step": gemm_ms / (main["total_ms"] / K)},
        "routing": load_report(counts),
        "memory_bound": {
            "peak_gb_s": peaks["hbm_gbs"], "peak_source": f"{peak_kind} copy",
            "timing": "each call alone, CUDA events, L2 flushed before it, median of 10 (rank 0)",
            **{n: {**v, "frac": v["gb_s"] / peaks["hbm_gbs"]} for n, v in main["memory_bound"].items()}},
        "clocks": clocks,
    }
    if ratio is not None:
        r_value = CONFIGS["e128"].T * K * ws / (ratio["total_ms"] / 1e3)
        line["e128"] = {"value": r_value, "unit": UNIT, "vs_e8": r_value / value,
                        "grouped_gemm_tflops": CONFIGS["e128"].gemm_flops_fwd_bwd()
                        / (statistics.mean(ratio["gemm_ms"]) / 1e3) / 1e12}
    if skew is not None:
        sc = CONFIGS["skew"]
        sk_counts = skew["counts"]
        line["skew"] = {
            "workload": f"skew: T={sc.T} d_model={sc.d} d_ff={sc.f} E={sc.E} top_k={sc.k}, router "
                        "bias 2*ln(1/(e+1)), dropless (no capacity cap)",
            "value": sc.T * K * ws / (skew["total_ms"] / 1e3), "unit": UNIT,
            "ms_per_step": skew["total_ms"] / K,
            "grouped_gemm_tflops": sc.gemm_flops_fwd_bwd()
            / (statistics.mean(skew["gemm_ms"]) / 1e3) / 1e12,
            "routing": load_report(sk_counts)}
    if variants:
        base_ms = main["total_ms"] / K
        line["variants"] = {}
        for name, v in variants.items():
            ms = v["total_ms"] / K
            line["variants"][name] = {
                "value": cfg.T * K * ws / (v["total_ms"] / 1e3), "unit": UNIT, "ms_per_step": ms,
                "overhead_ms": ms - base_ms, "launches_per_step": v["launches"] / K}
        line["variants"]["aux_loss"]["what"] = (
            "the same step plus the load-balancing loss (alpha 0.01): load statistics, loss and "
            "its probability gradient in the router backward")
        if "recompute" in variants:
            M = cfg.T * cfg.k
            line["variants"]["recompute"]["what"] = (
                "activation recompute: the forward keeps no [A|U], the backward recomputes the "
                f"gate/up GEMM (+{4 * cfg.d * cfg.f * M / 1e9:.0f} GFLOP/step); activations "
                f"kept from forward to backward shrink by {(2 * cfg.f + cfg.f) * 2 * M / 2**20:.0f} "
                "MiB of [A|U] and H")
        if "gather" in variants:
            line["variants"]["gather"]["what"] = (
                "no permuted copy of x: the gate/up GEMM and its weight gradient gather the routed "
                "rows from x with TMA tile::gather4 (moe_route + *_gather entry points)")
        if "fused_combine" in variants:
            line["variants"]["fused_combine"]["what"] = (
                "the weighted unpermute-combine inside the down projection's epilogue "
                "(moe_permute_src + moe_grouped_swiglu_fwd_combine): the arrival that completes "
                "a token's rows sums them, same bits as the combine kernel, no separate launch")
        if "shared_expert" in variants:
            sc = CONFIGS["e8_shared"]
            v = variants["shared_expert"]
            line["variants"]["shared_expert"].update({
                "what": f"the same step plus a shared expert of d_ff {sc.shared_ff} on every token",
                "grouped_gemm_tflops": (sc.gemm_flops_fwd_bwd() + sc.shared_flops_fwd_bwd())
                / (statistics.mean(v["gemm_ms"]) / 1e3) / 1e12})
    if mx is not None:
        mc = CONFIGS["mxfp8"]
        line["mxfp8"] = {
            "workload": f"mxfp8: T={mc.T} d_model={mc.d} d_ff={mc.f} E={mc.E} top_k={mc.k}, "
                        "uniform random expert ids, E4M3 + E8M0/32 expert GEMM operands",
            "value": mc.T * K * ws / (mx["total_ms"] / 1e3), "unit": UNIT,
            "ms_per_step": mx["total_ms"] / K,
            "expert_calls_tflops": mc.gemm_flops_fwd_bwd() / (statistics.mean(mx["gemm_ms"]) / 1e3) / 1e12,
            "expert_calls_note": "18*d*f*T*k GEMM FLOPs over the two expert calls, MXFP8 "
                                 "quantisation kernels included"}
        mx_tf = line["mxfp8"]["expert_calls_tflops"]
        fp8_peak = FP8_OVER_BF16 * peaks["bf16_tflops"]
        line["mxfp8"]["roofline"] = {
            "bound": "tensor", "achieved": mx_tf, "peak": fp8_peak, "unit": "TFLOP/s",
            "frac": mx_tf / fp8_peak,
            "peak_source": f"{peak_kind} bf16 burst x {FP8_OVER_BF16} (the dense fp8/bf16 ratio "
                           "of the datasheet; no fp8 peak is measured)",
            "datasheet_peak": FP8_OVER_BF16 * DATASHEET_BF16_TFLOPS,
            "frac_of_datasheet": mx_tf / (FP8_OVER_BF16 * DATASHEET_BF16_TFLOPS),
            "note": "achieved counts the quantisation kernels' time too"}
        if mx_bf16 is not None:
            bf_value = mc.T * K * ws / (mx_bf16["total_ms"] / 1e3)
            line["mxfp8"].update({
                "bf16_value": bf_value, "bf16_ms_per_step": mx_bf16["total_ms"] / K,
                "vs_bf16": line["mxfp8"]["value"] / bf_value,
                "bf16_note": "the same workload and routing with bf16 expert GEMM operands"})
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = {k: v for k, v in cpu_baseline(cfg, args.cpu_seconds).items()
                                if k in ("value", "unit", "cores", "kind", "sample")}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if ws > 1:
        dist.barrier()
        dist.destroy_process_group()


# ------------------------------------------------------------------ API trace
SYNC_CALLS = ("Synchronize", "cudaMemcpy", "cuMemcpy", "cudaMemset", "cuMemset",
              "cudaMalloc", "cuMemAlloc", "cudaFree", "cuMemFree", "cudaStreamQuery",
              "cudaEventQuery")


def run_api_trace(args):
    """Eager steps of the layer under the CUDA profiler (CUPTI activity
    records through torch.profiler).  For every step, between its first and
    last host call: the runtime and driver API calls by name, the calls that
    copy, allocate or wait (SYNC_CALLS), and on the device timeline the
    kernels, copies and memsets the step's calls caused."""
    import torch
    from torch.profiler import ProfilerActivity, profile, record_function
    from mixture_experts_layer_39_b200.inputs import CONFIGS, make_inputs
    from mixture_experts_layer_39_b200.layer import MoELayer

    cfg = CONFIGS[args.workload]
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    g = make_inputs(cfg, seed=0, device=dev)
    L = MoELayer(cfg.T, cfg.d, cfg.f, cfg.E, cfg.k, device=dev, dtype=args.dtype)
    step = lambda: L.step(g["x"], g["w_r"], g["w_gu"], g["w_d"], g["dy"], g["bias"], g["route"])
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    n0 = L.handle.launch_count()
    with profile(activities=[ProfilerActivity.CPU, ProfilerActivity.CUDA]) as prof:
        for i in range(args.steps):
            with record_function(f"moe_layer_step_{i}"):
                step()
        torch.cuda.synchronize(dev)
    launches = (L.handle.launch_count() - n0) // max(1, args.steps)
    fd, path = tempfile.mkstemp(suffix=".json")
    os.close(fd)
    prof.export_chrome_trace(path)
    with open(path) as fh:
        trace = json.load(fh)
    os.unlink(path)
    ev = [e for e in trace.get("traceEvents", []) if e.get("ph") == "X"]
    steps = sorted((e for e in ev if e.get("cat") == "user_annotation"
                    and e.get("name", "").startswith("moe_layer_step_")), key=lambda e: e["ts"])
    api = [e for e in ev if e.get("cat") in ("cuda_runtime", "cuda_driver")]
    dev_ev = [e for e in ev if e.get("cat") in ("kernel", "gpu_memcpy", "gpu_memset")]
    per_step = []
    for sev in steps:
        t0, t1 = sev["ts"], sev["ts"] + sev["dur"]
        calls = [e for e in api if t0 <= e["ts"] <= t1]
        corr = {e.get("args", {}).get("correlation") for e in calls}
        caused = [e for e in dev_ev if e.get("args", {}).get("correlation") in corr]
        names = {}
        for e in calls:
            names[e["name"]] = names.get(e["name"], 0) + 1
        sync = {n: c for n, c in names.items() if any(k in n for k in SYNC_CALLS)
                and "Async" not in n}
        per_step.append({
            "api_calls": names,
            "sync_or_alloc_calls": sync,
            "async_copy_calls": {n: c for n, c in names.items() if "Memcpy" in n and "Async" in n},
            "device_kernels": sum(1 for e in caused if e["cat"] == "kernel"),
            "device_copies": [e["name"] for e in caused if e["cat"] == "gpu_memcpy"],
            "device_memsets": sum(1 for e in caused if e["cat"] == "gpu_memset"),
            "kernel_names": sorted({e["name"].split("(")[0][:80] for e in caused
                                    if e["cat"] == "kernel"}),
        })
    out = {"workload": cfg.name, "dtype": args.dtype, "steps": args.steps, "warmup": args.warmup,
           "tool": f"torch.profiler (Kineto/CUPTI) {torch.__version__}", "per_step": per_step,
           "library_launches_per_step": launches}
    with open(args.api_trace, "w") as fh:
        json.dump(out, fh, indent=1)
    print(json.dumps({"api_trace": args.api_trace,
                      "steps": [{"kernels": p["device_kernels"], "copies": len(p["device_copies"]),
                                 "sync_or_alloc": sum(p["sync_or_alloc_calls"].values())}
                                for p in per_step]}), flush=True)


# ------------------------------------------------------------------ reference arm
def run_reference(args):
    """The oracle, as it stands, on the host cores: each step is the layer's
    fwd+bwd on a bounded sample of the workload's tokens."""
    ws, rank, _ = dist_env()
    if rank != 0:
        return
    from mixture_experts_layer_39_b200.inputs import CONFIGS
    cfg = CONFIGS[args.workload]
    per_step = max(0.5, 150.0 / max(1, args.steps + args.warmup))
    T_s = size_oracle_sample(cfg, min(per_step, 4.0))
    inp = _oracle_inputs(cfg, T_s)
    for _ in range(args.warmup):
        _oracle_step(*inp[:4], inp[4], cfg.k, inp[5], inp[6])
    t0 = time.perf_counter()
    for _ in range(args.steps):
        _oracle_step(*inp[:4], inp[4], cfg.k, inp[5], inp[6])
    dt = time.perf_counter() - t0
    value = T_s * args.steps / dt
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3 / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": f"{cfg.name}: T={cfg.T} d_model={cfg.d} "
                                                    f"d_ff={cfg.f} E={cfg.E} top_k={cfg.k}"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                         "sample": f"each step: oracle fwd+bwd on the first {T_s} of {cfg.T} tokens"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse_args()
    if args.impl == "reference":
        run_reference(args)
    elif args.api_trace:
        run_api_trace(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
