"""Benchmark of the W4 + per-token-gated low-rank EC linear layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--workloads all|NAME,...] [--impl ours|reference]

One step is a pass of the whole hot path (gate, EC down-projection, W4 GEMM,
EC up-projection and combine, dispatch) over a stack of L distinct layers of
the workload's shape, once for every batch size M of the workload, through
the library's layer-stack call (spear_w4ec_stack_forward).  For a square
layer (K == N) the layers are chained (y of one layer is x of the next), as
in a decode pass through a model; otherwise each layer reads the same x.  L
is chosen so the packed weights of the stack exceed three times the L2 cache
(126 MB), so every forward streams its weights from HBM.

Headline workload (the JSON line's value): decode, attention q/o projection,
K = N = 4096, rank 32, M in {1, 4, 16}: algorithmic bytes moved per second
(GB/s).  The same run measures, the same way, the rest of the metric under
"workloads": the MLP up and down projections at decode batch sizes (GB/s)
and the prefill MLP shape (K = 4096, N = 14336, rank 64, M in {2048, 4096};
TFLOP/s).  Each record has its own roofline, EC overhead, end-to-end figure
(the host-buffer stack call, spear_w4ec_stack_forward_host) and clocks.

Under torchrun every rank runs the same stack on its own GPU (independent
replicas, no data-path collective: weak scaling); the time is the maximum
over ranks.  ``--impl reference`` times the fp64 CPU oracle on the host cores
on a bounded sample of the same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "W4+EC linear: decode weight GB/s and prefill TFLOP/s vs B200 roofline"
L2_BYTES = 126 * 1024 * 1024

WORKLOADS = {
    "decode_qo_4096x4096_r32": dict(Ms=(1, 4, 16), K=4096, N=4096, r=32, kind="decode", layer_kw={}),
    "decode_mlp_gateup_4096x14336_r64": dict(Ms=(1, 16, 64, 128), K=4096, N=14336, r=64, kind="decode",
                                             layer_kw={}),
    "decode_mlp_down_14336x4096_r64": dict(Ms=(1, 16, 64, 128), K=14336, N=4096, r=64, kind="decode",
                                           layer_kw={}),
    "prefill_mlp_4096x14336_r64": dict(Ms=(2048, 4096), K=4096, N=14336, r=64, kind="prefill",
                                       layer_kw=dict(w_row_outlier_frac=0.005, gate_open_frac=0.3)),
}


def reduce_over_ranks(ms: float, units: float, world: int, device=None):
    """Whole-job figures of a replicas run: the slowest rank's time and the
    units all ranks processed (every rank does the same work)."""
    if world <= 1:
        return ms, units
    import torch
    import torch.distributed as dist
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    u = torch.tensor([units], dtype=torch.float64, device=device)
    dist.all_reduce(u, op=dist.ReduceOp.SUM)
    return float(t.item()), float(u.item())


def alg_bytes(M, K, N, r):
    """Bytes the method must move for one forward (no split-K partials, no padding)."""
    return N * K // 2 + 4 * N + N + 2 * K * r + 2 * r * N + 2 * K + 2 * M * K + 2 * M * N


def alg_flops(M, K, N, r):
    return 2 * M * N * K + 2 * M * K + 2 * M * K * r + 2 * M * r * N


def packed_bytes(K, N, r):
    return N * K // 2 + 5 * N + 2 * K * (r + 1) + 2 * r * N


TRAFFIC_FILE = os.path.join(ROOT, "bench_traffic.json")


def load_traffic():
    """Measured DRAM bytes per launch of each workload's dominant kernel (one
    ncu capture per kernel source state; see bench_traffic.json)."""
    with open(TRAFFIC_FILE) as f:
        data = json.load(f)["workloads"]
    return {name: dict(t, bytes={int(m): float(b) for m, b in t["bytes"].items()}) for name, t in data.items()}


def sources_sha(files):
    import hashlib
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "w4_gemm_error_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def traffic_per_launch(workload, Ms):
    """Mean measured DRAM bytes per launch over the step's batch sizes, or None
    (no capture, or the kernel sources changed since it was taken)."""
    t = load_traffic().get(workload)
    if t is None or any(M not in t["bytes"] for M in Ms):
        return None
    if sources_sha(t["files"]) != t["sha"]:
        return None
    return round(sum(t["bytes"][M] for M in Ms) / len(Ms))


def path_name(choice):
    from w4_gemm_error_b200 import spear
    path = "decode" if choice & spear.SPEAR_FORCE_DECODE else "tcgen05"
    return path + ("+split" if choice & spear.SPEAR_FORCE_SPLIT else "+fused")


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return dict(hbm=float(p["hbm_gbs"]), bf16=float(p["bf16_tflops"]),
                    bf16_sustained=float(p.get("bf16_tflops_sustained", p["bf16_tflops"])), source="measured")
    except Exception:
        return dict(hbm=6650.0, bf16=1590.0, bf16_sustained=1400.0, source="fallback")


# ------------------------------------------------------------------ clocks (NVML)

_REASONS = {
    0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
    0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
    0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
}


class ClockSampler:
    """Samples SM clock and clock-event reasons every few ms while running."""

    def __init__(self, device_index: int, period_s: float = 0.005):
        self.samples = []
        self.max_mhz = None
        self.period = period_s
        self._stop = threading.Event()
        self._thr = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nvml = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._nvml = None

    def _run(self):
        nv = self._nvml
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM)
                reasons = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                self.samples.append((mhz, reasons))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self._nvml:
            self._thr = threading.Thread(target=self._run, daemon=True)
            self._thr.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._thr:
            self._thr.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unsampled"]}
        busy = [s for s in self.samples if not (s[1] & 0x1)] or self.samples
        reasons = set()
        for _, bits in busy:
            for b, name in _REASONS.items():
                if bits & b and name != "gpu_idle":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(m for m, _ in busy), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(reasons), "samples": len(busy)}


# ------------------------------------------------------------------ our arm

def _timed_region_peak(peaks, seconds):
    """bf16 denominator for a timed region of `seconds`: the burst figure for a
    region under two seconds, the sustained (power-capped) one for longer."""
    if seconds < 2.0:
        return peaks["bf16"], peaks["source"] + " (burst: timed region %.2f s)" % seconds
    return peaks["bf16_sustained"], peaks["source"] + " (sustained: timed region %.2f s)" % seconds


def measure_workload(name, args, rank, world, local_rank, cpu_seconds):
    """Time one workload on this rank's GPU: the graph-captured stack (EC on and
    EC off) on device-resident inputs, and the host-buffer stack call end to
    end.  Returns the rank-0 record (None elsewhere)."""
    import torch
    import torch.distributed as dist
    from w4_gemm_error_b200.inputs import make_layer, make_x
    from w4_gemm_error_b200 import spear

    wl = WORKLOADS[name]
    K, N, r, Ms = wl["K"], wl["N"], wl["r"], wl["Ms"]
    dev = torch.device("cuda", local_rank)
    stream = torch.cuda.Stream(device=dev)

    L = args.layers or max(1, math.ceil(3 * L2_BYTES / packed_bytes(K, N, r)))
    if wl["kind"] == "prefill" and not args.layers:
        L = 2  # each forward moves > L2 bytes of activations already; two layers alternate weights
    chain = (K == N)
    base = make_layer(K, N, r, seed=0, **wl["layer_kw"])
    layers = []
    with torch.cuda.stream(stream):
        W0, A0, B0 = base.W.to(dev), base.A.to(dev), base.B.to(dev)
        wg = base.wg.to(dev)
        for i in range(L):
            # distinct weights per layer: rows / columns rotated copies of the seeded layer
            W = torch.roll(W0, shifts=97 * i, dims=0).contiguous()
            A = torch.roll(A0, shifts=13 * i, dims=0).contiguous()
            B = torch.roll(B0, shifts=31 * i, dims=1).contiguous()
            layers.append(spear.W4ECLinear(W, A, B, wg, base.b_g, max_M=max(Ms), stream=stream))
        del W0, A0, B0
    torch.cuda.synchronize(dev)
    # the step's layer sequence as one stack (spear_w4ec_stack_*): chained
    # (square layers: y of layer l is x of layer l + 1) or all reading x;
    # intermediates alternate between two buffers; every EC placed
    ops = []
    for i, lin in enumerate(layers):
        src = 0 if (i == 0 or not chain) else 2 + (i - 1) % 2
        dst = 1 if i == L - 1 else 2 + i % 2
        ops.append((lin, src, dst, 1))
    stack = spear.W4ECStack(ops, max(Ms))
    if args.no_prefetch:
        for lin in layers:
            lin.set_next(None)

    xs = {M: make_x(M, K, seed=0).to(dev) for M in Ms}
    ys = {M: torch.empty((M, N), dtype=torch.bfloat16, device=dev) for M in Ms}

    def step(flags=0):
        for M in Ms:
            stack.forward(xs[M], flags, out=ys[M], stream=stream)

    def capture(flags):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            step(flags)  # first call outside capture: lazy allocations, kernel attributes
            torch.cuda.synchronize(dev)
            with torch.cuda.graph(g, stream=stream):
                step(flags)
        torch.cuda.synchronize(dev)
        return g

    def timed(g, steps, warmup, sample_clocks=False):
        for _ in range(warmup):
            g.replay()
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        sampler = ClockSampler(local_rank) if sample_clocks else None
        ctx = sampler if sampler else _Null()
        with ctx:
            with torch.cuda.stream(stream):
                e0.record(stream)
                for _ in range(steps):
                    g.replay()
                e1.record(stream)
            e1.synchronize()
        torch.cuda.synchronize(dev)
        ms, _ = reduce_over_ranks(e0.elapsed_time(e1), 0.0, world, dev)
        if world > 1:
            dist.barrier()
        return ms, (sampler.summary() if sampler else None)

    # the library's default dispatch, then the adaptive one: layer 0 times every
    # legal path per batch size (spear_w4ec_tune), its table goes out as JSON and
    # into every layer (spear_w4ec_table_save / _load; the layers share a shape);
    # the faster of the two is the step that is reported
    g_def_on, g_def_off = capture(0), capture(spear.SPEAR_EC_OFF)
    paths_default = {str(M): path_name(layers[0].dispatch(M)) for M in Ms}
    table_text = None
    if not args.no_tune:
        with torch.cuda.stream(stream):
            for M in Ms:
                layers[0].tune(xs[M], ys[M], stream=stream)
        torch.cuda.synchronize(dev)
        table_text = layers[0].table_json()
        for lin in layers[1:]:
            lin.load_table(table_text)
    paths_tuned = {str(M): path_name(layers[0].dispatch(M)) for M in Ms}
    ms_def, clocks_def = timed(g_def_on, args.steps, args.warmup, sample_clocks=True)
    if table_text is not None and paths_tuned != paths_default:
        g_tun_on, g_tun_off = capture(0), capture(spear.SPEAR_EC_OFF)
        ms_tun, clocks_tun = timed(g_tun_on, args.steps, args.warmup, sample_clocks=True)
    else:
        g_tun_on = g_tun_off = None
        ms_tun, clocks_tun = float("inf"), None
    tuned_wins = ms_tun < ms_def
    if tuned_wins:
        ms_on, clocks, g_off = ms_tun, clocks_tun, g_tun_off
        paths = paths_tuned
    else:
        ms_on, clocks, g_off = ms_def, clocks_def, g_def_off
        paths = paths_default
        if table_text is not None:
            # back to the default rule for the end-to-end run below
            untuned = json.loads(table_text)
            for b in untuned["buckets"]:
                b["choice"] = None
            for lin in layers:
                lin.load_table(json.dumps(untuned))
    ms_off, _ = timed(g_off, args.steps, args.warmup)
    del g_def_on, g_def_off, g_tun_on, g_tun_off

    forwards_per_step = L * len(Ms)
    if wl["kind"] == "decode":
        units_per_step = sum(alg_bytes(M, K, N, r) for M in Ms) * L
        unit, scale = "GB/s", 1e9
    else:
        units_per_step = sum(alg_flops(M, K, N, r) for M in Ms) * L
        unit, scale = "TFLOP/s", 1e12
    _, total_units = reduce_over_ranks(0.0, float(units_per_step * args.steps), world, dev)
    value = total_units / (ms_on * 1e-3) / scale
    per_gpu = value / world
    ms_per_step = ms_on / args.steps
    ec_overhead = ms_on / ms_off - 1.0

    # end to end through the public C ABI: one host-buffer stack call per batch
    # size and step (spear_w4ec_stack_forward_host: pinned x in, the layers on
    # the device, y out, stream synchronised), wall clock
    x_host = {M: make_x(M, K, seed=0).pin_memory() for M in Ms}
    y_host = {M: torch.empty((M, N), dtype=torch.bfloat16).pin_memory() for M in Ms}
    e2e_steps = max(3, min(args.steps, 50))

    def e2e_step():
        for M in Ms:
            stack.forward_host(x_host[M], y_host[M], stream=stream)

    for _ in range(3):
        e2e_step()
    if world > 1:
        dist.barrier()
    t0 = time.perf_counter()
    for _ in range(e2e_steps):
        e2e_step()
    e2e_s, e2e_units = reduce_over_ranks(time.perf_counter() - t0, float(units_per_step * e2e_steps), world, dev)
    e2e_value = e2e_units / e2e_s / scale
    h2d = sum(M * K * 2 for M in Ms)
    d2h = sum(M * N * 2 for M in Ms)

    peaks = load_peaks()
    tr = load_traffic().get(name, {})
    if wl["kind"] == "decode":
        roof = {"bound": "hbm", "achieved": round(per_gpu, 1), "peak": peaks["hbm"], "unit": "GB/s",
                "frac": round(per_gpu / peaks["hbm"], 4), "traffic": traffic_per_launch(name, Ms),
                "alg_bytes_per_launch": round(sum(alg_bytes(M, K, N, r) for M in Ms) / len(Ms)),
                "kernel": tr.get("kernel", "decode kernels") +
                          ": per-forward time in the stack (one decode launch per forward; at 64 and 128 "
                          "tokens the tcgen05 kernel and its prepass)",
                "peak_source": peaks["source"] + " (HBM copy)"}
    else:
        pk, src_note = _timed_region_peak(peaks, ms_on * 1e-3)
        roof = {"bound": "tensor", "achieved": round(per_gpu, 1), "peak": pk, "unit": "TFLOP/s",
                "frac": round(per_gpu / pk, 4), "traffic": traffic_per_launch(name, Ms),
                "alg_flops_per_launch": round(sum(alg_flops(M, K, N, r) for M in Ms) / len(Ms)),
                "kernel": "tc_w4ec_kernel: per-forward time, which also holds the tc_prepass_kernel launch, "
                          "so the kernel's own rate is higher",
                "peak_source": src_note}

    launches_per_forward = {}
    for M in Ms:
        ch = layers[0].dispatch(M)   # the dispatch of the reported step
        if ch & spear.SPEAR_FORCE_DECODE:
            split = bool(r and ch & spear.SPEAR_FORCE_SPLIT)
            n = math.ceil(M / 32) + (2 if split else 0)   # split: prepass + separate EC kernel
        else:
            n = 1 + (1 if r else 0) + (1 if (r and ch & spear.SPEAR_FORCE_SPLIT) else 0)
        launches_per_forward[M] = n
    gpu_launches = args.steps * L * sum(launches_per_forward.values())

    # bytes one step touches: every layer's packed weights, each M's input and its output buffers
    touched = packed_bytes(K, N, r) * L + sum(M * K * 2 + min(L, 3) * M * N * 2 for M in Ms)
    out = None
    if rank == 0:
        cpu = cpu_baseline(wl, cpu_seconds) if (world == 1 and cpu_seconds > 0) else None
        out = {
            "value": round(value, 2), "unit": unit, "ms_per_step": round(ms_per_step, 4),
            "config": {"workload": name, "M": list(Ms), "K": K, "N": N, "r": r, "layers": L,
                       "chained": chain, "forwards_per_step": forwards_per_step,
                       "weights": "int4 per output channel (RTN), A/B/w_g bf16",
                       "l2": f"inputs larger than L2: each step touches {touched / 1e6:.0f} MB "
                             f"({L} distinct packed layers, {packed_bytes(K, N, r) * L / 1e6:.0f} MB, "
                             f"plus activations) > 126 MB",
                       "api": "spear_w4ec_stack_forward (one stack of the L layers, every EC placed) per M",
                       "graph": "one CUDA graph per step, kernels chained with programmatic dependent launch",
                       "prefetch": "off" if args.no_prefetch else
                                   "each layer's decode kernel reads the next layer's codes from HBM into L2",
                       "dispatch": ("tuned (spear_w4ec_tune on layer 0 per M, table loaded into every layer as "
                                    "JSON): faster than the default rule") if tuned_wins else
                                   ("library default rule" + ("" if table_text is None else
                                    " (the tuned table was measured too and was not faster)")),
                       "paths": paths,
                       "step_ms": {"default": round(ms_def / args.steps, 4),
                                   "tuned": None if ms_tun == float("inf") else round(ms_tun / args.steps, 4)},
                       "parallelism": f"replicas x{world}"},
            "ec_overhead": round(ec_overhead, 4),
            "e2e": {"value": round(e2e_value, 2), "unit": unit, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h,
                    "api": "spear_w4ec_stack_forward_host per M (C ABI, pinned host x and y, copies and "
                           "stream sync inside the timed region)"},
            "roofline": roof, "clocks": clocks, "gpu_launches": gpu_launches,
            "cpu_baseline": cpu,
        }
    stack.close()
    for lin in layers:
        lin.close()
    del layers
    torch.cuda.synchronize(dev)
    torch.cuda.empty_cache()
    return out


def run_ours(args, rank, world, local_rank):
    import torch
    torch.cuda.set_device(local_rank)
    names = [args.workload]
    if args.workloads == "all":
        names += [n for n in WORKLOADS if n != args.workload]
    elif args.workloads:
        names += [n for n in args.workloads.split(",") if n and n != args.workload]
    records = {}
    for i, name in enumerate(names):
        if name not in WORKLOADS:
            raise SystemExit(f"unknown workload {name}")
        cpu_s = 0.0 if args.no_cpu_baseline else (10.0 if i == 0 else 3.0)
        records[name] = measure_workload(name, args, rank, world, local_rank, cpu_s)
    if rank != 0:
        return None
    head = records[args.workload]
    out = {"metric": METRIC, "value": head["value"], "unit": head["unit"], "n_gpus": world, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": head["ms_per_step"], "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
           "config": head["config"], "ec_overhead": head["ec_overhead"], "e2e": head["e2e"],
           "roofline": head["roofline"], "clocks": head["clocks"], "gpu_launches": head["gpu_launches"],
           "cpu_baseline": head["cpu_baseline"]}
    if len(names) > 1:
        # the metric's other half and the other shapes, measured the same way in this process
        out["workloads"] = {n: records[n] for n in names}
    return out


class _Null:
    def __enter__(self):
        return self

    def __exit__(self, *a):
        return False


# ------------------------------------------------------------------ oracle timing

def _oracle_sample(wl):
    """The bounded CPU sample: one layer of the workload, every M (prefill: a row band)."""
    import numpy as np
    from w4_gemm_error_b200.inputs import make_layer, make_x
    import oracle
    K, N, r, Ms = wl["K"], wl["N"], wl["r"], wl["Ms"]
    lay = make_layer(K, N, r, seed=0, **wl["layer_kw"])
    codes, s, z = oracle.pack(lay.W)
    jobs = []
    for M in Ms:
        x = make_x(M, K, seed=0)
        if wl["kind"] == "decode":
            jobs.append(("full", M, x))
        else:
            rng = np.random.default_rng(M)
            cnt = 256
            jobs.append(("sampled", M, x, rng.integers(0, M, cnt), rng.integers(0, N, cnt)))
    return lay, codes, s, z, jobs


def _run_oracle_sample(wl, lay, codes, s, z, jobs):
    import oracle
    K, N, r = wl["K"], wl["N"], wl["r"]
    units = 0.0
    for job in jobs:
        if job[0] == "full":
            _, M, x = job
            oracle.forward(x, codes, s, z, lay.A, lay.B, lay.wg, lay.b_g)
            units += alg_bytes(M, K, N, r) if wl["kind"] == "decode" else alg_flops(M, K, N, r)
        else:
            _, M, x, t, n = job
            oracle.forward_sampled(x, codes, s, z, lay.A, lay.B, lay.wg, lay.b_g, t, n)
            units += len(t) * (2 * K + 2 * K * (r + 1) + 2 * r)   # flops of the sampled outputs
    return units


def cpu_baseline(wl, min_seconds=10.0):
    import oracle
    lay, codes, s, z, jobs = _oracle_sample(wl)
    _run_oracle_sample(wl, lay, codes, s, z, jobs)  # warm
    t0 = time.perf_counter()
    units, reps = 0.0, 0
    while time.perf_counter() - t0 < min_seconds:
        units += _run_oracle_sample(wl, lay, codes, s, z, jobs)
        reps += 1
    dt = time.perf_counter() - t0
    scale = 1e9 if wl["kind"] == "decode" else 1e12
    what = ("one layer, M in %s, full outputs" % (list(wl["Ms"]),)) if wl["kind"] == "decode" else \
        ("one layer, 256 sampled outputs per M in %s" % (list(wl["Ms"]),))
    return {"value": units / dt / scale, "unit": "GB/s" if wl["kind"] == "decode" else "TFLOP/s",
            "cores": oracle.num_threads(), "kind": "oracle", "seconds": round(dt, 2),
            "sample": f"{what}, repeated {reps}x"}


def run_reference(args, rank, world):
    if rank != 0:
        return None
    import oracle
    wl = WORKLOADS[args.workload]
    lay, codes, s, z, jobs = _oracle_sample(wl)
    for _ in range(args.warmup):
        _run_oracle_sample(wl, lay, codes, s, z, jobs)
    t0 = time.perf_counter()
    units = 0.0
    for _ in range(args.steps):
        units += _run_oracle_sample(wl, lay, codes, s, z, jobs)
    dt = time.perf_counter() - t0
    scale = 1e9 if wl["kind"] == "decode" else 1e12
    unit = "GB/s" if wl["kind"] == "decode" else "TFLOP/s"
    value = units / dt / scale
    sample = (f"one layer of {args.workload}, M in {list(wl['Ms'])}"
              + (" (full outputs)" if wl["kind"] == "decode" else " (256 sampled outputs per M)") + " per step")
    return {"metric": METRIC, "value": round(value, 4), "unit": unit, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(dt * 1e3 / max(args.steps, 1), 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": {"workload": args.workload, "M": list(wl["Ms"]), "K": wl["K"], "N": wl["N"], "r": wl["r"]},
            "cpu_baseline": {"value": round(value, 4), "unit": unit, "cores": oracle.num_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 4), "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="decode_qo_4096x4096_r32", choices=sorted(WORKLOADS),
                    help="the headline workload of the JSON line")
    ap.add_argument("--workloads", default="all",
                    help="further workloads measured in the same run and reported under 'workloads' "
                         "(comma-separated names, 'all' (default) or '' for none)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--layers", type=int, default=0, help="layers in the stack (0: enough to exceed 3x L2)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-prefetch", action="store_true",
                    help="do not chain the layers with the cross-layer L2 prefetch hint")
    ap.add_argument("--no-tune", action="store_true",
                    help="skip the adaptive dispatch (spear_w4ec_tune) and report the library's default rule")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        out = run_reference(args, rank, world)
        if out:
            print(json.dumps(out), flush=True)
        return

    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        out = run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    if out:
        print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
