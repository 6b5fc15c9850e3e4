#!/usr/bin/env python
"""Benchmark of the MXSens mixed-width MXINT hot path on B200.

One STEP is one pass of the whole path over one batch of synthetic
Llama-3-8B-shaped layers (every call through the C ABI):
  attention projection  W 4096x4096 (3% Student-t(3) columns), calibration
                        X 2048x4096 (8 outlier channels x50), GEMM M in
                        {2048, 16, 1};
  MLP gate/up           W 14336x4096, X as above, GEMM M in {8192, 16, 1};
  MLP down              W 4096x14336, X and A Laplace(0, 0.1) with 0.5%
                        spikes x100, GEMM M in {8192, 16, 1};
each: sensitivity(X, W) -> allocate (budget 4.5 bits) -> quantize W ->
for each M: quantize A_M -> gemm(A_M, W); then the K/V cache of the stack
workload (8192 tokens x 8 kv heads x 128, K and V) is quantised to MXINT4
and one decode step of attention (32 query heads) reads it.
`value` = the step's GEMM FLOPs (2 M N K summed over all GEMMs) per second of
whole-step time, summed over ranks; the per-call numbers, the roofline of the
dominant kernel, the mixed-width overhead against uniform MXINT4 and the
average-bit budget sweep are reported beside it.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

With --gpus N > 1 and no torchrun environment, the script relaunches itself
under torch.distributed.run with N processes (one per GPU).  `--impl
reference` times the CPU oracle (plain single-threaded C, fp64) on the host
cores instead, on a bounded row sample of the same workload per step.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import platform
import re
import socket
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

T_CAL = 2048
BUDGET = (9, 2)
SEED = 2000
KV_SHAPE = (8192, 8, 128)          # tokens, kv heads, head dim
N_QH = 32                          # query heads of the decode step
CALL_REPS, CALL_TRIALS = 10, 5     # per-call timing: calls per graph, replays per graph
METRIC = "mxs_gemm TFLOP/s (% of roofline); MXINT quantize GB/s (% of HBM peak)"
# (name, N, K, calibration/activation kind, M values)
LAYERS = (("attn", 4096, 4096, "gauss", (2048, 16, 1)),
          ("mlp_up", 14336, 4096, "gauss", (8192, 16, 1)),
          ("mlp_down", 4096, 14336, "laplace", (8192, 16, 1)))
WORKLOAD = ("llama3-8b layer: attention projection W 4096x4096 (M 2048/16/1), MLP gate/up W 14336x4096 and "
            "down W 4096x14336 (M 8192/16/1), bf16, calib X 2048 rows, budget 4.5 bits each; K/V cache "
            "8192x8x128 bf16 x2 to MXINT4 + one decode-attention step (32 query heads)")
SWEEP_BUDGETS = ((7, 2), (129, 32), (17, 4), (9, 2), (5, 1), (23, 4))     # 3.5 ... 5.75 average bits
# Llama-2-70B-shaped stack: 80 layers of these linears (N, K), N(0, 0.015^2)
# weights with 2% of the columns x20, 4.25 bits each, all quantised in place
L70_SHAPES = (("q", 8192, 8192), ("k", 1024, 8192), ("v", 1024, 8192), ("o", 8192, 8192),
              ("gate", 28672, 8192), ("up", 28672, 8192), ("down", 8192, 28672))
L70_LAYERS = 80
L70_BUDGET = (17, 4)
L70_SEED = 5000                    # matrix j of layer l: seed L70_SEED + 16 l + j
# Llama-3-8B-shaped stack: 32 layers of these linears, the attention weight
# recipe, one 4.5-bit budget over all 224 matrices
L8_SHAPES = (("q", 4096, 4096), ("k", 1024, 4096), ("v", 1024, 4096), ("o", 4096, 4096),
             ("gate", 14336, 4096), ("up", 14336, 4096), ("down", 4096, 14336))
L8_LAYERS = 32
L8_SEED = 4000


def peaks():
    p = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}
    try:
        m = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
        p.update({k: float(m[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")})
        p["source"] = "measured"
    except (OSError, KeyError, ValueError):
        pass
    # Until measured on the device (measure_fp8_tflops), the E4M3 peak is
    # taken as 2x bf16 (the nominal dense ratio, 4.5 vs 2.25 PFLOP/s).
    p["fp8_tflops"] = 2.0 * p["bf16_tflops"]
    p["fp8_source"] = "2x measured bf16 (no fp8 measurement)"
    return p


def measure_fp8_tflops(torch, dev, n=8192, reps=20):
    """Dense E4M3 GEMM rate of this GPU, measured the way the bf16 peak was:
    a library GEMM of two n x n E4M3 matrices (torch._scaled_mm, tensorwise
    unit scales, bf16 out), median of `reps` back-to-back calls after
    warm-up.  None if the library call is unavailable."""
    try:
        a = torch.randn(n, n, device=dev).to(torch.float8_e4m3fn)
        b = torch.randn(n, n, device=dev).to(torch.float8_e4m3fn)
        one = torch.ones((), device=dev)
        f = lambda: torch._scaled_mm(a, b.t(), scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
        for _ in range(3):
            f()
        ev = []
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            f()
            e1.record()
            ev.append((e0, e1))
        torch.cuda.synchronize()
        ms = statistics.median(x.elapsed_time(y) for x, y in ev)
        del a, b
        return 2.0 * n ** 3 / (ms * 1e-3) / 1e12
    except (RuntimeError, AttributeError, TypeError):
        return None


def layout_bytes(rows, counts, in_bytes):
    n8, n6, n4 = counts
    pad = lambda n: (n + 31) // 32 * 32
    codes = rows * (pad(n8) + pad(n6) * 6 // 8 + pad(n4) // 2)
    scales = rows * (pad(n8) + pad(n6) + pad(n4)) // 32
    return rows * (n8 + n6 + n4) * in_bytes + codes + scales


def gemm_roofline_s(M, N, counts, pk):
    """max(compute, bytes) time of one mxs_gemm: 4-bit at the FP8 peak, 6/8-bit at bf16."""
    n8, n6, n4 = counts
    t_c = 2.0 * M * N * n4 / (pk["fp8_tflops"] * 1e12) + 2.0 * M * N * (n8 + n6) / (pk["bf16_tflops"] * 1e12)
    byts = layout_bytes(M, counts, 0) + layout_bytes(N, counts, 0) + M * N * 2
    return max(t_c, byts / (pk["hbm_gbs"] * 1e9))


def attn_bytes(T, n_kvh, n_qh, d=128):
    """Algorithmic bytes of one decode-attention call: packed K and V (codes
    and one scale byte per 32 values), the bf16 query and the fp32 output."""
    cache = T * n_kvh * (d // 2 + d // 32)
    return 2 * cache + n_qh * d * 2 + n_qh * d * 4


def host_info():
    model = platform.processor() or ""
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                model = line.split(":", 1)[1].strip()
                break
    except OSError:
        pass
    return {"host_cores": os.cpu_count(), "cpu_model": model}


# --------------------------------------------------------------------- clocks
class ClockSampler:
    """NVML samples of SM clock and throttle reasons while running."""

    def __init__(self, index, period=0.001):
        self.index, self.period = index, period
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._t = None

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        except Exception as e:  # noqa: BLE001 - clocks are reported, not required
            self.error = str(e)
        return self

    def _run(self):
        nv = self._nv
        names = {getattr(nv, k): k for k in dir(nv) if k.startswith("nvmlClocksEventReason") or
                 k.startswith("nvmlClocksThrottleReason")}
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h) if hasattr(
                    nv, "nvmlDeviceGetCurrentClocksEventReasons") else nv.nvmlDeviceGetCurrentClocksThrottleReasons(self._h)
                for bit, name in names.items():
                    if isinstance(bit, int) and bit and bit != 0xFFFFFFFFFFFFFFFF and r & bit and bin(bit).count("1") == 1:
                        self.reasons.add(re.sub(r"^nvmlClocks(Event|Throttle)Reason", "", name))
            except Exception:  # noqa: BLE001
                pass
            time.sleep(self.period)

    def __exit__(self, *a):
        self._stop.set()
        if self._t:
            self._t.join()

    def summary(self):
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ------------------------------------------------------------------ GPU arm
def _layer_inputs(inputs, dev, seed, name, N, K, kind, Ms):
    W = inputs.attn_weight(dev, seed, N, K)
    if kind == "gauss":
        X = inputs.gaussian_acts(dev, seed + 1, T_CAL, K)
        A = {M: inputs.gaussian_acts(dev, seed + 2 + M, M, K) for M in Ms}
    else:
        X = inputs.laplace_acts(dev, seed + 1, T_CAL, K)
        A = {M: inputs.laplace_acts(dev, seed + 2 + M, M, K) for M in Ms}
    return W, X, A


class Layer:
    """One linear layer of the step: its inputs, quantised tensors and calls."""

    def __init__(self, c, inputs, dev, seed, name, N, K, kind, Ms):
        import torch
        self.c, self.name, self.N, self.K, self.Ms = c, name, N, K, Ms
        self.W, self.X, self.A = _layer_inputs(inputs, dev, seed, name, N, K, kind, Ms)
        self.sens_ws = torch.empty(c.mxs_sensitivity_workspace_bytes(T_CAL, N, K) + 1024, dtype=torch.uint8, device=dev)
        self.H = torch.empty(K, dtype=torch.float64, device=dev)
        self.E, self.s = torch.empty_like(self.H), torch.empty_like(self.H)
        self.perm = torch.empty(K, dtype=torch.int32, device=dev)
        self.alloc_ws = torch.empty(1 << 20, dtype=torch.uint8, device=dev)
        c.mxs_sensitivity(self.X, self.W, workspace=self.sens_ws, out=(self.H, self.E, self.s))
        _, counts = c.mxs_allocate([self.s], [N], mode="budget", budget=BUDGET, perms=[self.perm],
                                   workspace=self.alloc_ws)
        self.counts = counts[0]
        self.lay = c.mxs_layout_make(K, self.counts, self.perm)
        self.Wq = c.mxtensor_empty(N, self.lay, dev)
        self.Aq = {M: c.mxtensor_empty(M, self.lay, dev) for M in Ms}
        self.Y = {M: torch.empty(M, N, dtype=torch.bfloat16, device=dev) for M in Ms}
        c.mxs_quantize_weight(self.W, self.Wq)
        for M in Ms:
            c.mxs_quantize_act(self.A[M], self.Aq[M])
        gws = max(c.mxs_gemm_workspace_bytes(self.Aq[M], self.Wq) for M in Ms)
        self.gemm_ws = torch.empty(gws + 1024, dtype=torch.uint8, device=dev)

    def work(self):
        n = self.name
        w = {f"{n}.mxs_sensitivity": ("GB/s", (T_CAL + self.N) * self.K * 2),
             f"{n}.mxs_allocate": ("GB/s", self.K * 8 + self.K * 4),
             f"{n}.mxs_quantize_weight": ("GB/s", layout_bytes(self.N, self.counts, 2))}
        for M in self.Ms:
            w[f"{n}.mxs_quantize_act_M{M}"] = ("GB/s", layout_bytes(M, self.counts, 2))
            w[f"{n}.mxs_gemm_M{M}"] = ("TFLOP/s", 2 * M * self.N * self.K)
        return w

    def calls(self):
        c, n = self.c, self.name

        def alloc():
            _, counts = c.mxs_allocate([self.s], [self.N], mode="budget", budget=BUDGET, perms=[self.perm],
                                       workspace=self.alloc_ws)
            assert counts[0] == self.counts
        out = [(f"{n}.mxs_sensitivity", lambda: c.mxs_sensitivity(self.X, self.W, workspace=self.sens_ws,
                                                                    out=(self.H, self.E, self.s))),
               (f"{n}.mxs_allocate", alloc),
               (f"{n}.mxs_quantize_weight", lambda: c.mxs_quantize_weight(self.W, self.Wq))]
        for M in self.Ms:
            out.append((f"{n}.mxs_quantize_act_M{M}", lambda M=M: c.mxs_quantize_act(self.A[M], self.Aq[M])))
            out.append((f"{n}.mxs_gemm_M{M}", lambda M=M: c.mxs_gemm(self.Aq[M], self.Wq, Y=self.Y[M],
                                                                     workspace=self.gemm_ws)))
        return out


class Path:
    """Device buffers and the step of the hot path (all kernels through the C ABI)."""

    def __init__(self, dev, seed):
        import math
        import torch
        from mx_microscaling_mixed_b200 import capi, inputs
        self.torch, self.c = torch, capi
        c = capi
        self.layers = [Layer(c, inputs, dev, seed + 100 * i, *spec) for i, spec in enumerate(LAYERS)]
        T, H, D = KV_SHAPE
        self.KV = [inputs.kv_cache(dev, seed + 10 + i, T, H, D).reshape(-1, D) for i in range(2)]
        self.q = inputs.random_matrix(N_QH, D, device=dev, seed=seed + 20, dtype=torch.bfloat16, outlier_frac=0.0)
        self.kv_lay = c.mxs_layout_make(D, (0, 0, D))
        self.KVq = [c.mxtensor_empty(kv.shape[0], self.kv_lay, dev) for kv in self.KV]
        self.attn_out = torch.empty(N_QH, D, dtype=torch.float32, device=dev)
        self.attn_ws = torch.empty(c.mxs_attn_decode_workspace_bytes(T, N_QH, H, D) + 1024, dtype=torch.uint8,
                                   device=dev)
        self.sm_scale = 1.0 / math.sqrt(D)
        for i in range(2):
            c.mxs_quantize_act(self.KV[i], self.KVq[i])
        self.flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
        self.flush_small = self.flush[: 256 << 20]          # per-call timing: twice the L2
        # algorithmic bytes / FLOPs per launch of each timed call
        self.work = {}
        for L in self.layers:
            self.work.update(L.work())
        for i in range(2):
            self.work[f"kv.mxs_quantize_act_{'KV'[i]}"] = ("GB/s", layout_bytes(T * H, (0, 0, D), 2))
        self.work["kv.mxs_attn_decode"] = ("GB/s", attn_bytes(T, H, N_QH, D))
        self.gemm_flops = sum(2 * M * L.N * L.K for L in self.layers for M in L.Ms)

    def calls(self):
        """The step as (name, call) pairs in order; each call is one C-ABI entry point."""
        c = self.c
        out = []
        for L in self.layers:
            out += L.calls()
        for i in range(2):
            out.append((f"kv.mxs_quantize_act_{'KV'[i]}", lambda i=i: c.mxs_quantize_act(self.KV[i], self.KVq[i])))
        T, H, _ = KV_SHAPE
        out.append(("kv.mxs_attn_decode", lambda: c.mxs_attn_decode(self.q, self.KVq[0], self.KVq[1], T, H,
                                                                     self.sm_scale, out=self.attn_out,
                                                                     workspace=self.attn_ws)))
        return out

    def gemm_spec(self, name):
        layer, call = name.split(".", 1)
        L = next(x for x in self.layers if x.name == layer)
        return int(call.split("M")[-1]), L.N, L.counts


def max_over_ranks(t: float, world: int, device) -> float:
    """The job's time for a per-rank time t: the slowest rank's (a MAX
    all-reduce over the process group, which every rank joins)."""
    if world == 1:
        return t
    import torch
    import torch.distributed as dist
    tt = torch.tensor([t], device=device, dtype=torch.float64)
    dist.all_reduce(tt, op=dist.ReduceOp.MAX)
    return float(tt.item())


def job_tflops(flops_per_rank_step: float, steps: int, world: int, job_s: float) -> float:
    """Whole-job throughput: the work of every rank (each runs its own replica
    of the workload: weak scaling) over the slowest rank's time."""
    return world * flops_per_rank_step * steps / job_s / 1e12


def traffic_from_profile(pk_name: str, layer: str, per_units: float = 1.0):
    """dram bytes of one call of `layer`'s GEMM recorded in profiles/ (a line
    `dram_bytes_per_call[layer]: B`), if the GEMM source is unchanged since the
    capture; scaled by `per_units` (units of the bench launch per unit of the
    captured one) when the capture was a smaller case."""
    prof = os.path.join(ROOT, "profiles", pk_name)
    try:
        text = open(prof).read()
    except OSError:
        return None
    m = re.search(r"dram_bytes_per_call\[" + re.escape(layer) + r"\]:\s*([0-9.eE+]+)", text)
    h = re.search(r"source_sha256:\s*([0-9a-f]{64})", text)
    if not m or not h:
        return None
    src = os.path.join(ROOT, "mx_microscaling_mixed_b200", "csrc", "mxs_gemm.cu")
    if hashlib.sha256(open(src, "rb").read()).hexdigest() != h.group(1):
        return None
    return float(m.group(1)) * per_units


def _graph_timer(torch, cap):
    def timed(g):
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        g.replay()
        e.record()
        return s, e
    return timed


def run_gpu(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    from mx_microscaling_mixed_b200 import build
    build.build()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    from mx_microscaling_mixed_b200 import capi as c
    path = Path(dev, SEED + 97 * rank)
    pk = peaks()
    fp8 = measure_fp8_tflops(torch, dev)
    if fp8:
        pk["fp8_tflops"] = fp8
        pk["fp8_source"] = "measured on this GPU: torch._scaled_mm E4M3 8192^3, median of 20"
    for _ in range(args.warmup):
        path.flush.zero_()
        for _, fn in path.calls():
            fn()
    c.mxs_sync()

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    # The step is captured once as one CUDA graph (its kernels back to back,
    # no host launch gaps) and replayed once per timed step.  Each call is
    # then timed on its own by difference: a graph of CALL_REPS x (L2 flush,
    # call) against a graph of CALL_REPS flushes alone, both replayed
    # between CUDA events; the call's time is the difference / CALL_REPS, so
    # neither graph-launch gaps nor the flush enter it, and every call starts
    # with a cold L2.
    calls = path.calls()
    cap = torch.cuda.Stream()
    launches0 = c.mxs_launch_count()
    g_step = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_step, stream=cap):
        for _, fn in calls:
            fn()
    launches_per_step = c.mxs_launch_count() - launches0

    def rep_graph(fn):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=cap):
            for _ in range(CALL_REPS):
                path.flush_small.zero_()
                if fn is not None:
                    fn()
        return g
    g_flush = rep_graph(None)
    graphs = [(name, rep_graph(fn)) for name, fn in calls]
    for _ in range(3):
        path.flush.zero_()
        g_step.replay()
        g_flush.replay()
        for _, g in graphs:
            g.replay()
    c.mxs_sync()
    timed = _graph_timer(torch, cap)

    rec = {}
    step_ev = []
    barrier()
    with ClockSampler(local_rank) as clocks:
        t0 = time.perf_counter()
        for _ in range(args.steps):
            path.flush.zero_()                      # L2 flush, outside the step events
            step_ev.append(timed(g_step))
        barrier()
        wall = time.perf_counter() - t0
        for _ in range(CALL_TRIALS):
            rec.setdefault("", []).append(timed(g_flush))
            for name, g in graphs:
                rec.setdefault(name, []).append(timed(g))
        barrier()
    launches = launches_per_step * args.steps
    c.mxs_sync()
    step_ms = [s.elapsed_time(e) for s, e in step_ev]
    total_s = max_over_ranks(sum(step_ms) * 1e-3, world, dev)
    value = job_tflops(path.gemm_flops, args.steps, world, total_s)
    best = {name: min(s.elapsed_time(e) for s, e in evs) * 1e-3 for name, evs in rec.items()}
    per_call = {name: max(best[name] - best[""], 0.0) / CALL_REPS for name, _ in calls}
    call_sum = sum(per_call.values())
    del graphs, g_flush

    kernels = {}
    for name, per in per_call.items():
        unit, work = path.work[name]
        ach = work / per / (1e12 if unit == "TFLOP/s" else 1e9) if per > 0 else None
        kd = {"us": per * 1e6, "achieved": ach, "unit": unit, "share": per / call_sum}
        if unit == "GB/s":
            kd["frac_hbm"] = ach / pk["hbm_gbs"] if ach else None
            kd["frac_nominal_8tbs"] = ach / 8000.0 if ach else None
        else:
            M, N, counts = path.gemm_spec(name)
            rt = gemm_roofline_s(M, N, counts, pk)
            kd["roofline_us"] = rt * 1e6
            kd["frac"] = rt / per if per > 0 else None
            kd["bound"] = "hbm" if rt == (layout_bytes(M, counts, 0) + layout_bytes(N, counts, 0) + M * N * 2) / (
                pk["hbm_gbs"] * 1e9) else "tensor"
        kernels[name] = kd
    # the dominant kernel: the GEMM call with the largest share of the step
    dom = max((n for n in kernels if ".mxs_gemm_M" in n), key=lambda n: kernels[n]["us"])
    g = kernels[dom]
    M, N, counts = path.gemm_spec(dom)
    K = sum(counts)
    rt = g["roofline_us"] * 1e-6
    roof = {"kernel": f"{dom} (one call: gemm_stage_kernel + gemm_tc2_kernel), M={M} N={N} K={K}",
            "bound": "tensor", "achieved": g["achieved"], "peak": 2 * M * N * K / rt / 1e12, "unit": "TFLOP/s",
            "frac": g["frac"],
            "traffic": traffic_from_profile("gemm_mlp_prefill_M8192.md", dom.split(".")[0]) if dom.endswith("M8192") else None,
            "peak_basis": f"4-bit segment at the E4M3 peak ({pk['fp8_tflops']:.0f} TFLOP/s, {pk['fp8_source']}), "
                          f"6/8-bit at measured bf16 ({pk['bf16_tflops']:.0f}); of {pk['source']}"}

    # HBM-bound calls with a working set below L2 also timed back to back on
    # rotated input copies (more than twice the L2 between reuses)
    if not args.no_stream:
        for name, (us, frac) in run_stream(c, dev, path, torch, pk).items():
            kernels[name]["us_stream"] = us
            kernels[name]["frac_stream"] = frac
    e2e = run_e2e(path, args, dev, world)
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total_s / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "mxint4/6/8 codes; e4m3+bf16 MMA, f32 acc",
        "data": "synthetic (seeded; shapes and outlier structure of the workload)",
        "config": {"workload": WORKLOAD, "counts_n8_n6_n4": {L.name: list(L.counts) for L in path.layers},
                   "l2": "flushed between steps (512 MB write outside the step events)",
                   "parallelism": f"replicas x{world} (no data-path collective)",
                   "timing": "step = one CUDA graph of all C-ABI calls, replayed per step between CUDA events; "
                             f"kernels{{}}: per call, (graph of {CALL_REPS} x [L2 flush, call]) - (graph of "
                             f"{CALL_REPS} flushes), best of {CALL_TRIALS} replays each, / {CALL_REPS}; cold L2 per call, "
                             "launch gap included; us_stream/frac_stream (decode GEMMs, quantisers, sensitivity, decode "
                             "attention): "
                             "a graph of back-to-back calls cycling through input copies with > 2x L2 read between "
                             "reuses of a copy, best of 3 replays / calls",
                   "launches_per_step": launches_per_step},
        "roofline": roof, "kernels": kernels, "e2e": e2e, "gpu_launches": launches,
        "clocks": clocks.summary(), "wall_s_timed_region": wall,
    }
    if not args.no_extras:
        line["mixed_overhead"] = run_mixed_overhead(c, dev, path, torch)
        line["budget_sweep"] = run_budget_sweep(c, dev, path, torch, pk)
        line["stack70b_inplace"] = run_70b_inplace(c, dev, path, torch, pk)
        line["stack8b_global"] = run_8b_stack(c, dev, torch, pk)
    return line


L2_BYTES = 126 << 20


def run_stream(c, dev, path, torch, pk, trials=3):
    """Back-to-back time per call of the HBM-bound calls (decode GEMMs, K/V
    quantiser, decode attention, each layer's weight and prefill activation
    quantisers and sensitivity): a CUDA graph of 2 x n calls cycling through n copies
    of the call's large input, n chosen so more than twice the L2 of other
    copies is read between two uses of one copy (every call reads its input
    from HBM), replayed between CUDA events; best of `trials` / (2 n).  No L2
    flush sits between the calls, so the launch gap the isolated per-call
    timing pays is hidden by the programmatic launch chaining."""
    out = {}

    def measure(name, calls, unit_work, unit):
        g = torch.cuda.CUDAGraph()
        cap = torch.cuda.Stream()
        for fn in calls:
            fn()
        with torch.cuda.graph(g, stream=cap):
            for _ in range(2):
                for fn in calls:
                    fn()
        best = None
        for _ in range(trials):
            s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s0.record()
            g.replay()
            s1.record()
            torch.cuda.synchronize()
            t = s0.elapsed_time(s1) * 1e-3 / (2 * len(calls))
            best = t if best is None else min(best, t)
        return best

    ncopy = lambda nbytes: max(2, -(-2 * L2_BYTES // max(nbytes, 1)) + 1)
    for L in path.layers:
        wbytes = layout_bytes(L.N, L.counts, 0)
        copies = []
        for _ in range(ncopy(wbytes)):
            Wq = c.mxtensor_empty(L.N, L.lay, dev)
            c.mxs_quantize_weight(L.W, Wq)
            copies.append(Wq)
        for M in L.Ms[1:]:                                   # the decode rows
            calls = [lambda Wq=Wq, M=M: c.mxs_gemm(L.Aq[M], Wq, Y=L.Y[M], workspace=L.gemm_ws) for Wq in copies]
            t = measure(f"{L.name}.mxs_gemm_M{M}", calls, None, None)
            out[f"{L.name}.mxs_gemm_M{M}"] = (t * 1e6, gemm_roofline_s(M, L.N, L.counts, pk) / t)
        del copies
    T, H, D = KV_SHAPE
    kv_bytes = path.KV[0].numel() * 2
    srcs = [path.KV[0].clone() for _ in range(ncopy(kv_bytes))]
    calls = [lambda x=x: c.mxs_quantize_act(x, path.KVq[0]) for x in srcs]
    t = measure("kv.mxs_quantize_act_K", calls, None, None)
    work = path.work["kv.mxs_quantize_act_K"][1]
    out["kv.mxs_quantize_act_K"] = (t * 1e6, work / t / 1e9 / pk["hbm_gbs"])
    del srcs
    cache_bytes = 2 * layout_bytes(T * H, (0, 0, D), 0)
    pairs = []
    for _ in range(ncopy(cache_bytes)):
        kq, vq = c.mxtensor_empty(T * H, path.kv_lay, dev), c.mxtensor_empty(T * H, path.kv_lay, dev)
        c.mxs_quantize_act(path.KV[0], kq)
        c.mxs_quantize_act(path.KV[1], vq)
        pairs.append((kq, vq))
    calls = [lambda kq=kq, vq=vq: c.mxs_attn_decode(path.q, kq, vq, T, H, path.sm_scale, out=path.attn_out,
                                                    workspace=path.attn_ws) for kq, vq in pairs]
    t = measure("kv.mxs_attn_decode", calls, None, None)
    out["kv.mxs_attn_decode"] = (t * 1e6, path.work["kv.mxs_attn_decode"][1] / t / 1e9 / pk["hbm_gbs"])
    del pairs
    # the per-layer quantisers and the sensitivity on rotated source copies
    hbm = lambda name, t: (t * 1e6, path.work[name][1] / t / 1e9 / pk["hbm_gbs"])
    for L in path.layers:
        Wc = [L.W] + [L.W.clone() for _ in range(ncopy(L.W.numel() * 2) - 1)]
        name = f"{L.name}.mxs_quantize_weight"
        out[name] = hbm(name, measure(name, [lambda w=w: c.mxs_quantize_weight(w, L.Wq) for w in Wc], None, None))
        M = L.Ms[0]
        Ac = [L.A[M]] + [L.A[M].clone() for _ in range(ncopy(L.A[M].numel() * 2) - 1)]
        name = f"{L.name}.mxs_quantize_act_M{M}"
        out[name] = hbm(name, measure(name, [lambda x=x: c.mxs_quantize_act(x, L.Aq[M]) for x in Ac], None, None))
        Xc = [L.X] + [L.X.clone() for _ in range(ncopy(L.X.numel() * 2 + L.W.numel() * 2) - 1)]
        name = f"{L.name}.mxs_sensitivity"
        calls = [lambda x=x, w=w: c.mxs_sensitivity(x, w, workspace=L.sens_ws, out=(L.H, L.E, L.s))
                 for x, w in zip(Xc, (Wc * len(Xc))[:len(Xc)])]
        out[name] = hbm(name, measure(name, calls, None, None))
        del Wc, Ac, Xc
    c.mxs_sync()
    torch.cuda.empty_cache()
    return out


def run_e2e(path, args, dev, world):
    """Same metric through the C ABI with pinned host buffers: H2D of the
    step's inputs and D2H of its outputs inside the timed region.  The copies
    run on their own streams in the order the step consumes the inputs; each
    call waits only for the inputs it reads, and each output leaves as soon as
    it is written, so transfers overlap the kernels."""
    import torch
    dst = {}
    needs = {}
    for L in path.layers:
        dst[f"{L.name}.X"], dst[f"{L.name}.W"] = L.X, L.W
        needs[f"{L.name}.mxs_sensitivity"] = (f"{L.name}.X", f"{L.name}.W")
        needs[f"{L.name}.mxs_quantize_weight"] = (f"{L.name}.W",)
        for M in L.Ms:
            dst[f"{L.name}.A{M}"] = L.A[M]
            needs[f"{L.name}.mxs_quantize_act_M{M}"] = (f"{L.name}.A{M}",)
    for i in range(2):
        dst[f"kv.{'KV'[i]}"] = path.KV[i]
        needs[f"kv.mxs_quantize_act_{'KV'[i]}"] = (f"kv.{'KV'[i]}",)
    dst["kv.q"] = path.q
    needs["kv.mxs_attn_decode"] = ("kv.q",)
    host = {k: v.cpu().pin_memory() for k, v in dst.items()}
    outs = {}
    for L in path.layers:
        for M in L.Ms:
            outs[f"{L.name}.mxs_gemm_M{M}"] = (L.Y[M], torch.empty(L.Y[M].shape, dtype=L.Y[M].dtype).pin_memory())
    outs["kv.mxs_attn_decode"] = (path.attn_out, torch.empty(path.attn_out.shape, dtype=torch.float32).pin_memory())
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = sum(h.numel() * h.element_size() for _, h in outs.values())
    calls = path.calls()
    order = list(dst)                                   # the order the step consumes them
    main = torch.cuda.current_stream()
    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    steps = max(3, min(args.steps, 10))
    ms = []
    for i in range(steps + 1):
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record(main)
        up.wait_stream(main)
        landed = {}
        with torch.cuda.stream(up):
            for k in order:
                dst[k].copy_(host[k], non_blocking=True)
                landed[k] = torch.cuda.Event()
                landed[k].record(up)
        for name, fn in calls:
            for k in needs.get(name, ()):
                main.wait_event(landed[k])
            fn()
            if name in outs:
                down.wait_stream(main)
                with torch.cuda.stream(down):
                    outs[name][1].copy_(outs[name][0], non_blocking=True)
        main.wait_stream(down)
        main.wait_stream(up)
        e.record(main)
        torch.cuda.synchronize()
        if i:
            ms.append(s.elapsed_time(e))
    t = max_over_ranks(sum(ms) / len(ms) * 1e-3, world, dev)
    return {"value": job_tflops(path.gemm_flops, 1, world, t), "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": t * 1e3}


def _time_call(torch, call, flush, reps):
    """Median of `reps` CUDA-graph replays of one call, each after an L2 flush."""
    for _ in range(3):
        call()
    g = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream()
    with torch.cuda.graph(g, stream=cap):
        call()
    ev = []
    for _ in range(reps):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        g.replay()
        e1.record()
        ev.append((e0, e1))
    torch.cuda.synchronize()
    return statistics.median(a.elapsed_time(b) for a, b in ev) * 1e3


def l70_weight(inputs, torch, dev, layer, j):
    _, N, K = L70_SHAPES[j]
    return inputs.random_matrix(N, K, device=dev, seed=L70_SEED + 16 * layer + j, dtype=torch.bfloat16,
                                std=0.015, outlier_frac=0.02, outlier_scale=20.0)


def run_8b_stack(c, dev, torch, pk):
    """The Llama-3-8B-shaped stack under one budget: the sensitivities of all
    224 matrices (each generated on the device, scored on a 2048-row X of its
    input width, freed), one mxs_allocate call whose greedy spans the whole
    stack at 4.5 bits, then every matrix generated again from its seed and
    quantised into resident storage.  Reports the three phases' times (CUDA
    events around each call, summed; the allocation's host arithmetic and its
    one synchronisation included), the bits achieved and the bytes held."""
    from mx_microscaling_mixed_b200 import inputs
    X = {K: inputs.gaussian_acts(dev, L8_SEED - 1 - i, T_CAL, K) for i, K in enumerate((4096, 14336))}
    ev = lambda: torch.cuda.Event(enable_timing=True)
    mats = [(l, j, N, K) for l in range(L8_LAYERS) for j, (_, N, K) in enumerate(L8_SHAPES)]
    gen = lambda l, j, N, K: inputs.attn_weight(dev, L8_SEED + 16 * l + j, N, K)
    ss, marks = [], []
    for l, j, N, K in mats:
        W = gen(l, j, N, K)
        e0, e1 = ev(), ev()
        e0.record()
        _, _, s = c.mxs_sensitivity(X[K], W)
        e1.record()
        ss.append(s)
        marks.append((e0, e1))
        del W
    torch.cuda.synchronize()
    sens_ms = sum(a.elapsed_time(b) for a, b in marks)
    t0 = time.perf_counter()
    perms, counts = c.mxs_allocate(ss, [N for _, _, N, _ in mats], mode="budget", budget=BUDGET)
    torch.cuda.synchronize()
    alloc_ms = (time.perf_counter() - t0) * 1e3
    del ss
    store, qmarks = [], []
    for (l, j, N, K), perm, cnt in zip(mats, perms, counts):
        W = gen(l, j, N, K)
        Wq = c.mxtensor_empty(N, c.mxs_layout_make(K, cnt, perm), dev)
        e0, e1 = ev(), ev()
        e0.record()
        c.mxs_quantize_weight(W, Wq)
        e1.record()
        store.append(Wq)
        qmarks.append((e0, e1, N, tuple(cnt)))
        del W
    torch.cuda.synchronize()
    quant_ms = sum(a.elapsed_time(b) for a, b, _, _ in qmarks)
    q_bytes = sum(layout_bytes(N, cnt, 2) for _, _, N, cnt in qmarks)
    bits = sum(N * (8 * n8 + 6 * n6 + 4 * n4) for (_, _, N, _), (n8, n6, n4) in zip(mats, counts))
    elems = sum(N * K for _, _, N, K in mats)
    out = {"layers": L8_LAYERS, "matrices": len(mats), "weights": elems,
           "budget_bits": BUDGET[0] / BUDGET[1], "achieved_bits": bits / elems,
           "packed_bytes": sum(layout_bytes(N, cnt, 0) for _, _, N, cnt in qmarks),
           "sensitivity_ms_total": sens_ms,
           "sensitivity_gbs": sum(T_CAL * K * 2 + N * K * 2 for _, _, N, K in mats) / (sens_ms * 1e-3) / 1e9,
           "allocate_ms": alloc_ms, "quantize_weight_ms_total": quant_ms,
           "quantize_weight_gbs": q_bytes / (quant_ms * 1e-3) / 1e9,
           "quantize_weight_frac_hbm": q_bytes / (quant_ms * 1e-3) / 1e9 / pk["hbm_gbs"],
           "counts_layer0_n8_n6_n4": {name: list(counts[j]) for j, (name, _, _) in enumerate(L8_SHAPES)}}
    del store, X
    torch.cuda.empty_cache()
    return out


def run_70b_inplace(c, dev, path, torch, pk, reps=5):
    """The Llama-2-70B-shaped stack, all 80 layers' weights quantised in place:
    each matrix is generated on the device in bf16, its sensitivity taken on
    a 2048-row calibration X of its input width, its columns allocated at
    4.25 bits and the weight quantised into storage that stays resident,
    then the bf16 is freed.  Reports the per-call sensitivity and
    quantisation times summed over the 560 matrices, the packed bytes held,
    the prefill GEMM of layer 0's gate projection at M = 4096 (L2 flushed)
    and one decode step over the whole stack: per matrix a one-row
    activation quantisation and the M = 1 GEMM, 1120 launches in one CUDA
    graph, reading every packed weight once."""
    from mx_microscaling_mixed_b200 import inputs
    X = {K: inputs.gaussian_acts(dev, L70_SEED - 1 - i, T_CAL, K) for i, K in enumerate((8192, 28672))}
    ev = lambda: torch.cuda.Event(enable_timing=True)
    store, marks = [], []
    wbytes = sbytes = 0
    for layer in range(L70_LAYERS):
        for j, (name, N, K) in enumerate(L70_SHAPES):
            W = l70_weight(inputs, torch, dev, layer, j)
            e = [ev() for _ in range(3)]
            e[0].record()
            _, _, s = c.mxs_sensitivity(X[K], W)
            e[1].record()
            perms, counts = c.mxs_allocate([s], [N], mode="budget", budget=L70_BUDGET)
            lay = c.mxs_layout_make(K, counts[0], perms[0])
            Wq = c.mxtensor_empty(N, lay, dev)
            e2 = ev()
            e2.record()
            c.mxs_quantize_weight(W, Wq)
            e[2].record()
            marks.append((e[0], e[1], e2, e[2], N, K, tuple(counts[0])))
            store.append((name, N, K, lay, Wq, tuple(counts[0])))
            wbytes += layout_bytes(N, counts[0], 0)
            del W, s
    torch.cuda.synchronize()
    sens_ms = sum(a.elapsed_time(b) for a, b, _, _, _, _, _ in marks)
    quant_ms = sum(x.elapsed_time(y) for _, _, x, y, _, _, _ in marks)
    q_bytes = sum(layout_bytes(N, cnt, 2) for _, _, _, _, N, _, cnt in marks)
    s_bytes = sum(T_CAL * K * 2 + N * K * 2 for _, _, _, _, N, K, _ in marks)
    del X
    out = {"layers": L70_LAYERS, "matrices": len(store), "budget_bits": L70_BUDGET[0] / L70_BUDGET[1],
           "counts_n8_n6_n4": {f"K={K}": list(cnt) for _, _, K, _, _, cnt in store[:7]},
           "weights": sum(N * K for _, N, K, _, _, _ in store), "packed_bytes": wbytes,
           "device_bytes_peak": torch.cuda.max_memory_allocated(dev),
           "sensitivity_ms_total": sens_ms, "sensitivity_gbs": s_bytes / (sens_ms * 1e-3) / 1e9,
           "quantize_weight_ms_total": quant_ms, "quantize_weight_gbs": q_bytes / (quant_ms * 1e-3) / 1e9,
           "quantize_weight_frac_hbm": q_bytes / (quant_ms * 1e-3) / 1e9 / pk["hbm_gbs"],
           "timing": "calls in stream order with CUDA events around each, summed over the 560 matrices"}
    per = {}
    for (x0, x1, y0, y1, N, K, cnt), (name, *_rest) in zip(marks, store):
        d = per.setdefault(name, [0.0, 0.0, 0])
        d[0] += y0.elapsed_time(y1)
        d[1] += layout_bytes(N, cnt, 2)
        d[2] += 1
    out["quantize_weight_by_matrix"] = {n: {"ms": ms, "gbs": b / (ms * 1e-3) / 1e9,
                                            "frac_hbm": b / (ms * 1e-3) / 1e9 / pk["hbm_gbs"]}
                                        for n, (ms, b, _) in per.items()}
    # prefill: layer 0's gate projection at M = 4096
    _, N, K, lay, Wq, cnt = store[4]
    M = 4096
    Aq = c.mxtensor_empty(M, lay, dev)
    c.mxs_quantize_act(inputs.gaussian_acts(dev, L70_SEED - 3, M, K), Aq)
    ws = torch.empty(c.mxs_gemm_workspace_bytes(Aq, Wq) + 1024, dtype=torch.uint8, device=dev)
    Y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
    us = _time_call(torch, lambda: c.mxs_gemm(Aq, Wq, Y=Y, workspace=ws), path.flush, reps)
    out["gemm_gate_M4096"] = {"us": us, "tflops": 2 * M * N * K / us / 1e6,
                              "frac": gemm_roofline_s(M, N, cnt, pk) / (us * 1e-6)}
    del Aq, ws, Y
    # decode: every matrix once, one activation row each
    a1 = {K: inputs.gaussian_acts(dev, L70_SEED - 5 - i, 1, K) for i, K in enumerate((8192, 28672))}
    calls = []
    for _, N, K, lay, Wq, _ in store:
        Aq = c.mxtensor_empty(1, lay, dev)
        Y = torch.empty(1, N, dtype=torch.bfloat16, device=dev)
        calls.append((a1[K], Aq, Wq, Y))

    def step():
        for x, Aq, Wq, Y in calls:
            c.mxs_quantize_act(x, Aq)
            c.mxs_gemm(Aq, Wq, Y=Y)
    step()
    c.mxs_sync()
    g = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream()
    with torch.cuda.graph(g, stream=cap):
        step()
    times = []
    for _ in range(reps):
        e0, e1 = ev(), ev()
        e0.record()
        g.replay()
        e1.record()
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1))
    ms = statistics.median(times)
    out["decode_step_M1"] = {"ms": ms, "launches": 2 * len(calls), "w_bytes": wbytes,
                             "gbs": wbytes / (ms * 1e-3) / 1e9, "frac_hbm": wbytes / (ms * 1e-3) / 1e9 / pk["hbm_gbs"]}
    del g, calls, store
    c.mxs_sync()
    torch.cuda.empty_cache()
    return out


def run_mixed_overhead(c, dev, path, torch, reps=30):
    """What the wider blocks cost: mxs_gemm on each layer's weight under
    uniform MXINT4, the 32 fixed 8-bit columns alone (4 + 4*32/K bits) and the
    4.5-bit budget, at every M of the layer ([TS §4] estimates ~3% latency at
    ~4.03 bits)."""
    out = {"unit": "us", "reps": reps, "timing": "median of CUDA-graph replays, L2 flushed before each",
           "layers": {}}
    for L in path.layers:
        layouts = {"uniform4": ((0, 0, L.K), torch.arange(L.K, dtype=torch.int32, device=dev)),
                   "fixed8_only": None, "b4.5": (L.counts, L.perm)}
        perms, counts = c.mxs_allocate([L.s], [L.N], mode="budget", budget=(4 * L.K + 128, L.K))
        layouts["fixed8_only"] = (counts[0], perms[0])
        row = {"counts": {k: list(v[0]) for k, v in layouts.items()}, "us": {}, "overhead": {}}
        for M in L.Ms:
            for lname, (cnt, perm) in layouts.items():
                lay = c.mxs_layout_make(L.K, cnt, perm)
                Wq, Aq = c.mxtensor_empty(L.N, lay, dev), c.mxtensor_empty(M, lay, dev)
                c.mxs_quantize_weight(L.W, Wq)
                c.mxs_quantize_act(L.A[M], Aq)
                ws = torch.empty(c.mxs_gemm_workspace_bytes(Aq, Wq) + 1024, dtype=torch.uint8, device=dev)
                Y = torch.empty(M, L.N, dtype=torch.bfloat16, device=dev)
                row["us"][f"M{M}/{lname}"] = _time_call(torch, lambda: c.mxs_gemm(Aq, Wq, Y=Y, workspace=ws),
                                                        path.flush, reps)
                del Wq, Aq, ws, Y
            base = row["us"][f"M{M}/uniform4"]
            for lname in ("fixed8_only", "b4.5"):
                row["overhead"][f"M{M}/{lname}"] = row["us"][f"M{M}/{lname}"] / base - 1.0
        out["layers"][L.name] = row
    c.mxs_sync()
    return out


def run_budget_sweep(c, dev, path, torch, pk, reps=20):
    """Average-bit budget sweep ([TS §4] ablation, ~3.28 to 5.75 bits): the
    allocation's counts and the prefill mxs_gemm time of each layer at each
    budget; budgets below what the fixed 8-bit block costs are infeasible."""
    out = {"unit": "us", "reps": reps, "budgets": [f"{n}/{d}" for n, d in SWEEP_BUDGETS], "layers": {}}
    for L in path.layers:
        M = L.Ms[0]
        rows = []
        for num, den in SWEEP_BUDGETS:
            r = {"budget_bits": num / den}
            try:
                perms, counts = c.mxs_allocate([L.s], [L.N], mode="budget", budget=(num, den))
            except c.MxsError as e:
                r["status"] = c.mxs_status_str(e.status).split(":")[0]
                rows.append(r)
                continue
            cnt = counts[0]
            lay = c.mxs_layout_make(L.K, cnt, perms[0])
            Wq, Aq = c.mxtensor_empty(L.N, lay, dev), c.mxtensor_empty(M, lay, dev)
            c.mxs_quantize_weight(L.W, Wq)
            c.mxs_quantize_act(L.A[M], Aq)
            ws = torch.empty(c.mxs_gemm_workspace_bytes(Aq, Wq) + 1024, dtype=torch.uint8, device=dev)
            Y = torch.empty(M, L.N, dtype=torch.bfloat16, device=dev)
            us = _time_call(torch, lambda: c.mxs_gemm(Aq, Wq, Y=Y, workspace=ws), path.flush, reps)
            n8, n6, n4 = cnt
            r.update({"counts": list(cnt), "achieved_bits": (8 * n8 + 6 * n6 + 4 * n4) / L.K,
                      f"gemm_M{M}_us": us, "tflops": 2 * M * L.N * L.K / us / 1e6,
                      "roofline_frac": gemm_roofline_s(M, L.N, cnt, pk) / (us * 1e-6)})
            rows.append(r)
            del Wq, Aq, ws, Y
        out["layers"][L.name] = {"M": M, "rows": rows}
    c.mxs_sync()
    return out


# ----------------------------------------------------------- oracle (CPU) arm
class OraclePath:
    """The CPU oracle on a row sample of the same workload.  Every piece of the
    step is linear in the rows it processes, so a sample of fraction f is timed
    and scaled by 1/f (allocation, which sorts one vector, runs in full; the
    attention step runs on a token prefix of the cache)."""

    def __init__(self, seed, frac_hint=1.0 / 16):
        import numpy as np
        import torch
        import oracle
        from mx_microscaling_mixed_b200 import inputs
        self.np, self.o = np, oracle
        f64 = lambda t: t.float().numpy().astype(np.float64)
        self.layers = []
        for i, (name, N, K, kind, Ms) in enumerate(LAYERS):
            # the draws of the GPU arm, of which a sample of fraction <= 1/8 uses the leading rows
            W, X, A = _layer_inputs(inputs, "cpu", seed + 100 * i, name, N, K, kind, Ms)
            self.layers.append((name, N, K, Ms, f64(W[: N // 8]), f64(X[: T_CAL // 8]),
                                {M: f64(A[M][: max(1, M // 8)]) for M in Ms}))
        T, H, D = KV_SHAPE
        self.KV = [f64(inputs.kv_cache("cpu", seed + 10 + i, T // 8, H, D).reshape(-1, D)) for i in range(2)]
        self.q = f64(inputs.random_matrix(N_QH, D, device="cpu", seed=seed + 20, dtype=torch.bfloat16,
                                          outlier_frac=0.0))
        self.gemm_flops = sum(2 * M * N * K for _, N, K, Ms, *_ in self.layers for M in Ms)

    def step(self, frac):
        o = self.o
        rows = lambda n: max(1, int(round(n * frac)))
        t = {}
        for name, N, K, Ms, W, X, A in self.layers:
            tx, tw = rows(T_CAL), rows(N)
            t0 = time.perf_counter()
            _, _, s = o.sensitivity(X[:tx], W[:tw])
            t[f"{name}.sensitivity"] = (time.perf_counter() - t0) * ((T_CAL + N) / (tx + tw))
            t0 = time.perf_counter()
            perms, counts = o.allocate([s], [N], mode="budget", budget=BUDGET)
            t[f"{name}.allocate"] = time.perf_counter() - t0
            perm, counts = perms[0], counts[0]
            t0 = time.perf_counter()
            wc, ws = o.quantize_rows(W[:tw], perm, counts)
            t[f"{name}.quantize_weight"] = (time.perf_counter() - t0) * N / tw
            for M in Ms:
                m = rows(M)
                t0 = time.perf_counter()
                ac, as_ = o.quantize_rows(A[M][:m], perm, counts)
                t[f"{name}.quantize_act_M{M}"] = (time.perf_counter() - t0) * M / m
                t0 = time.perf_counter()
                o.gemm(ac, as_, wc, ws, counts)                   # m x tw block of Y
                t[f"{name}.gemm_M{M}"] = (time.perf_counter() - t0) * (M * N) / (m * tw)
        T, H, D = KV_SHAPE
        n_tok = rows(T)
        t0 = time.perf_counter()
        kv = [o.quantize_rows(x[: n_tok * H], None, (0, 0, D)) for x in self.KV]
        t["kv.quantize"] = (time.perf_counter() - t0) * T / n_tok
        t0 = time.perf_counter()
        o.attn_decode(self.q, kv[0][0][2], kv[0][1][2], kv[1][0][2], kv[1][1][2], n_tok, H, 1.0 / D ** 0.5)
        t["kv.attn_decode"] = (time.perf_counter() - t0) * T / n_tok
        return sum(t.values()), t


def run_reference(args, world):
    """The oracle as the reference arm: rank 0 only, host cores."""
    op = OraclePath(SEED)
    budget_s = 150.0 / max(1, args.steps + args.warmup)
    frac = 1.0 / 256
    t_probe = time.perf_counter()
    op.step(frac)
    dt = time.perf_counter() - t_probe
    frac = max(1.0 / 2048, min(1.0 / 8, frac * budget_s / max(dt, 1e-3)))
    for _ in range(args.warmup):
        op.step(frac)
    est = []
    for _ in range(args.steps):
        est.append(op.step(frac)[0])
    per_step = statistics.mean(est)
    value = op.gemm_flops / per_step / 1e12
    sample = (f"row fraction {frac:.5f} of every piece (X, W, A, K/V rows; GEMM on the sampled A x W block; "
              f"attention on a token prefix), time scaled by 1/fraction; allocation in full; single thread")
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": per_step * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)",
            "config": {"workload": WORKLOAD},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": 1, "kind": "oracle", "sample": sample,
                             **host_info()},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def cpu_baseline():
    """The oracle timed once on ~10-30 s of host work (rank 0, N=1 only)."""
    op = OraclePath(SEED)
    frac = 1.0 / 128
    total, parts = op.step(frac)
    return {"value": op.gemm_flops / total / 1e12, "unit": "TFLOP/s", "cores": 1, "kind": "oracle",
            "sample": f"row fraction {frac:.4f} of each piece of one step (sensitivity, quantisers, a "
                      f"{frac:.4f}-row x {frac:.4f}-row block of each GEMM, attention on a {frac:.4f} token prefix),"
                      f" scaled by 1/fraction; allocation in full; single-threaded C, fp64",
            "ms_per_step_extrapolated": total * 1e3, **host_info(),
            "parts_s": {k: round(v, 4) for k, v in parts.items()}}


# ------------------------------------------------------------ multi-process
def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def spawn_ranks(n: int, argv) -> int:
    """Relaunch this script under torch.distributed.run with n processes on
    this node (rendezvous on 127.0.0.1) and return its exit status; rank 0
    prints the JSON line."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr=127.0.0.1", f"--master-port={_free_port()}", os.path.abspath(__file__), *argv]
    return subprocess.call(cmd)


def probe_ranks(world, rank):
    """Launch check only (no GPU work): every rank joins the process group
    and contributes its rank; rank 0 prints what it saw."""
    import datetime
    import torch
    import torch.distributed as dist
    backend = "nccl" if torch.cuda.is_available() else "gloo"
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0"))) if backend == "nccl" else torch.device("cpu")
    if backend == "nccl":
        torch.cuda.set_device(dev)
    dist.init_process_group(backend, timeout=datetime.timedelta(seconds=60))
    t = torch.zeros(world, dtype=torch.float64, device=dev)
    t[rank] = rank + 1
    dist.all_reduce(t)
    job = max_over_ranks(0.1 * (rank + 1), world, dev)
    if rank == 0:
        print(json.dumps({"probe": "ranks", "n_gpus": world, "backend": backend,
                          "ranks_seen": [int(x) - 1 for x in t.tolist()], "max_over_ranks": job}), flush=True)
    dist.barrier()
    dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true", help="skip the mixed-overhead table and the budget sweep")
    ap.add_argument("--no-stream", action="store_true", help="skip the back-to-back per-call timing")
    ap.add_argument("--probe-ranks", action="store_true", help="launch check: join the process group and exit")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        sys.exit(spawn_ranks(args.gpus, sys.argv[1:]))
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.probe_ranks:
        probe_ranks(world, rank)
        return
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, world)), flush=True)
        return
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    line = run_gpu(args, rank, world, local_rank)
    if rank == 0:
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline()
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
