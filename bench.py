#!/usr/bin/env python
"""Benchmark of the MXSens mixed-width MXINT hot path on B200.

One STEP is one pass of the whole path over one synthetic Llama-3-8B-shaped
attention projection (W 4096x4096 bf16 with 3% Student-t(3) columns,
calibration X 2048x4096 bf16 with 8 outlier channels x50, average budget 4.5
bits) plus the K/V cache of the stack workload (8192 tokens x 8 heads x 128,
K and V):
  sensitivity(X, W) -> allocate (budget 4.5) -> quantize W ->
  for M in (2048, 16, 1): quantize A_M -> gemm(A_M, W)  ->  quantize K, V.
`value` = GEMM FLOPs of the step (2 M N K_real summed over the three M) per
second of whole-step time, all ranks; the per-kernel numbers and the roofline
of the dominant kernel are reported beside it.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

`--impl reference` times the CPU oracle (plain single-threaded C, fp64) on the
host cores instead, on a bounded row sample of the same workload per step.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

M_LIST = (2048, 16, 1)
N_OUT, K_IN, T_CAL = 4096, 4096, 2048
KV_SHAPE = (8192, 8, 128)
BUDGET = (9, 2)
SEED = 2000
CALL_REPS, CALL_TRIALS = 10, 5   # per-call timing: calls per graph, replays per graph
METRIC = "mxs_gemm TFLOP/s (% of roofline); MXINT quantize GB/s (% of HBM peak)"
WORKLOAD = ("llama3-8b attention projection: W 4096x4096 bf16 (3% t3 columns), calib X 2048x4096 bf16 "
            "(8 channels x50), budget 4.5 bits, GEMM M in {2048,16,1}; + K/V cache 8192x8x128 bf16 x2")


def peaks():
    p = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}
    try:
        m = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
        p.update({k: float(m[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")})
        p["source"] = "measured"
    except (OSError, KeyError, ValueError):
        pass
    # No measured FP8 figure: the block-scaled E4M3 peak is taken as 2x bf16
    # (the nominal dense ratio, 4.5 vs 2.25 PFLOP/s).
    p["fp8_tflops"] = 2.0 * p["bf16_tflops"]
    return p


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
class Path:
    """Device buffers and the step of the hot path (all kernels through the C ABI)."""

    def __init__(self, dev, seed):
        import torch
        from mx_microscaling_mixed_b200 import capi, inputs
        self.torch, self.c = torch, capi
        self.W = inputs.attn_weight(dev, seed, N_OUT, K_IN)
        self.X = inputs.gaussian_acts(dev, seed + 1, T_CAL, K_IN)
        self.A = {M: inputs.gaussian_acts(dev, seed + 2 + M, M, K_IN) for M in M_LIST}
        self.KV = [inputs.kv_cache(dev, seed + 10 + i, *KV_SHAPE).reshape(-1, KV_SHAPE[2]) for i in range(2)]
        c = capi
        self.sens_ws = torch.empty(c.mxs_sensitivity_workspace_bytes(T_CAL, N_OUT, K_IN) + 1024,
                                   dtype=torch.uint8, device=dev)
        self.H = torch.empty(K_IN, dtype=torch.float64, device=dev)
        self.E, self.s = torch.empty_like(self.H), torch.empty_like(self.H)
        self.perm = torch.empty(K_IN, dtype=torch.int32, device=dev)
        self.alloc_ws = torch.empty(1 << 20, dtype=torch.uint8, device=dev)
        c.mxs_sensitivity(self.X, self.W, workspace=self.sens_ws, out=(self.H, self.E, self.s))
        _, counts = c.mxs_allocate([self.s], [N_OUT], mode="budget", budget=BUDGET, perms=[self.perm],
                                   workspace=self.alloc_ws)
        self.counts = counts[0]
        self.lay = c.mxs_layout_make(K_IN, self.counts, self.perm)
        self.Wq = c.mxtensor_empty(N_OUT, self.lay, dev)
        self.Aq = {M: c.mxtensor_empty(M, self.lay, dev) for M in M_LIST}
        self.kv_lay = c.mxs_layout_make(KV_SHAPE[2], (0, 0, KV_SHAPE[2]))
        self.KVq = [c.mxtensor_empty(kv.shape[0], self.kv_lay, dev) for kv in self.KV]
        self.Y = {M: torch.empty(M, N_OUT, dtype=torch.bfloat16, device=dev) for M in M_LIST}
        c.mxs_quantize_weight(self.W, self.Wq)
        for M in M_LIST:
            c.mxs_quantize_act(self.A[M], self.Aq[M])
        gws = max(c.mxs_gemm_workspace_bytes(self.Aq[M], self.Wq) for M in M_LIST)
        self.gemm_ws = torch.empty(gws + 1024, dtype=torch.uint8, device=dev)
        self.flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
        self.flush_small = self.flush[: 256 << 20]          # per-call timing: twice the L2
        # algorithmic bytes / FLOPs per launch of each timed call
        n8, n6, n4 = self.counts
        self.work = {
            "mxs_sensitivity": ("GB/s", (T_CAL + N_OUT) * K_IN * 2),
            "mxs_allocate": ("GB/s", K_IN * 8 + K_IN * 4),
            "mxs_quantize_weight": ("GB/s", layout_bytes(N_OUT, self.counts, 2)),
            "mxs_quantize_kv0": ("GB/s", layout_bytes(KV_SHAPE[0] * KV_SHAPE[1], (0, 0, KV_SHAPE[2]), 2)),
            "mxs_quantize_kv1": ("GB/s", layout_bytes(KV_SHAPE[0] * KV_SHAPE[1], (0, 0, KV_SHAPE[2]), 2)),
        }
        for M in M_LIST:
            self.work[f"mxs_quantize_act_M{M}"] = ("GB/s", layout_bytes(M, self.counts, 2))
            self.work[f"mxs_gemm_M{M}"] = ("TFLOP/s", 2 * M * N_OUT * K_IN)
        self.gemm_flops = sum(2 * M * N_OUT * K_IN for M in M_LIST)

    def calls(self):
        """The step as (name, call) pairs in order; each call is one C-ABI entry point."""
        c = self.c

        def alloc():
            _, counts = c.mxs_allocate([self.s], [N_OUT], mode="budget", budget=BUDGET, perms=[self.perm],
                                       workspace=self.alloc_ws)
            assert counts[0] == self.counts
        out = [("mxs_sensitivity", lambda: c.mxs_sensitivity(self.X, self.W, workspace=self.sens_ws,
                                                               out=(self.H, self.E, self.s))),
               ("mxs_allocate", alloc),
               ("mxs_quantize_weight", lambda: c.mxs_quantize_weight(self.W, self.Wq))]
        for M in M_LIST:
            out.append((f"mxs_quantize_act_M{M}", lambda M=M: c.mxs_quantize_act(self.A[M], self.Aq[M])))
            out.append((f"mxs_gemm_M{M}", lambda M=M: c.mxs_gemm(self.Aq[M], self.Wq, Y=self.Y[M],
                                                                 workspace=self.gemm_ws)))
        for i in range(2):
            out.append((f"mxs_quantize_kv{i}", lambda i=i: c.mxs_quantize_act(self.KV[i], self.KVq[i])))
        return out

    def step(self):
        for _, fn in self.calls():
            fn()


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


def traffic_from_profile(pk_name: str):
    """dram bytes per launch recorded in profiles/, if the kernel source is unchanged since."""
    prof = os.path.join(ROOT, "profiles", pk_name)
    try:
        text = open(prof).read()
    except OSError:
        return None
    m = re.search(r"dram_bytes_per_call:\s*([0-9.eE+]+)", text)
    h = re.search(r"source_sha256:\s*([0-9a-f]{64})", text)
    if not m or not h:
        return None
    src = os.path.join(ROOT, "mx_microscaling_mixed_b200", "csrc", "mxs_gemm.cu")
    if hashlib.sha256(open(src, "rb").read()).hexdigest() != h.group(1):
        return None
    return float(m.group(1))


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
    for _ in range(args.warmup):
        path.flush.zero_()
        path.step()
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

    def timed(g):
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        g.replay()
        e.record()
        return s, e

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

    kernels = {}
    for name, per in per_call.items():
        unit, work = path.work[name]
        ach = work / per / (1e12 if unit == "TFLOP/s" else 1e9)
        kd = {"us": per * 1e6, "achieved": ach, "unit": unit, "share": per / call_sum}
        if unit == "GB/s":
            kd["frac_hbm"] = ach / pk["hbm_gbs"]
            kd["frac_nominal_8tbs"] = ach / 8000.0
        else:
            M = int(name.split("M")[-1])
            rt = gemm_roofline_s(M, N_OUT, path.counts, pk)
            kd["roofline_us"] = rt * 1e6
            kd["frac"] = rt / per
        kernels[name] = kd
    # the dominant kernel: the prefill GEMM
    g = kernels["mxs_gemm_M2048"]
    rt = g["roofline_us"] * 1e-6
    roof = {"kernel": "mxs_gemm M=2048 (one call: gemm_stage_kernel + gemm_tc2_kernel)", "bound": "tensor",
            "achieved": g["achieved"], "peak": 2 * 2048 * N_OUT * K_IN / rt / 1e12, "unit": "TFLOP/s",
            "frac": g["frac"], "traffic": traffic_from_profile("gemm_attn_prefill_M2048.md"),
            "peak_basis": f"4-bit segment at 2x measured bf16 ({pk['fp8_tflops']:.0f} TFLOP/s, no measured fp8), "
                          f"6/8-bit at measured bf16 ({pk['bf16_tflops']:.0f}); of {pk['source']}"}

    e2e = run_e2e(path, args, dev, world)
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total_s / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "mxint4/6/8 codes; e4m3+bf16 MMA, f32 acc",
        "data": "synthetic (seeded; shapes and outlier structure of the workload)",
        "config": {"workload": WORKLOAD, "counts_n8_n6_n4": list(path.counts), "l2": "flushed between steps "
                   "(512 MB write outside the step events)", "parallelism": f"replicas x{world} (no data-path collective)",
                   "timing": "step = one CUDA graph of all C-ABI calls, replayed per step between CUDA events; "
                             f"kernels{{}}: per call, (graph of {CALL_REPS} x [L2 flush, call]) - (graph of "
                             f"{CALL_REPS} flushes), best of {CALL_TRIALS} replays each, / {CALL_REPS}; cold L2 per call",
                   "launches_per_step": launches_per_step},
        "roofline": roof, "kernels": kernels, "e2e": e2e, "gpu_launches": launches,
        "clocks": clocks.summary(), "wall_s_timed_region": wall,
    }
    return line


def run_e2e(path, args, dev, world):
    """Same metric through the C ABI with pinned host buffers: H2D of the
    step's inputs and D2H of its outputs inside the timed region.  The copies
    run on their own streams in the order the step consumes the inputs; each
    call waits only for the inputs it reads, and each GEMM's output leaves as
    soon as it is written, so transfers overlap the kernels."""
    import torch
    host = {"X": path.X.cpu().pin_memory(), "W": path.W.cpu().pin_memory(),
            **{f"A{M}": path.A[M].cpu().pin_memory() for M in M_LIST},
            **{f"KV{i}": path.KV[i].cpu().pin_memory() for i in range(2)}}
    dst = {"X": path.X, "W": path.W, **{f"A{M}": path.A[M] for M in M_LIST},
           **{f"KV{i}": path.KV[i] for i in range(2)}}
    outs = {M: torch.empty(path.Y[M].shape, dtype=torch.bfloat16).pin_memory() for M in M_LIST}
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = sum(t.numel() * t.element_size() for t in outs.values())
    # inputs each call reads (the rest read only device results of earlier calls)
    needs = {"mxs_sensitivity": ("X", "W"), "mxs_quantize_weight": ("W",),
             **{f"mxs_quantize_act_M{M}": (f"A{M}",) for M in M_LIST},
             **{f"mxs_quantize_kv{i}": (f"KV{i}",) for i in range(2)}}
    calls = path.calls()
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
            for k in ("X", "W", *[f"A{M}" for M in M_LIST], "KV0", "KV1"):
                dst[k].copy_(host[k], non_blocking=True)
                landed[k] = torch.cuda.Event()
                landed[k].record(up)
        for name, fn in calls:
            for k in needs.get(name, ()):
                main.wait_event(landed[k])
            fn()
            if name.startswith("mxs_gemm_M"):
                M = int(name[len("mxs_gemm_M"):])
                down.wait_stream(main)
                with torch.cuda.stream(down):
                    outs[M].copy_(path.Y[M], non_blocking=True)
        main.wait_stream(down)
        main.wait_stream(up)
        e.record(main)
        torch.cuda.synchronize()
        if i:
            ms.append(s.elapsed_time(e))
    t = max_over_ranks(sum(ms) / len(ms) * 1e-3, world, dev)
    return {"value": job_tflops(path.gemm_flops, 1, world, t), "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": t * 1e3}


# ----------------------------------------------------------- oracle (CPU) arm
class OraclePath:
    """The CPU oracle on a row sample of the same workload.  Every piece of the
    step is linear in the rows it processes, so a sample of fraction f is timed
    and scaled by 1/f (allocation, which sorts one vector, runs in full)."""

    def __init__(self, seed):
        import numpy as np
        import torch
        import oracle
        from mx_microscaling_mixed_b200 import inputs
        self.np, self.o = np, oracle
        f64 = lambda t: t.float().numpy().astype(np.float64)
        self.W = f64(inputs.attn_weight("cpu", seed, N_OUT, K_IN))
        self.X = f64(inputs.gaussian_acts("cpu", seed + 1, T_CAL, K_IN))
        self.A = {M: f64(inputs.gaussian_acts("cpu", seed + 2 + M, M, K_IN)) for M in M_LIST}
        self.KV = [f64(inputs.kv_cache("cpu", seed + 10 + i, *KV_SHAPE).reshape(-1, KV_SHAPE[2])) for i in range(2)]
        self.gemm_flops = sum(2 * M * N_OUT * K_IN for M in M_LIST)
        _, _, s = oracle.sensitivity(self.X[:256], self.W[:256])
        self.perm, self.counts = None, None

    def step(self, frac):
        o, np = self.o, self.np
        rows = lambda n: max(1, int(round(n * frac)))
        t = {}
        tx, tw = rows(T_CAL), rows(N_OUT)
        t0 = time.perf_counter()
        _, _, s = o.sensitivity(self.X[:tx], self.W[:tw])
        t["sensitivity"] = (time.perf_counter() - t0) * ((T_CAL + N_OUT) / (tx + tw))
        t0 = time.perf_counter()
        perms, counts = o.allocate([s], [N_OUT], mode="budget", budget=BUDGET)
        t["allocate"] = time.perf_counter() - t0
        perm, counts = perms[0], counts[0]
        t0 = time.perf_counter()
        wc, ws = o.quantize_rows(self.W[:tw], perm, counts)
        t["quantize_weight"] = (time.perf_counter() - t0) * N_OUT / tw
        for M in M_LIST:
            m = rows(M)
            t0 = time.perf_counter()
            ac, as_ = o.quantize_rows(self.A[M][:m], perm, counts)
            t[f"quantize_act_M{M}"] = (time.perf_counter() - t0) * M / m
            t0 = time.perf_counter()
            o.gemm(ac, as_, wc, ws, counts)                   # m x tw block of Y
            t[f"gemm_M{M}"] = (time.perf_counter() - t0) * (M * N_OUT) / (m * tw)
        n_kv = rows(KV_SHAPE[0] * KV_SHAPE[1])
        t0 = time.perf_counter()
        for kv in self.KV:
            o.quantize_rows(kv[:n_kv], None, (0, 0, KV_SHAPE[2]))
        t["quantize_kv"] = (time.perf_counter() - t0) * (KV_SHAPE[0] * KV_SHAPE[1]) / n_kv
        return sum(t.values()), t


def run_reference(args, world):
    """The oracle as the reference arm: rank 0 only, host cores."""
    op = OraclePath(SEED)
    budget_s = 150.0 / max(1, args.steps + args.warmup)
    frac = 1.0 / 64
    t_probe = time.perf_counter()
    op.step(frac)
    dt = time.perf_counter() - t_probe
    frac = max(1.0 / 512, min(1.0 / 8, frac * budget_s / max(dt, 1e-3)))
    for _ in range(args.warmup):
        op.step(frac)
    est = []
    for _ in range(args.steps):
        est.append(op.step(frac)[0])
    per_step = statistics.mean(est)
    value = op.gemm_flops / per_step / 1e12
    sample = (f"row fraction {frac:.5f} of every piece (X, W, A, K/V rows; GEMM on the sampled A x W block), "
              f"time scaled by 1/fraction; allocation in full; single thread")
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": per_step * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)",
            "config": {"workload": WORKLOAD},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": 1, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def cpu_baseline():
    """The oracle timed once on ~10-30 s of host work (rank 0, N=1 only)."""
    op = OraclePath(SEED)
    frac = 1.0 / 32
    total, parts = op.step(frac)
    return {"value": op.gemm_flops / total / 1e12, "unit": "TFLOP/s", "cores": 1, "kind": "oracle",
            "sample": f"row fraction {frac:.4f} of each piece of one step (sensitivity, quantisers, a "
                      f"{frac:.4f}-row x {frac:.4f}-row block of each GEMM), scaled by 1/fraction; allocation "
                      f"in full; single-threaded C, fp64",
            "ms_per_step_extrapolated": total * 1e3,
            "parts_s": {k: round(v, 4) for k, v in parts.items()}}


def run_mixed_overhead(args):
    """Time mxs_gemm on one weight under three layouts -- uniform MXINT4, the
    32 fixed 8-bit columns alone (budget 4.03125 bits) and the 4.5-bit budget
    -- to measure what the wider blocks cost (the pages estimate ~3% at
    ~4.03 bits).  CUDA-graph replays of one call, L2 flushed before each,
    CUDA events around each replay."""
    import torch
    from mx_microscaling_mixed_b200 import build
    build.build()
    from mx_microscaling_mixed_b200 import capi as c, inputs
    dev = torch.device("cuda", 0)
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
    reps = max(10, min(args.steps, 100))
    out = {"metric": "mxs_gemm time by layout", "unit": "us", "reps": reps, "shapes": []}
    for (N, K) in ((4096, 4096), (14336, 4096)):
        W = inputs.attn_weight(dev, SEED, N, K)
        X = inputs.gaussian_acts(dev, SEED + 1, T_CAL, K)
        _, _, s = c.mxs_sensitivity(X, W)
        layouts = {"uniform4": ((0, 0, K), torch.arange(K, dtype=torch.int32, device=dev))}
        for name, budget in (("b4.03125", (129, 32)), ("b4.5", (9, 2))):
            perms, counts = c.mxs_allocate([s], [N], mode="budget", budget=budget)
            layouts[name] = (counts[0], perms[0])
        row = {"N": N, "K": K, "counts": {k: list(v[0]) for k, v in layouts.items()}, "us": {}}
        for M in M_LIST:
            A = inputs.gaussian_acts(dev, SEED + 2 + M, M, K)
            for name, (counts, perm) in layouts.items():
                lay = c.mxs_layout_make(K, counts, perm)
                Wq, Aq = c.mxtensor_empty(N, lay, dev), c.mxtensor_empty(M, lay, dev)
                c.mxs_quantize_weight(W, Wq)
                c.mxs_quantize_act(A, Aq)
                ws = torch.empty(c.mxs_gemm_workspace_bytes(Aq, Wq) + 1024, dtype=torch.uint8, device=dev)
                Y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
                call = lambda: c.mxs_gemm(Aq, Wq, Y=Y, workspace=ws)
                for _ in range(3):
                    call()
                g = torch.cuda.CUDAGraph()
                cap = torch.cuda.Stream()
                with torch.cuda.graph(g, stream=cap):
                    call()
                ms = []
                for _ in range(reps):
                    flush.zero_()
                    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    e0.record()
                    g.replay()
                    e1.record()
                    ms.append((e0, e1))
                torch.cuda.synchronize()
                row["us"][f"M{M}/{name}"] = statistics.median(a.elapsed_time(b) for a, b in ms) * 1e3
            base = row["us"][f"M{M}/uniform4"]
            for name in ("b4.03125", "b4.5"):
                row["us"][f"M{M}/{name}/overhead"] = row["us"][f"M{M}/{name}"] / base - 1.0
        out["shapes"].append(row)
    c.mxs_sync()
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--mixed-overhead", action="store_true",
                    help="time mxs_gemm under uniform-4-bit vs mixed layouts and exit")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", str(args.gpus if args.gpus == 1 else 1)))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.mixed_overhead:
        print(json.dumps(run_mixed_overhead(args)), flush=True)
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
