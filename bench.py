#!/usr/bin/env python
"""Benchmark of the routed NVFP4 MoE site on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload decode_t1]

One step = one routed MoE site forward (router logits, sigmoid top-k, routing
plan, expert gate/up + clamped SwiGLU, expert down x routing weight, BF16
shared expert, combine) over one batch of synthetic inputs already resident in
HBM, replayed from a CUDA graph of the public moe_forward call. L2 is flushed
(a 2x-L2 buffer is read) before every timed step; each step is timed
with CUDA events on the launching stream; the reported time is the max over
ranks. The roofline of the dominant kernel comes from stage events recorded
by the library inside the same graph: the expert GEMVs against HBM bandwidth
on decode workloads (decode_t*), the tcgen05 FP4 grouped GEMMs against the
dense FP4 tensor peak on prefill workloads (prefill_t4096, stress_t16384).

`e2e` measures the same metric through moe_forward with host buffers: pinned
host->device copy of x, the forward, device->host copy of y, all inside the
events.

Multi-GPU: the site does not shard here (replicas only): every rank runs its
own independent replica, value = all ranks' tokens / max-over-ranks time.

--impl reference times the CPU oracle (the deliberately plain fp64 restatement)
on the host cores for the same workload and prints the same JSON line.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE-layer tokens/s and achieved HBM GB/s (decode) / FP4 TFLOP/s (prefill) vs roofline"
FP4_PER_BF16 = 4.0     # nominal dense FP4 / BF16 tensor throughput ratio of B200 (9 / 2.25 PFLOP/s)
PER_EXPERT_NOTE = "gate+up+down codes, E4M3 scales and tensor scales of each touched expert"


def nvfp4_bank_bytes(rows: int, cols: int) -> int:
    return rows * cols // 2 + rows * cols // 16 + 4


def expert_bytes(wl) -> int:
    return 2 * nvfp4_bank_bytes(wl.I, wl.H) + nvfp4_bank_bytes(wl.H, wl.I)


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm_gbs=d["hbm_gbs"], bf16_tflops=d["bf16_tflops"],
                    bf16_tflops_sustained=d.get("bf16_tflops_sustained"), source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0, source="fallback")


# ------------------------------------------------------------------ clocks

class NvmlClocks:
    """SM clock and clock-event reasons read through NVML between timed steps
    (inside the timed loop, outside the CUDA-event intervals)."""
    BITS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown", 0x4: "sw_power_cap"}

    def __init__(self, gpu_index: int):
        import pynvml
        self.nv = pynvml
        pynvml.nvmlInit()
        self.h = pynvml.nvmlDeviceGetHandleByIndex(gpu_index)
        self.sm, self.reasons = [], set()
        self.max = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)

    def sample(self):
        nv = self.nv
        self.sm.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
        get = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or nv.nvmlDeviceGetCurrentClocksThrottleReasons
        bits = get(self.h)
        for b, name in self.BITS.items():
            if bits & b:
                self.reasons.add(name)

    def result(self):
        if not self.sm:
            return None
        return {"sm_mhz": statistics.median(self.sm), "sm_max_mhz": self.max, "reasons": sorted(self.reasons),
                "samples": len(self.sm), "source": "nvml, sampled after every timed step"}


def clock_sampler(gpu_index: int):
    try:
        return NvmlClocks(gpu_index)
    except Exception:          # no NVML: fall back to the nvidia-smi poller
        return ClockSampler(gpu_index)


class ClockSampler:
    """nvidia-smi clock / throttle sampling during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.lines: list[str] = []

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                                          "-lms", "100", "-i", str(self.idx)], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
        except (FileNotFoundError, OSError):
            self.proc = None
            return
        self.t = threading.Thread(target=self._read, daemon=True)
        self.t.start()

    def _read(self):
        for ln in self.proc.stdout:
            self.lines.append(ln.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.t.join(timeout=2)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [v.strip() for v in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------ ours

def decode_mma(wl) -> bool:
    """The tensor-core decode expert kernels run for this workload; mirrors
    the library's eligibility rule (a handful of tokens, shapes that stage in
    shared memory)."""
    if wl.kind != "decode" or not (1 <= wl.T <= 8):
        return False
    if wl.H % 1024 or wl.H > 8192 or wl.I % 128 or wl.I > 2048 or wl.k > 16 or wl.E > 1024 or wl.T * wl.k > 128:
        return False
    budget = 200 * 1024
    gu = ((wl.T * (wl.H + 8) * 2 + 15) // 16) * 16 + 2 * 4 * 4 * 256 * 4
    dn = wl.T * wl.k * (wl.I + 8) * 2
    return gu <= budget and dn <= budget


def measure(wl, args, rank, world, local_rank, dev, clocks=None):
    """Time one workload: K replays of the forward's CUDA graph (the value),
    interleaved with K replays of the same forward with events around the
    dominant kernels (their live duration, for the roofline). Returns the
    per-rank numbers (max over ranks taken by the caller)."""
    import torch
    from routed_nvfp4_expert_b200 import capi
    from routed_nvfp4_expert_b200 import synthetic as syn

    inp = syn.make_site(wl, seed=0)
    site = capi.site_to_device(inp, dev)
    cfg = capi.config_for(wl)
    if wl.kind == "decode":
        path = capi.PATH_DECODE
    else:
        path = capi.PATH_PREFILL_W4A16 if getattr(args, "prefill_path", "w4a4") == "w4a16" else capi.PATH_PREFILL
    prefill = path != capi.PATH_DECODE
    T, H = wl.T, wl.H
    # the block-scale atoms of the grouped GEMMs (prefill, and decode batches
    # of 9 or more tokens): weight preparation, once, outside the timed region
    capi.moe_prepare_weights(cfg, site)

    # rotating activations: a different routing every step (seeded per rank)
    n_x = 4 if prefill else 16
    x_pool = torch.stack([capi.bf16_tensor(syn.random_x(wl, T, seed=1000 * rank + i), dev) for i in range(n_x)])
    x = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
    y = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
    ws = capi.alloc_workspace(cfg, T, path, dev)
    views = capi.moe_workspace_views(cfg, T, path, ws)
    ids_view = capi.view_tensor(views.ids, (T, wl.k), torch.int32, dev)

    # L2 flush between timed steps: READ a buffer of 2x L2 plus margin. A
    # write-based flush leaves ~L2-size of dirty lines whose write-back then
    # lands inside the next timed kernel; reading evicts with clean lines.
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush = torch.zeros((2 * l2 + (64 << 20)) // 8, dtype=torch.int64, device=dev)
    flush_sink = torch.zeros((), dtype=torch.int64, device=dev)

    stream = torch.cuda.Stream(dev)
    nst = len(capi.STAGES) + 1
    ev = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(nst)]
    outer = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    with torch.cuda.stream(stream):
        for e in ev + outer:
            e.record(stream)               # creates the CUDA events
    stream.synchronize()
    w_c = site.c()
    i_gu, i_sh = capi.STAGES.index("expert_gate_up"), capi.STAGES.index("shared")
    i_hq, i_dn = capi.STAGES.index("h_quant"), capi.STAGES.index("expert_down")
    # intervals of the dominant kernels: decode = both expert launches
    # (adjacent); prefill = the two grouped GEMMs (the h encoding between them
    # excluded)
    spans = [(i_gu, i_hq), (i_dn, i_sh)] if prefill else [(i_gu, i_sh)]

    # warm the kernels once outside capture, then capture the forward into graphs:
    #   plain: the forward as a user runs it (no stage events) -- the value;
    #   timed: stage events only around the dominant kernels (an event node
    #   between two kernels also ends their launch overlap) -- the roofline;
    #   stages: every stage boundary (diagnostic)
    x.copy_(x_pool[0])
    with torch.cuda.stream(stream):
        capi.moe_forward(cfg, site, x, path, y, ws, stream=stream, w_c=w_c)
    stream.synchronize()
    capi.moe_read_device_status(ws, stream)

    def capture(events):
        g = torch.cuda.CUDAGraph()
        capi.moe_set_stage_events(events)
        try:
            with torch.cuda.graph(g, stream=stream):
                capi.moe_forward(cfg, site, x, path, y, ws, stream=stream, w_c=w_c)
        finally:
            capi.moe_set_stage_events(None)
        return g

    sparse = [None] * nst
    for a_, b_ in spans:
        sparse[a_], sparse[b_] = ev[a_], ev[b_]
    g_timed = capture(sparse)
    g_plain = capture(None)
    g_stages = capture(ev)

    def one_step(g, i, with_stages=False):
        with torch.cuda.stream(stream):
            torch.sum(flush, dim=0, out=flush_sink)
            x.copy_(x_pool[i % n_x])
            outer[0].record(stream)
            g.replay()
            outer[1].record(stream)
        stream.synchronize()
        step = outer[0].elapsed_time(outer[1])
        if with_stages == "all":
            return step, [ev[s].elapsed_time(ev[s + 1]) for s in range(nst - 1)]
        if with_stages:
            return step, sum(ev[a_].elapsed_time(ev[b_]) for a_, b_ in spans)
        return step, None

    for i in range(args.warmup):
        one_step(g_plain, i)
        one_step(g_timed, i, True)
    capi.moe_read_device_status(ws, stream)

    dist_barrier(world)
    torch.cuda.synchronize(dev)
    # K steps of the plain forward (the value) interleaved with K steps of the
    # forward with events around the dominant kernels (their live duration)
    step_ms, timed_ms, kern_ms_l, uniq = [], [], [], []
    for i in range(args.steps):
        step_ms.append(one_step(g_plain, args.warmup + i)[0])
        ms_t, gm = one_step(g_timed, args.warmup + i, True)
        timed_ms.append(ms_t)
        kern_ms_l.append(gm)
        if isinstance(clocks, NvmlClocks):
            clocks.sample()
        uniq.append(int(torch.unique(ids_view).numel()))
    torch.cuda.synchronize(dev)
    dist_barrier(world)
    capi.moe_read_device_status(ws, stream)

    # diagnostics (outside the timed region): every stage
    stage_ms = [one_step(g_stages, i, "all")[1] for i in range(min(args.steps, 10))]

    # e2e: the public call with host buffers (pinned), copies inside the events
    xh = torch.empty((T, H), dtype=torch.bfloat16, pin_memory=True)
    yh = torch.empty((T, H), dtype=torch.bfloat16, pin_memory=True)
    xh_pool = [x_pool[i].cpu() for i in range(n_x)]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_ms = []
    for i in range(args.warmup + args.steps):
        xh.copy_(xh_pool[i % n_x])
        with torch.cuda.stream(stream):
            torch.sum(flush, dim=0, out=flush_sink)
            e0.record(stream)
            x.copy_(xh, non_blocking=True)
            capi.moe_forward(cfg, site, x, path, y, ws, stream=stream, w_c=w_c)
            yh.copy_(y, non_blocking=True)
            e1.record(stream)
        stream.synchronize()
        if i >= args.warmup:
            e2e_ms.append(e0.elapsed_time(e1))
    capi.moe_read_device_status(ws, stream)
    res = dict(wl=wl, inp=inp, prefill=prefill, w4a16=path == capi.PATH_PREFILL_W4A16, ms=float(np.mean(step_ms)), timed_ms=float(np.mean(timed_ms)),
               kern_ms=float(np.mean(kern_ms_l)), e2e_ms=float(np.mean(e2e_ms)),
               stage_avg=np.mean(np.array(stage_ms), axis=0), U=float(np.mean(uniq)), n_spans=len(spans))
    del g_timed, g_plain, g_stages
    return res


def measure_dense(wl, args, rank, world, local_rank, dev, clocks=None):
    """Time the dense BF16 FFN (dense_ffn_bf16) at hidden H, intermediate
    dense_I over T tokens: K replays of its CUDA graph, L2 flushed before each."""
    import torch
    from routed_nvfp4_expert_b200 import capi
    from routed_nvfp4_expert_b200 import synthetic as syn

    d = syn.make_dense(wl)
    T, H, I = wl.T, wl.H, wl.dense_I
    wg, wu, wd = (capi.bf16_tensor(d[f"dense_{n}"], dev) for n in ("gate", "up", "down"))
    x_pool = torch.stack([capi.bf16_tensor(syn.random_x(wl, T, seed=1000 * rank + i), dev) for i in range(4)])
    x = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
    y = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
    ws = torch.empty(capi.dense_ffn_workspace_size(H, I, T), dtype=torch.uint8, device=dev)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush = torch.zeros((2 * l2 + (64 << 20)) // 8, dtype=torch.int64, device=dev)
    flush_sink = torch.zeros((), dtype=torch.int64, device=dev)
    stream = torch.cuda.Stream(dev)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    x.copy_(x_pool[0])
    with torch.cuda.stream(stream):
        capi.dense_ffn_bf16(wl.limit, x, wg, wu, wd, y, ws, stream=stream)
    stream.synchronize()
    capi.moe_read_device_status(ws, stream)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        capi.dense_ffn_bf16(wl.limit, x, wg, wu, wd, y, ws, stream=stream)

    def one(i):
        with torch.cuda.stream(stream):
            torch.sum(flush, dim=0, out=flush_sink)
            x.copy_(x_pool[i % 4])
            ev[0].record(stream)
            g.replay()
            ev[1].record(stream)
        stream.synchronize()
        return ev[0].elapsed_time(ev[1])

    for i in range(args.warmup):
        one(i)
    dist_barrier(world)
    ms = []
    for i in range(args.steps):
        ms.append(one(args.warmup + i))
        if isinstance(clocks, NvmlClocks):
            clocks.sample()
    dist_barrier(world)
    capi.moe_read_device_status(ws, stream)
    del g
    return dict(wl=wl, ms=float(np.mean(ms)))


def dense_line(res, pk, world):
    wl = res["wl"]
    T, H, I = wl.T, wl.H, wl.dense_I
    ms = res["ms"]
    flops = 2.0 * T * 3 * H * I
    if T >= 128:
        achieved = flops / (ms * 1e-3) / 1e12
        roof = {"bound": "tensor", "kernel": "bf16_gemm_kernel (tcgen05 kind::f16; gate/up + down launches)",
                "achieved": round(achieved, 1), "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                "frac": round(achieved / pk["bf16_tflops"], 4), "peak_source": f"{pk['source']} bf16 burst",
                "algorithmic_flops_per_step": flops, "traffic": None}
    else:
        nbytes = 3 * H * I * 2
        achieved = nbytes / (ms * 1e-3) / 1e9
        roof = {"bound": "hbm", "kernel": "bf16_gemv_kernel (gate/up + down launches)", "achieved": round(achieved, 1),
                "peak": pk["hbm_gbs"], "unit": "GB/s", "frac": round(achieved / pk["hbm_gbs"], 4),
                "peak_source": pk["source"], "algorithmic_bytes_per_step": nbytes, "traffic": None}
    return {"workload": wl.name, "T": T, "hidden": H, "intermediate": I, "value": round(world * T / (ms * 1e-3), 2),
            "unit": "tokens/s", "ms_per_step": round(ms, 5), "roofline": roof}


def decode_grouped(wl) -> bool:
    """Decode batches of 9 or more tokens run their experts on the grouped
    W4A16 GEMM (the weights' scale atoms are prepared); mirrors the library's
    rule."""
    return wl.kind == "decode" and wl.T >= 9 and wl.I % 128 == 0 and wl.H % 256 == 0


def roofline_of(res, pk):
    """The dominant kernels' roofline from measure()'s kernel time."""
    wl = res["wl"]
    T, H = wl.T, wl.H
    if res["prefill"]:
        flops = 2.0 * T * wl.k * 3 * H * wl.I          # gate + up + down over the T*k assignments
        achieved = flops / (res["kern_ms"] * 1e-3) / 1e12
        if res.get("w4a16"):
            # kind::f16 tensor math (f16 operands): the measured bf16 peak is the roof
            peak, src = pk["bf16_tflops"], f"{pk['source']} bf16 burst (f16 operands, same rate)"
            kernel, stem = "w4a16_gemm_kernel (tcgen05 kind::f16; gate/up + down launches)", "w4a16_grouped_gemm"
        else:
            peak = pk["bf16_tflops"] * FP4_PER_BF16
            src = f"{pk['source']} bf16 burst x nominal FP4/BF16 ratio {FP4_PER_BF16:g}"
            kernel, stem = "nvfp4_grouped_gemm (tcgen05 mxf4nvf4; gate/up + down launches)", "nvfp4_grouped_gemm"
        return {"bound": "tensor", "kernel": kernel, "achieved": round(achieved, 1), "peak": round(peak, 1),
                "unit": "TFLOP/s", "frac": round(achieved / peak, 4), "peak_source": src,
                "algorithmic_flops_per_step": flops, "unique_experts_per_step": res["U"],
                "traffic": read_traffic_profile(f"{stem}_{wl.name}")}
    routed = res["U"] * expert_bytes(wl)
    if decode_mma(wl):
        kernel = "mma_gate_up_kernel + mma_down_bulk_kernel (register-ring and bulk-copy weight streams, mma.sync m16n8k16; timed together)"
    elif decode_grouped(wl):
        kernel = ("w4a16_gemm_kernel (grouped W4A16 GEMM, tcgen05 kind::f16, padding halves skipped; "
                  "gate/up + down launches, timed together)")
    else:
        kernel = "nvfp4_expert_gemv (gate/up + down launches, timed together)"
    achieved = routed / (res["kern_ms"] * 1e-3) / 1e9
    return {"bound": "hbm", "kernel": kernel, "achieved": round(achieved, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
            "frac": round(achieved / pk["hbm_gbs"], 4), "peak_source": pk["source"],
            "algorithmic_bytes_per_step": int(routed), "unique_experts_per_step": res["U"],
            "bytes_per_expert": expert_bytes(wl),
            "traffic": read_traffic_profile(f"decode_experts_{wl.name}")}


def launches_per_step(wl, w4a16=False) -> int:
    T = wl.T
    if wl.kind != "decode":
        # router, top-k, permute (hist, scan, scatter, first), tile rows, x
        # encoding (W4A16: x gather), gate/up GEMM, h encoding (W4A4 only),
        # down GEMM, shared gate/up + down, unpermute + combine
        return 13 if w4a16 else 14
    # router, top-k + plan (one launch up to 8 tokens at E <= 320, else top-k
    # and the permute), expert gate/up, expert down, combine, and the shared
    # expert's two GEMVs on the auxiliary stream
    # (grouped W4A16 GEMM: also the tile rows and the x gather)
    fused_plan = T <= 8 and wl.E <= 320 and T * wl.k <= 1024
    n = 7 if fused_plan else (8 if T * wl.k <= 1024 else 11)
    return n + (2 if decode_grouped(wl) else 0)


def run_ours(args, rank, world, local_rank):
    import torch
    from routed_nvfp4_expert_b200 import capi
    from routed_nvfp4_expert_b200 import synthetic as syn

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    wl = syn.WORKLOADS[args.workload]
    clocks = clock_sampler(local_rank)
    if isinstance(clocks, ClockSampler):
        clocks.start()
    if wl.kind == "dense":
        res = measure_dense(wl, args, rank, world, local_rank, dev, clocks)
        clk = clocks.stop() if isinstance(clocks, ClockSampler) else clocks.result()
        ms_max = dist_max(world, res["ms"], dev)
        if rank != 0:
            return None
        res["ms"] = ms_max
        line = dense_line(res, peaks(), world)
        return {"metric": METRIC, "value": line["value"], "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": line["ms_per_step"], "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "bf16 weights x bf16 activations, fp32 accumulate",
                "data": "synthetic (seeded)",
                "config": {"workload": wl.name, "T": wl.T, "hidden": wl.H, "intermediate": wl.dense_I,
                           "path": "dense BF16 FFN", "parallelism": f"replicas x{world}",
                           "l2": "flushed before every timed step (read of a 2x L2 buffer)",
                           "graph": "CUDA graph of dense_ffn_bf16"},
                "roofline": line["roofline"], "gpu_launches": 2 * args.steps, "clocks": clk,
                "e2e": None}
    res = measure(wl, args, rank, world, local_rank, dev, clocks)
    # the prefill grouped GEMM under the same clock, in the same process
    pre = None
    if args.with_prefill and wl.kind == "decode":
        pre = measure(syn.WORKLOADS[args.with_prefill], args, rank, world, local_rank, dev, clocks)
    clk = clocks.stop() if isinstance(clocks, ClockSampler) else clocks.result()

    ms_max = dist_max(world, res["ms"], dev)
    e2e_max = dist_max(world, res["e2e_ms"], dev)
    res["kern_ms"] = dist_max(world, res["kern_ms"], dev)
    if pre is not None:
        pre_ms = dist_max(world, pre["ms"], dev)
        pre["kern_ms"] = dist_max(world, pre["kern_ms"], dev)
        pre_e2e = dist_max(world, pre["e2e_ms"], dev)
    if rank != 0:
        return None

    pk = peaks()
    T, H = wl.T, wl.H
    prefill = res["prefill"]
    path_name = (("prefill grouped GEMM (W4A16, tcgen05 kind::f16)" if res["w4a16"] else
                  "prefill grouped GEMM (W4A4, tcgen05 block-scaled FP4)") if prefill else
                 "decode, tensor-core expert kernels (W4A16)" if decode_mma(wl) else
                 "decode, grouped W4A16 GEMM (tcgen05 kind::f16)" if decode_grouped(wl) else "decode GEMV (W4A16)")
    n_launch = launches_per_step(wl, res["w4a16"])
    out = {
        "metric": METRIC,
        "value": round(world * T / (ms_max * 1e-3), 2),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_max, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": (("nvfp4 weights x f16 activations (tcgen05 kind::f16), fp32 accumulate" if res["w4a16"] else
                   "nvfp4 weights x nvfp4 activations (tcgen05 mxf4nvf4), fp32 accumulate") if prefill
                  else "nvfp4 weights x bf16 activations, exact products, fp32 accumulate"),
        "data": "synthetic (seeded; NVFP4 experts drawn in the code domain)",
        "config": {"workload": wl.name, "T": T, "hidden": H, "experts": wl.E, "intermediate": wl.I, "top_k": wl.k,
                   "shared_intermediate": wl.Is, "path": path_name, "parallelism": f"replicas x{world}",
                   "l2": "flushed before every timed step (read of a 2x L2 buffer)", "graph": "CUDA graph of moe_forward"},
        "diagnostics": {
            "ms_per_step_with_stage_events": round(res["timed_ms"], 5),
            "stages_ms_all_events": {n: round(float(v), 5) for n, v in zip(capi.STAGES, res["stage_avg"])},
            "note": f"value: K replays of the forward's graph; interleaved with them in the timed region, K "
                    f"replays of the same forward with {2 * res['n_spans']} event nodes around the dominant "
                    "kernels give roofline.achieved (an event node also ends the launch overlap of the "
                    "kernels it separates); stages_ms_all_events comes from a graph with an event node at "
                    "every stage boundary"},
        "roofline": roofline_of(res, pk),
        "e2e": {"value": round(world * T / (e2e_max * 1e-3), 2), "unit": "tokens/s",
                "h2d_bytes_per_step": T * H * 2, "d2h_bytes_per_step": T * H * 2,
                "ms_per_step": round(e2e_max, 5)},
        "gpu_launches": 2 * n_launch * args.steps,   # both graphs of the timed region
        "clocks": clk,
    }
    if pre is not None:
        pwl = pre["wl"]
        out["prefill"] = {
            "workload": pwl.name, "T": pwl.T, "value": round(world * pwl.T / (pre_ms * 1e-3), 2), "unit": "tokens/s",
            "ms_per_step": round(pre_ms, 5), "roofline": roofline_of(pre, pk),
            "e2e": {"value": round(world * pwl.T / (pre_e2e * 1e-3), 2), "unit": "tokens/s",
                    "h2d_bytes_per_step": pwl.T * pwl.H * 2, "d2h_bytes_per_step": pwl.T * pwl.H * 2,
                    "ms_per_step": round(pre_e2e, 5)},
            "stages_ms_all_events": {n: round(float(v), 5) for n, v in zip(capi.STAGES, pre["stage_avg"])},
            "gpu_launches": 2 * launches_per_step(pwl, pre["w4a16"]) * args.steps,
            "note": "timed in the same process and under the same clock record as the decode line, after it",
        }
        out["gpu_launches"] += out["prefill"]["gpu_launches"]
    if not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(wl, res["inp"], budget_s=args.cpu_seconds)
    return out


def read_traffic_profile(stem: str):
    """DRAM bytes per step of the dominant kernel from the committed ncu
    summary profiles/<stem>.traffic.json, if one exists (else null)."""
    p = os.path.join(ROOT, "profiles", f"{stem}.traffic.json")
    if not os.path.exists(p):
        return None
    try:
        return json.load(open(p)).get("dram_bytes_per_step")
    except (ValueError, OSError):
        return None


# ------------------------------------------------------------------ oracle timing

def cpu_baseline(wl, inp, budget_s=15.0, steps=None):
    """The CPU oracle, as it stands, on this host's cores: whole site forwards
    of single tokens (fresh dequantisation cache per token, as a decode step
    would), repeated for about budget_s seconds."""
    from oracle import site as OS
    ocfg = OS.SiteConfig(wl.H, wl.I, wl.Is, wl.E, 0, wl.E, wl.k, wl.rsf, wl.limit)
    mode = "decode" if wl.kind == "decode" else "prefill"
    cores = len(os.sched_getaffinity(0))
    n = 0
    t0 = time.perf_counter()
    times = []
    while True:
        ts = time.perf_counter()
        OS.site_forward(inp, ocfg, mode, tokens=np.array([n % wl.T]), cache=OS.ExpertCache(inp))
        times.append(time.perf_counter() - ts)
        n += 1
        if (steps is not None and n >= steps) or (steps is None and time.perf_counter() - t0 > budget_s):
            break
    el = time.perf_counter() - t0
    return {"value": round(n / el, 4), "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"{n} single-token site forwards of {wl.name} (fp64 numpy, fresh expert dequant per token)",
            "seconds": round(el, 2)}


def run_reference(args, rank, world):
    if rank != 0:
        return None
    from routed_nvfp4_expert_b200 import synthetic as syn
    wl = syn.WORKLOADS[args.workload]
    inp = syn.make_site(wl, seed=0)
    cb = cpu_baseline(wl, inp, steps=args.warmup)      # warm-up
    cb = cpu_baseline(wl, inp, steps=args.steps)
    ms = 1e3 / cb["value"]
    return {
        "impl": "reference",
        "metric": METRIC,
        "value": cb["value"],
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms, 3),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic (seeded)",
        "config": {"workload": wl.name, "T": wl.T, "hidden": wl.H, "experts": wl.E, "intermediate": wl.I,
                   "top_k": wl.k, "shared_intermediate": wl.Is, "path": "CPU oracle"},
        "cpu_baseline": cb,
        "e2e": {"value": cb["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# ------------------------------------------------------------------ dist

_PG = None


def dist_init():
    global _PG
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=120))
        _PG = dist
    return rank, world, local


def dist_barrier(world):
    if world > 1 and _PG is not None:
        _PG.barrier()


def dist_max(world, v, dev=None):
    if world > 1 and _PG is not None:
        import torch
        t = torch.tensor([v], dtype=torch.float64)
        _PG.all_reduce(t, op=_PG.ReduceOp.MAX)
        return float(t.item())
    return v


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="decode_t1")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--prefill-path", default="w4a4", choices=["w4a4", "w4a16"],
                    help="prefill expert numerics: NVFP4 activations on the block-scaled FP4 tensor cores (w4a4) "
                         "or 16-bit activations on kind::f16 (w4a16)")
    ap.add_argument("--with-prefill", default="prefill_t4096",
                    help="after a decode workload, also time this prefill workload in the same run ('' = off)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    rank, world, local = dist_init()
    if args.impl == "reference":
        out = run_reference(args, rank, world)
    else:
        out = run_ours(args, rank, world, local)
    if out is not None:
        print(json.dumps(out), flush=True)
    if world > 1 and _PG is not None:
        _PG.destroy_process_group()


if __name__ == "__main__":
    main()
