"""Profiling driver: a few site forwards of one synthetic workload, nothing
else, so that a profiler run (ncu) sees a short, known launch sequence.

    python -m routed_nvfp4_expert_b200.profile_site --workload prefill_t4096 \
        [--experts 96] [--reps 2]

--experts overrides the expert count of the workload (smaller device
footprint for captures that replay each kernel many times). Prints the event
time of each forward (not a benchmark number: use bench.py for those).
"""
from __future__ import annotations

import argparse
import dataclasses

import torch

from . import capi
from . import synthetic as syn


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="decode_t1")
    ap.add_argument("--experts", type=int, default=0)
    ap.add_argument("--reps", type=int, default=2)
    args = ap.parse_args()
    wl = syn.WORKLOADS[args.workload]
    if args.experts:
        wl = dataclasses.replace(wl, E=args.experts, name=f"{wl.name}_E{args.experts}")
    inp = syn.make_site(wl, seed=0)
    site = capi.site_to_device(inp)
    cfg = capi.config_for(wl)
    path = capi.PATH_DECODE if wl.kind == "decode" else capi.PATH_PREFILL
    capi.moe_prepare_weights(cfg, site)   # the grouped GEMMs' scale atoms (prefill, decode batches >= 9)
    x = capi.bf16_tensor(inp["x"])
    y = torch.empty_like(x)
    ws = capi.alloc_workspace(cfg, wl.T, path)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    for i in range(args.reps):
        ev[0].record()
        capi.moe_forward(cfg, site, x, path, y, ws)
        ev[1].record()
        torch.cuda.synchronize()
        print(f"{wl.name} forward {i}: {ev[0].elapsed_time(ev[1]):.3f} ms")
    capi.moe_read_device_status(ws)
    print("ok")


if __name__ == "__main__":
    main()
