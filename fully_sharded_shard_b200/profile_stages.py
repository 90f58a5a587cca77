"""Time (or run under a profiler) single stages of one parameter group with
only the buffers those stages touch, so that a capture of a large group
stays within a few GB of device memory.

Usage::

    python -m fully_sharded_shard_b200.profile_stages --workload llama_block \
        --group 0 --stages copy_in,copy_out --iters 5

Stages: copy_in (fp32 master -> bf16 all-gather buffer), copy_out (buffer ->
unsharded arena), rs_reduce (fused reduce-scatter), adamw, rs_adamw (fused
reduce-scatter + AdamW + next copy-in).  Every buffer is allocated once and
filled with seeded values; each iteration runs the stages in that order, and
the per-stage CUDA-event times (median over the iterations) are printed as
one JSON line with the algorithmic bytes and GB/s of each stage.  Before
every stage a 256 MB buffer (twice the L2) is written outside the timed
events, so a stage never reads what the previous one left in L2 (a group of
small parameters fits there); --no-flush leaves L2 alone.
"""
from __future__ import annotations

import argparse
import json
import statistics
import sys

import torch

from . import abi
from . import workloads as W

STAGES = ("copy_in", "copy_out", "rs_reduce", "adamw", "rs_adamw")


def stage_bytes(stage: str, N: int, S: int, P: int) -> int:
    """Algorithmic bytes of one launch (the step's byte model, per stage)."""
    Pp = N * S
    return {"copy_in": 6 * Pp, "copy_out": 2 * Pp + 2 * P, "rs_reduce": 2 * N * P + 4 * Pp,
            "adamw": 28 * Pp, "rs_adamw": 2 * N * P + 26 * Pp}[stage]


def main(argv=None) -> int:
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="llama_block")
    ap.add_argument("--group", type=int, default=0)
    ap.add_argument("--stages", default="copy_in,copy_out")
    ap.add_argument("--iters", type=int, default=5)
    ap.add_argument("--no-flush", action="store_true",
                    help="do not write a buffer larger than L2 before each stage")
    args = ap.parse_args(argv)
    stages = [s for s in args.stages.split(",") if s]
    for s in stages:
        if s not in STAGES:
            raise SystemExit(f"unknown stage {s}; choose from {STAGES}")
    wl = W.by_name(args.workload)
    grp = wl.groups[args.group]
    N = wl.N
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    g = abi.fsdp_plan_group(grp.shapes, N)
    NS, A = N * g.S, g.P_arena
    need_state = any(s in ("adamw", "rs_adamw", "copy_in") for s in stages)
    need_grads = any(s in ("rs_reduce", "rs_adamw") for s in stages)
    master = m = v = grads = red = None
    if need_state:
        full = torch.empty(max(A, 1), dtype=torch.float32, device=dev)
        W.fill_master(full, wl, grp.name)
        master = torch.empty(max(NS, 1), dtype=torch.float32, device=dev)
        abi.fsdp_shard_params(g, full, master)
        del full
    if any(s in ("adamw", "rs_adamw") for s in stages):
        m = torch.zeros(max(NS, 1), dtype=torch.float32, device=dev)
        v = torch.zeros(max(NS, 1), dtype=torch.float32, device=dev)
    if need_grads:
        grads = torch.empty(N, max(A, 1), dtype=torch.bfloat16, device=dev)
        for r in range(N):
            W.fill_grads_bf16(grads[r], wl, grp.name, "profile", r)
    if any(s in ("rs_reduce", "adamw") for s in stages):
        # a gradient-like reduced gradient: AdamW's arithmetic (its divisions
        # in particular) takes different paths on zeros
        red = torch.empty(max(NS, 1), dtype=torch.float32, device=dev)
        W.fill_master(red, W.Workload(wl.name, N, [], wl.op, wl.seed, "normal",
                                      wl.grad_sigma, wl.grad_sigma), grp.name, "profile_red")
    ag = torch.empty(max(NS, 1), dtype=torch.bfloat16, device=dev)
    if "copy_in" not in stages:
        ag.view(torch.int16).copy_(torch.randint(-16000, 16000, (max(NS, 1),), dtype=torch.int16,
                                                 device=dev))
    arena = torch.empty(max(A, 1), dtype=torch.bfloat16, device=dev) if "copy_out" in stages \
        else None
    hp = dict(W.ADAMW_DEFAULTS)
    calls = {
        "copy_in": lambda t: abi.fsdp_copy_in(g, master, ag),
        "copy_out": lambda t: abi.fsdp_copy_out(g, ag, arena),
        "rs_reduce": lambda t: abi.fsdp_rs_reduce(g, grads, wl.op, red),
        "adamw": lambda t: abi.fsdp_adamw_step(g, master, m, v, red, step=t, **hp),
        "rs_adamw": lambda t: abi.fsdp_rs_adamw_step(g, grads, wl.op, master, m, v, step=t,
                                                     ag_next=ag, **hp),
    }
    flush = None if args.no_flush else torch.empty(64 << 20, dtype=torch.float32, device=dev)
    times = {s: [] for s in stages}
    for t in range(1, args.iters + 1):
        for s in stages:
            if flush is not None:
                flush.zero_()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
            calls[s](t)
            e1.record()
            times[s].append((e0, e1))
    torch.cuda.synchronize()
    out = {"workload": wl.name, "group": grp.name, "N": N, "S": g.S, "P": g.P,
           "l2": "not flushed" if flush is None else "256 MB written before each stage",
           "device_bytes": int(torch.cuda.max_memory_allocated(dev)), "stages": {}}
    for s in stages:
        ms = statistics.median(a.elapsed_time(b) for a, b in times[s])
        b = stage_bytes(s, N, g.S, g.P)
        out["stages"][s] = {"ms": round(ms, 4), "bytes": b, "GBps": round(b / (ms * 1e-3) / 1e9, 1)}
    print(json.dumps(out), flush=True)
    g.destroy()
    return 0


if __name__ == "__main__":
    sys.exit(main())
