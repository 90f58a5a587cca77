"""Benchmark of the FSDP2 per-parameter sharding step on B200.

One step = for every parameter group of the model, in order:
  copy-in (fp32 shards -> bf16 rank-major all-gather buffer),
  copy-out (all-gather buffer -> unsharded bf16 parameters),
  reduce-scatter (N ranks' bf16 gradients -> fp32 reduced shards, AVG, fused
  pack + rank-ordered fold),
  AdamW (fp32 master, m, v shards),
with the N data-parallel ranks emulated as N virtual ranks in one GPU's HBM.
The default workload is the 7B-shaped model: 32 Llama-2-7B blocks plus the
root group (embedding, final norm, LM head), N = 8, 6.74 G parameters.

Byte model (algorithmic bytes a group step must move, each once):
  B = 6*Pp (copy-in) + 2*Pp + 2*P (copy-out) + 2*N*P + 4*Pp (reduce-scatter)
      + 28*Pp (AdamW),     Pp = N*S padded elements, P real elements.
Reported value = total bytes of the step / step time (GB/s, 1e9 bytes).

Usage:
  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
Under torchrun each rank runs its own full workload (no data-path
collective; weak scaling) and rank 0 prints one JSON line.
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

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "FSDP2 step GB/s and params/s over N virtual ranks; % of HBM roofline"
FALLBACK_HBM_GBS = 6650.0
SPEC_HBM_GBS = 8000.0
KERNELS_DIR = os.path.join(ROOT, "fully_sharded_shard_b200", "csrc")
TRAFFIC_JSON = os.path.join(ROOT, "profiles", "dram_traffic.json")


# ---------------------------------------------------------------------------
# byte model
# ---------------------------------------------------------------------------
def stage_bytes(N: int, S: int, P: int) -> dict:
    Pp = N * S
    return {
        "copy_in": 6 * Pp,
        "copy_out": 2 * Pp + 2 * P,
        "rs_reduce": 2 * N * P + 4 * Pp,
        "adamw": 28 * Pp,
    }


def group_bytes(N: int, S: int, P: int) -> int:
    return sum(stage_bytes(N, S, P).values())


def fused_stage_bytes(N: int, S: int, P: int) -> dict:
    """The step with the reduce-scatter, AdamW and the next step's copy-in
    fused into one pass: copy-out, then one kernel that reads the N ranks'
    gradients and master/m/v and writes master/m/v and the bf16 all-gather
    input of the next step."""
    Pp = N * S
    return {
        "copy_out": 2 * Pp + 2 * P,
        "rs_adamw_copy_in": 2 * N * P + 24 * Pp + 2 * Pp,
    }


def fused_fp8_stage_bytes(N: int, S: int, P: int, n: int) -> dict:
    """The fused step with an FP8 all-gather (delayed scaling): the byte
    copy-out, then one kernel that reads the N ranks' gradients and
    master/m/v and writes master/m/v and the E4M3 all-gather input of the next
    step; the per-parameter scales (n of them, read and written) are
    negligible but counted."""
    Pp = N * S
    return {
        "copy_out": Pp + P,
        "rs_adamw_copy_in_fp8": 2 * N * P + 24 * Pp + Pp + 12 * n,
    }


# ---------------------------------------------------------------------------
# distributed plumbing
# ---------------------------------------------------------------------------
def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def init_dist(backend: str):
    import datetime
    import torch.distributed as dist
    if not dist.is_initialized():
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return dist


def max_over_ranks(value: float, device=None) -> float:
    """Max of a float over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return value
    on_dev = dist.get_backend() == "nccl"
    t = torch.tensor([value], dtype=torch.float64, device=device if on_dev else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(value: float, device=None) -> float:
    """Sum of a float over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return value
    on_dev = dist.get_backend() == "nccl"
    t = torch.tensor([value], dtype=torch.float64, device=device if on_dev else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def barrier(device=None):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        if device is not None and device.type == "cuda" and dist.get_backend() == "nccl":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# ---------------------------------------------------------------------------
# peaks, clocks, traffic record
# ---------------------------------------------------------------------------
def hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            v = float(json.load(f)["hbm_gbs"])
        return v, "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.out = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200", "-i", str(self.gpu)],
                stdout=self.out, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.out.flush()
        rows = []
        with open(self.out.name) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    rows.append((float(parts[1]), float(parts[2]), float(parts[3]), parts[5:9]))
                except ValueError:
                    continue
        os.unlink(self.out.name)
        if not rows:
            return None
        maxp = max(r[2] for r in rows)
        load = [r for r in rows if r[2] >= 0.5 * maxp] or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[k] for r in load for k in range(4) if r[3][k].lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in load),
                "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows), "samples_under_load": len(load),
                "power_w_max": maxp}


# The file each profiled kernel is compiled from (with the device header and
# the internal header every kernel file includes).
KERNEL_FILES = {
    "k_copy_in": "fsdpk_gather.cu", "k_copy_out": "fsdpk_gather.cu",
    "k_fp8_copy_in": "fsdpk_gather.cu", "k_fp8_amax": "fsdpk_gather.cu",
    "k_copy_out_tab": "fsdpk_gather.cu",
    "k_reduce_units": "fsdpk_reduce.cu", "k_accumulate": "fsdpk_reduce.cu",
    "k_reduce_acc": "fsdpk_reduce.cu", "k_reduce_units_tab": "fsdpk_reduce.cu",
    "k_adamw": "fsdpk_update.cu", "k_rs_adamw": "fsdpk_update.cu",
    "k_rs_adamw_fp8": "fsdpk_update.cu",
}


def kernel_source_hash(kernel: str) -> str:
    """Hash of the sources `kernel` is compiled from: its .cu file, the device
    header and the internal header."""
    h = hashlib.sha256()
    for name in (KERNEL_FILES[kernel], "fsdpk_device.cuh", "fsdpk_internal.h"):
        with open(os.path.join(KERNELS_DIR, name), "rb") as f:
            h.update(name.encode() + b"\0" + f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, workload: str):
    """Per-launch DRAM bytes of `kernel` from the committed ncu summary, or None
    when it is absent or the kernel's sources changed since it was captured."""
    try:
        with open(TRAFFIC_JSON) as f:
            rec = json.load(f)
        if rec.get("workload") != workload:
            return None
        if rec["sources_sha256_16"][kernel] != kernel_source_hash(kernel):
            return None
    except Exception:
        return None
    k = rec.get("per_launch_bytes", {}).get(kernel)
    return float(k) if k is not None else None


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------
class Model:
    """Device state of one workload replica: plans, fp32 sharded state per
    group instance, shared working buffers and a pool of gradient buffers."""

    def __init__(self, wl, device, grad_pool: int, rank: int):
        import torch
        from fully_sharded_shard_b200 import abi
        from fully_sharded_shard_b200 import workloads as W
        self.wl = wl
        self.device = device
        self.plans = []            # one abi.Group per distinct group
        self.instances = []        # (plan index, master, m, v, grad pool index)
        N = wl.N
        max_NS = 0
        max_A = 0
        for gi, grp in enumerate(wl.groups):
            g = abi.fsdp_plan_group(grp.shapes, N)
            self.plans.append(g)
            max_NS = max(max_NS, N * g.S)
            max_A = max(max_A, g.P_arena)
        self.ag = torch.empty(max(max_NS, 1), dtype=torch.bfloat16, device=device)
        self.arena = torch.empty(max(max_A, 1), dtype=torch.bfloat16, device=device)
        self.reduced = torch.empty(max(max_NS, 1), dtype=torch.float32, device=device)
        full = torch.empty(max(max_A, 1), dtype=torch.float32, device=device)
        # gradient pools: per plan, up to `grad_pool` distinct seeded buffers
        self.grads = []
        for gi, grp in enumerate(wl.groups):
            g = self.plans[gi]
            k = max(1, min(grad_pool, grp.repeat))
            pool = []
            for j in range(k):
                t = torch.empty(N, g.P_arena, dtype=torch.bfloat16, device=device)
                for r in range(N):
                    W.fill_grads_bf16(t[r], wl, grp.name, "rank", rank, "pool", j, r)
                    if grp.zero_grad:
                        W.zero_param_ranges(t[r], g.arena_off, g.numel, grp.zero_grad)
                pool.append(t)
            self.grads.append(pool)
        for gi, grp in enumerate(wl.groups):
            g = self.plans[gi]
            for rep in range(grp.repeat):
                NS = N * g.S
                master = torch.empty(NS, dtype=torch.float32, device=device)
                W.fill_master(full[:g.P_arena], wl, grp.name, "rank", rank, "layer", rep)
                abi.fsdp_shard_params(self.plans[gi], full, master)
                m = torch.zeros(NS, dtype=torch.float32, device=device)
                v = torch.zeros(NS, dtype=torch.float32, device=device)
                self.instances.append((gi, master, m, v, rep % len(self.grads[gi])))
        del full
        torch.cuda.synchronize(device)
        self.step_count = 0
        self.P_total = sum(self.plans[i[0]].P for i in self.instances)
        self.bytes_per_step = sum(group_bytes(N, self.plans[i[0]].S, self.plans[i[0]].P)
                                  for i in self.instances)
        self.stage_bytes = {k: 0 for k in ("copy_in", "copy_out", "rs_reduce", "adamw")}
        for i in self.instances:
            g = self.plans[i[0]]
            for k, b in stage_bytes(N, g.S, g.P).items():
                self.stage_bytes[k] += b
        self.launches_per_step = 4 * len(self.instances)
        self.ag_groups = None
        self._ag2 = None
        self._arena2 = None

    def enable_fused(self):
        """Per-group bf16 all-gather buffers: the fused update writes the next
        step's all-gather input for each group, so each group keeps its own."""
        import torch
        from fully_sharded_shard_b200 import abi
        self.ag_groups = []
        for gi, master, m, v, pj in self.instances:
            g = self.plans[gi]
            ag = torch.empty(max(g.N * g.S, 1), dtype=torch.bfloat16, device=self.device)
            abi.fsdp_copy_in(g, master, ag)
            self.ag_groups.append(ag)
        torch.cuda.synchronize(self.device)
        N = self.wl.N
        self.fused_bytes = {k: 0 for k in ("copy_out", "rs_adamw_copy_in")}
        for i in self.instances:
            g = self.plans[i[0]]
            for k, b in fused_stage_bytes(N, g.S, g.P).items():
                self.fused_bytes[k] += b

    def fused_step_two_streams(self, s_gather, s_update):
        """The fused step on two streams: each group's copy-out on
        `s_gather`, its fused update on `s_update` once the copy-out has read
        the group's all-gather buffer (the update rewrites it for the next
        step); group g+1's copy-out overlaps group g's update."""
        import torch
        from fully_sharded_shard_b200 import abi
        from fully_sharded_shard_b200 import workloads as W
        if self._arena2 is None:
            self._arena2 = [self.arena, torch.empty_like(self.arena)]
        self.step_count += 1
        hp = dict(W.ADAMW_DEFAULTS)
        for idx, (gi, master, m, v, pj) in enumerate(self.instances):
            g = self.plans[gi]
            ag = self.ag_groups[idx]
            abi.fsdp_copy_out(g, ag, self._arena2[idx % 2], s_gather)
            read = torch.cuda.Event()
            read.record(s_gather)
            s_update.wait_event(read)
            abi.fsdp_rs_adamw_step(g, self.grads[gi][pj], self.wl.op, master, m, v,
                                   step=self.step_count, ag_next=ag, stream=s_update, **hp)
        done = torch.cuda.Event()
        done.record(s_update)
        s_gather.wait_event(done)

    def fused_step(self, stream, events=None):
        """One step with the reduce-scatter, AdamW and next copy-in fused."""
        import torch
        from fully_sharded_shard_b200 import abi
        from fully_sharded_shard_b200 import workloads as W
        self.step_count += 1
        hp = dict(W.ADAMW_DEFAULTS)
        for idx, (gi, master, m, v, pj) in enumerate(self.instances):
            g = self.plans[gi]
            ag = self.ag_groups[idx]
            calls = (
                ("copy_out", lambda: abi.fsdp_copy_out(g, ag, self.arena, stream)),
                ("rs_adamw_copy_in", lambda: abi.fsdp_rs_adamw_step(
                    g, self.grads[gi][pj], self.wl.op, master, m, v, step=self.step_count,
                    ag_next=ag, stream=stream, **hp)),
            )
            for name, fn in calls:
                if events is None:
                    fn()
                else:
                    e0 = torch.cuda.Event(enable_timing=True)
                    e1 = torch.cuda.Event(enable_timing=True)
                    e0.record(stream)
                    fn()
                    e1.record(stream)
                    events[name].append((e0, e1))

    def run_group(self, idx, stream, step, grads=None, events=None, spacer=None):
        """Enqueue the four stages of group instance `idx` on `stream`.
        events: optional dict stage -> list receiving (start, end) events.
        spacer: optional callable enqueued before each stage's start event
        (outside the timed pair)."""
        import torch
        from fully_sharded_shard_b200 import abi
        from fully_sharded_shard_b200 import workloads as W
        gi, master, m, v, pj = self.instances[idx]
        g = self.plans[gi]
        if grads is None:
            grads = self.grads[gi][pj]
        hp = dict(W.ADAMW_DEFAULTS)
        calls = (
            ("copy_in", lambda: abi.fsdp_copy_in(g, master, self.ag, stream)),
            ("copy_out", lambda: abi.fsdp_copy_out(g, self.ag, self.arena, stream)),
            ("rs_reduce", lambda: abi.fsdp_rs_reduce(g, grads, self.wl.op, self.reduced,
                                                     stream=stream)),
            ("adamw", lambda: abi.fsdp_adamw_step(g, master, m, v, self.reduced, step=step,
                                                  stream=stream, **hp)),
        )
        for name, fn in calls:
            if events is None:
                fn()
            else:
                if spacer is not None:
                    spacer()
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                fn()
                e1.record(stream)
                events[name].append((e0, e1))

    def step(self, stream, events=None, spacer=None):
        """Enqueue one full step (every group, in order) on `stream`."""
        self.step_count += 1
        for idx in range(len(self.instances)):
            self.run_group(idx, stream, self.step_count, events=events, spacer=spacer)

    def step_two_streams(self, s_gather, s_update, events=None):
        """One full step on two streams, as FSDP2 splits communication from
        compute: the all-gather half of each group (copy-in, copy-out, double
        buffered) on `s_gather`, its reduce-scatter and AdamW on `s_update`
        once its copy-in has read the pre-update master.  Group g+1's
        all-gather overlaps group g's update.  The step ends with `s_gather`
        waiting for `s_update`, so the next step's copy-ins see this step's
        updates.  events: optional dict stage -> list receiving (start, end)
        events recorded around each launch on the stream it runs on."""
        import torch
        from fully_sharded_shard_b200 import abi
        from fully_sharded_shard_b200 import workloads as W

        def timed(name, st, fn):
            if events is None:
                fn()
                return
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(st)
            fn()
            e1.record(st)
            events[name].append((e0, e1))

        if self._ag2 is None:
            self._ag2 = [self.ag, torch.empty_like(self.ag)]
            self._arena2 = [self.arena, torch.empty_like(self.arena)]
        self.step_count += 1
        hp = dict(W.ADAMW_DEFAULTS)
        for idx, (gi, master, m, v, pj) in enumerate(self.instances):
            g = self.plans[gi]
            ag, arena = self._ag2[idx % 2], self._arena2[idx % 2]
            timed("copy_in", s_gather, lambda: abi.fsdp_copy_in(g, master, ag, s_gather))
            read = torch.cuda.Event()
            read.record(s_gather)
            timed("copy_out", s_gather, lambda: abi.fsdp_copy_out(g, ag, arena, s_gather))
            s_update.wait_event(read)
            timed("rs_reduce", s_update, lambda: abi.fsdp_rs_reduce(
                g, self.grads[gi][pj], self.wl.op, self.reduced, stream=s_update))
            timed("adamw", s_update, lambda: abi.fsdp_adamw_step(
                g, master, m, v, self.reduced, step=self.step_count, stream=s_update, **hp))
        done = torch.cuda.Event()
        done.record(s_update)
        s_gather.wait_event(done)


def run_ours(args, wl, device, rank, ws):
    import torch
    from fully_sharded_shard_b200 import workloads as W
    stream = torch.cuda.Stream(device)
    s_update = torch.cuda.Stream(device)
    t_setup = time.time()
    model = Model(wl, device, args.grad_pool, rank)
    setup_s = time.time() - t_setup

    def one_step(events=None):
        if args.one_stream:
            model.step(stream, events=events)
        else:
            model.step_two_streams(stream, s_update, events=events)

    # warm-up
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            one_step()
    torch.cuda.synchronize(device)

    # timed region: K whole steps between two events on the launching stream
    sampler = ClockSampler(device.index if device.index is not None else 0)
    barrier(device)
    torch.cuda.synchronize(device)
    sampler.start()
    e_start = torch.cuda.Event(enable_timing=True)
    e_end = torch.cuda.Event(enable_timing=True)
    # events around every launch, on its own stream, give the per-kernel
    # launch durations inside the timed region (the roofline's `achieved`)
    live = {k: [] for k in ("copy_in", "copy_out", "rs_reduce", "adamw")}
    marks = []   # the end of every step on the launching stream
    e_start.record(stream)
    for _ in range(args.steps):
        one_step(live)
        ev = torch.cuda.Event(enable_timing=True)
        ev.record(stream)
        marks.append(ev)
    e_end.record(stream)
    torch.cuda.synchronize(device)
    barrier(device)
    clocks = sampler.stop()
    ms_total = e_start.elapsed_time(e_end)
    ms_total = max_over_ranks(ms_total, device)
    ms_step = ms_total / args.steps
    per_step = [a.elapsed_time(b) for a, b in zip([e_start] + marks[:-1], marks)]
    ms_median = max_over_ranks(float(statistics.median(per_step)), device)

    # per-stage times: the same steps again, one stream, events around every
    # launch.  Before each start event a 256 MB buffer (twice the L2) is
    # written: no stage reads what the previous one left in L2, and the GPU
    # stays ahead of the host, so a short launch's time does not include the
    # host's call overhead.
    events = {k: [] for k in ("copy_in", "copy_out", "rs_reduce", "adamw")}
    stage_steps = max(1, min(args.steps, 3))
    flush = torch.empty(64 << 20, dtype=torch.float32, device=device)
    with torch.cuda.stream(stream):
        for _ in range(stage_steps):
            model.step(stream, events=events, spacer=flush.zero_)
    torch.cuda.synchronize(device)
    del flush
    stage_ms = {k: sum(a.elapsed_time(b) for a, b in v) / stage_steps for k, v in events.items()}

    peak, peak_kind = hbm_peak()
    gbs = ws * model.bytes_per_step / (ms_step * 1e-3) / 1e9
    params_s = ws * model.P_total / (ms_step * 1e-3)
    live_ms = {k: sum(a.elapsed_time(b) for a, b in v) / args.steps for k, v in live.items()}
    dom = max(live_ms, key=live_ms.get)
    dom_launch_ms = live_ms[dom] / len(model.instances)
    dom_achieved = model.stage_bytes[dom] / (live_ms[dom] * 1e-3) / 1e9
    iso_achieved = model.stage_bytes[dom] / (stage_ms[dom] * 1e-3) / 1e9
    kernel_names = {"copy_in": "k_copy_in", "copy_out": "k_copy_out",
                    "rs_reduce": "k_reduce_units", "adamw": "k_adamw"}
    traffic = recorded_traffic(kernel_names[dom], wl.name)
    roofline = {
        "bound": "hbm", "kernel": kernel_names[dom], "achieved": round(dom_achieved, 1),
        "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
        "frac": round(dom_achieved / peak, 4),
        "algorithmic_bytes_per_launch": int(model.stage_bytes[dom] / len(model.instances)),
        "avg_launch_ms": round(dom_launch_ms, 4),
        "launch_timing": "CUDA events around every launch of the kernel inside the timed steps, "
                         "on its own stream",
        "achieved_serial_pass": round(iso_achieved, 1),
        "traffic": traffic,
    }
    stages = {k: {"ms_per_step": round(stage_ms[k], 3),
                  "GBps": round(model.stage_bytes[k] / (stage_ms[k] * 1e-3) / 1e9, 1),
                  "frac_of_peak": round(model.stage_bytes[k] / (stage_ms[k] * 1e-3) / 1e9 / peak, 4)}
              for k in stage_ms}

    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, model, device, stream, ws)

    fused = None
    if not args.no_fused:
        fused = run_fused(args, model, device, stream, ws, ms_step, peak)

    fused8 = None
    if not args.no_fused and not args.no_fp8:
        fused8 = run_fused_fp8(args, model, device, stream, ws,
                               fused["ms_per_step"] if fused else None, peak)

    accum = None
    if not args.no_accumulate:
        accum = run_accumulate(args, model, device, stream)

    staged = None
    if not args.no_staged:
        staged = run_staged(args, model, device, stream)

    fp8 = None
    if not args.no_fp8:
        fp8 = run_fp8(args, model, device, stream)

    latency = None
    if not args.no_latency:
        latency = run_latency(device)

    out = {
        "metric": METRIC,
        "value": round(gbs, 1),
        "unit": "GB/s",
        "params_per_s": round(params_s, 1),
        "hbm_frac_of_measured": round(gbs / ws / peak, 4),
        "hbm_frac_of_spec_8TBs": round(gbs / ws / SPEC_HBM_GBS, 4),
        "n_gpus": ws,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_step, 3),
        "ms_per_step_median": round(ms_median, 3),
        "ms_per_step_min_max": [round(min(per_step), 3), round(max(per_step), 3)],
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f32",
        "storage_dtypes": "fp32 master/m/v/reduced grads; bf16 all-gather buffer, params, per-rank grads",
        "data": "synthetic: seeded N(0,0.02) fp32 master, N(0,1e-3) bf16 per-rank grads",
        "config": {
            "workload": wl.name,
            "N_virtual_ranks": wl.N,
            "groups_per_step": len(model.instances),
            "params": model.P_total,
            "bytes_per_step": model.bytes_per_step,
            "reduce_op": W.OP_NAMES[wl.op],
            "grad_pool_per_plan": args.grad_pool,
            "l2": "inputs larger than L2 (every group's state >> 126 MB); the per-stage pass "
                  "writes 256 MB before each launch",
            "parallelism": f"{ws} GPU(s), each a full {wl.N}-virtual-rank replica",
            "schedule": "one stream" if args.one_stream else
                        "two streams: all-gather half / reduce-scatter + update half",
        },
        "stages": stages,
        "roofline": roofline,
        "gpu_launches": model.launches_per_step * args.steps,
        "clocks": clocks,
        "e2e": e2e,
        "fused_step": fused,
        "fused_step_fp8_all_gather": fused8,
        "grad_accumulation": accum,
        "staged_reduce_scatter": staged,
        "fp8_all_gather": fp8,
        "tiny_latency": latency,
        "setup_s": round(setup_s, 1),
    }
    return out, model


def run_fused(args, model, device, stream, ws, ms_unfused, peak):
    """Time the fused step (copy-out, then reduce-scatter + AdamW + next
    copy-in in one kernel per group) on the same state, under its own byte
    model."""
    import torch
    model.enable_fused()
    s_update = torch.cuda.Stream(device)

    def one():
        if args.one_stream:
            model.fused_step(stream)
        else:
            model.fused_step_two_streams(stream, s_update)

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            one()
    torch.cuda.synchronize(device)
    barrier(device)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        one()
    e1.record(stream)
    torch.cuda.synchronize(device)
    ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, device)
    # per-stage times: events around every launch, averaged over a few steps
    events = {k: [] for k in ("copy_out", "rs_adamw_copy_in")}
    stage_steps = max(1, min(args.steps, 3))
    for _ in range(stage_steps):
        model.fused_step(stream, events=events)
    torch.cuda.synchronize(device)
    stage_ms = {k: sum(a.elapsed_time(b) for a, b in v) / stage_steps for k, v in events.items()}
    total = sum(model.fused_bytes.values())
    return {
        "ms_per_step": round(ms, 3),
        "bytes_per_step": total,
        "bytes_per_param": round(total / model.P_total, 3),
        "value": round(ws * total / (ms * 1e-3) / 1e9, 1),
        "unit": "GB/s (own byte model)",
        "frac_of_measured_peak": round(total / (ms * 1e-3) / 1e9 / peak, 4),
        "params_per_s": round(ws * model.P_total / (ms * 1e-3), 1),
        "speedup_vs_unfused_step": round(ms_unfused / ms, 3),
        "stages": {k: {"ms_per_step": round(stage_ms[k], 3),
                       "GBps": round(model.fused_bytes[k] / (stage_ms[k] * 1e-3) / 1e9, 1)}
                   for k in stage_ms},
        "launches_per_step": 2 * len(model.instances),
    }


def run_fused_fp8(args, model, device, stream, ws, ms_fused, peak):
    """Time the fused step with an FP8 all-gather (per-group byte copy-out,
    then reduce-scatter + AdamW + E4M3 next copy-in with the previous step's
    scales + next scales) on the same state, under its own byte model.  Each
    group's FP8 all-gather input lives in the first half of its bf16 buffer;
    each group keeps two scale buffers that swap every step."""
    import torch
    from fully_sharded_shard_b200 import abi
    from fully_sharded_shard_b200 import workloads as W
    if not hasattr(model, "ag_groups"):
        model.enable_fused()
    N = model.wl.N
    ag8s, scales = [], []
    for idx, (gi, master, m, v, pj) in enumerate(model.instances):
        g = model.plans[gi]
        ag8 = model.ag_groups[idx].view(torch.uint8)[:max(N * g.S, 1)]
        sc = [torch.empty(max(g.n, 1), dtype=torch.float32, device=device) for _ in range(2)]
        abi.fsdp_copy_in_fp8(g, master, ag8, sc[0])
        ag8s.append(ag8)
        scales.append(sc)
    arena8 = [model.arena.view(torch.uint8), torch.empty_like(model.arena).view(torch.uint8)]
    s_update = torch.cuda.Stream(device)
    hp = dict(W.ADAMW_DEFAULTS)
    state = {"t": 0}

    def one(events=None):
        state["t"] += 1
        model.step_count += 1
        t = state["t"]
        for idx, (gi, master, m, v, pj) in enumerate(model.instances):
            g = model.plans[gi]
            prev, nxt = scales[idx][(t - 1) % 2], scales[idx][t % 2]
            if events is not None or args.one_stream:
                calls = (("copy_out", lambda: abi.fsdp_copy_out_fp8(g, ag8s[idx], arena8[0], stream)),
                         ("rs_adamw_copy_in_fp8", lambda: abi.fsdp_rs_adamw_step_fp8(
                             g, model.grads[gi][pj], model.wl.op, master, m, v,
                             step=model.step_count, scales_prev=prev, ag8_next=ag8s[idx],
                             scales_next=nxt, stream=stream, **hp)))
                for name, fn in calls:
                    if events is None:
                        fn()
                        continue
                    e0 = torch.cuda.Event(enable_timing=True)
                    e1 = torch.cuda.Event(enable_timing=True)
                    e0.record(stream)
                    fn()
                    e1.record(stream)
                    events[name].append((e0, e1))
                continue
            abi.fsdp_copy_out_fp8(g, ag8s[idx], arena8[idx % 2], stream)
            read = torch.cuda.Event()
            read.record(stream)
            s_update.wait_event(read)
            abi.fsdp_rs_adamw_step_fp8(g, model.grads[gi][pj], model.wl.op, master, m, v,
                                       step=model.step_count, scales_prev=prev,
                                       ag8_next=ag8s[idx], scales_next=nxt, stream=s_update,
                                       **hp)
        if events is None and not args.one_stream:
            done = torch.cuda.Event()
            done.record(s_update)
            stream.wait_event(done)

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            one()
    torch.cuda.synchronize(device)
    barrier(device)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        one()
    e1.record(stream)
    torch.cuda.synchronize(device)
    ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, device)
    events = {k: [] for k in ("copy_out", "rs_adamw_copy_in_fp8")}
    stage_steps = max(1, min(args.steps, 3))
    for _ in range(stage_steps):
        one(events)
    torch.cuda.synchronize(device)
    stage_ms = {k: sum(a.elapsed_time(b) for a, b in v) / stage_steps for k, v in events.items()}
    sb = {k: 0 for k in stage_ms}
    for i in model.instances:
        g = model.plans[i[0]]
        for k, b in fused_fp8_stage_bytes(N, g.S, g.P, g.n).items():
            sb[k] += b
    total = sum(sb.values())
    del arena8
    return {
        "ms_per_step": round(ms, 3),
        "bytes_per_step": total,
        "bytes_per_param": round(total / model.P_total, 3),
        "value": round(ws * total / (ms * 1e-3) / 1e9, 1),
        "unit": "GB/s (own byte model)",
        "frac_of_measured_peak": round(total / (ms * 1e-3) / 1e9 / peak, 4),
        "params_per_s": round(ws * model.P_total / (ms * 1e-3), 1),
        "speedup_vs_bf16_fused_step": round(ms_fused / ms, 3) if ms_fused else None,
        "stages": {k: {"ms_per_step": round(stage_ms[k], 3),
                       "GBps": round(sb[k] / (stage_ms[k] * 1e-3) / 1e9, 1)}
                   for k in stage_ms},
        "launches_per_step": 3 * len(model.instances),
    }


def peer_stage_bytes(N: int, S: int, P: int, L: int, P_local: int) -> dict:
    """Per-device bytes of one group step when the N virtual ranks are spread
    over devices, L per device (P_local real elements in the local shards):
    the local copy-in, the copy-out of the whole group on every device (it
    pulls every rank's rows), the reduce-scatter of the local destination
    rows (N source arenas each) and the local AdamW."""
    LS = L * S
    return {"copy_in": 6 * LS, "copy_out": 2 * N * S + 2 * P,
            "rs_reduce": 2 * N * P_local + 4 * LS, "adamw": 28 * LS}


def local_real_elems(shapes, chunk_rows, r0: int, L: int) -> int:
    """Real (unpadded) elements in the shards of ranks [r0, r0 + L): rank j
    holds clamp(d0 - j * c, 0, c) rows of each parameter."""
    total = 0
    for shape, c in zip(shapes, chunk_rows):
        d0 = shape[0] if len(shape) else 1
        cols = 1
        for d in shape[1:]:
            cols *= d
        total += sum(max(0, min(c, d0 - j * c)) * cols for j in range(r0, r0 + L))
    return total


def peer_exchange_bytes(N: int, S: int, L: int, P_local: int, D: int) -> int:
    """Bytes one device pulls from the other devices per group step: the
    other ranks' slot rows (copy-out) and the other ranks' gradient rows of
    the local shards (reduce-scatter)."""
    if D == 1:
        return 0
    return 2 * (N - L) * S + 2 * (N - L) * P_local


def run_peer(args, wl, device, rank, ws):
    """The step with the N virtual ranks of every group spread over the ws
    processes (L = N / ws per device; one model, so the total work is fixed
    and the scaling is strong).  Each device copies its ranks in into a slot
    that every device maps (CUDA IPC), then pulls every rank's rows in its
    copy-out; its reduce-scatter pulls the N source arenas of its own rows;
    AdamW is local.  Host barriers order the phases across devices: after the
    copy-ins, and at the end of the step (no slot is rewritten while a peer
    may still read it)."""
    import torch
    from fully_sharded_shard_b200 import abi
    from fully_sharded_shard_b200 import peer
    from fully_sharded_shard_b200 import workloads as W
    N = wl.N
    if N % ws:
        raise SystemExit(f"--exchange peer needs N = {N} divisible by the {ws} processes")
    stream = torch.cuda.Stream(device)
    t_setup = time.time()
    hp = dict(W.ADAMW_DEFAULTS)
    shared, instances, plans = [], [], []
    max_A, max_LS = 1, 1
    for gi, grp in enumerate(wl.groups):
        first = peer.PeerGroup(grp.shapes, N, device=device)
        L, S, A, r0 = first.L, first.S, first.P_arena, first.r0
        g = first.g
        for r in range(r0, r0 + L):
            W.fill_grads_bf16(first.grads[r - r0], wl, grp.name, "peer", "pool", 0, r)
            if grp.zero_grad:
                W.zero_param_ranges(first.grads[r - r0], g.arena_off, g.numel, grp.zero_grad)
        P_local = local_real_elems(grp.shapes, g.chunk_rows, r0, L)
        plans.append((g, L, S, A, P_local))
        full = torch.empty(max(A, 1), dtype=torch.float32, device=device)
        master_full = torch.empty(max(N * S, 1), dtype=torch.float32, device=device)
        for rep_i in range(grp.repeat):
            pg = first if rep_i == 0 else peer.PeerGroup(grp.shapes, N, device=device,
                                                          grads=first.grad_buf)
            W.fill_master(full[:A], wl, grp.name, "peer", "layer", rep_i)
            abi.fsdp_shard_params(g, full, master_full)
            master = master_full[r0 * S:(r0 + L) * S].clone()
            m = torch.zeros(L * S, dtype=torch.float32, device=device)
            v = torch.zeros(L * S, dtype=torch.float32, device=device)
            instances.append((gi, pg, master, m, v))
            shared.append(pg)
        del full, master_full
        max_A, max_LS = max(max_A, A), max(max_LS, L * S)
    arenas = [torch.empty(max_A, dtype=torch.bfloat16, device=device) for _ in range(2)]
    reduced = torch.empty(max_LS, dtype=torch.float32, device=device)
    torch.cuda.synchronize(device)
    setup_s = time.time() - t_setup
    state = {"t": 0}

    def one_step(events=None):
        state["t"] += 1

        def timed(name, fn):
            if events is None:
                fn()
                return
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            events[name].append((e0, e1))

        for gi, pg, master, m, v in instances:
            timed("copy_in", lambda: pg.copy_in(master, stream))
        peer.barrier(device)
        for idx, (gi, pg, master, m, v) in enumerate(instances):
            timed("copy_out", lambda: pg.copy_out(arenas[idx % 2], stream))
            timed("rs_reduce", lambda: pg.rs_reduce(wl.op, reduced, stream))
            timed("adamw", lambda: pg.adamw_step(master, m, v, reduced, stream=stream,
                                                 step=state["t"], **hp))
        peer.barrier(device)

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            one_step()
    sampler = ClockSampler(device.index if device.index is not None else 0)
    barrier(device)
    torch.cuda.synchronize(device)
    sampler.start()
    e_start = torch.cuda.Event(enable_timing=True)
    e_end = torch.cuda.Event(enable_timing=True)
    e_start.record(stream)
    with torch.cuda.stream(stream):
        for _ in range(args.steps):
            one_step()
    e_end.record(stream)
    torch.cuda.synchronize(device)
    barrier(device)
    clocks = sampler.stop()
    ms_step = max_over_ranks(e_start.elapsed_time(e_end), device) / args.steps
    events = {k: [] for k in ("copy_in", "copy_out", "rs_reduce", "adamw")}
    with torch.cuda.stream(stream):
        one_step(events)
    torch.cuda.synchronize(device)
    stage_ms = {k: sum(a.elapsed_time(b) for a, b in v) for k, v in events.items()}
    sb = {k: 0 for k in stage_ms}
    xbytes = 0
    P_total = 0
    for gi, pg, master, m, v in instances:
        g, L, S, A, P_local = plans[gi]
        for k, b in peer_stage_bytes(N, S, g.P, L, P_local).items():
            sb[k] += b
        xbytes += peer_exchange_bytes(N, S, L, P_local, ws)
        P_total += g.P
    dev_bytes = sum(sb.values())
    job_bytes = sum_over_ranks(float(dev_bytes), device)
    peak, peak_kind = hbm_peak()
    dom = max(stage_ms, key=stage_ms.get)
    dom_achieved = sb[dom] / (stage_ms[dom] * 1e-3) / 1e9
    kernel_names = {"copy_in": "k_copy_in", "copy_out": "k_copy_out<TAB>",
                    "rs_reduce": "k_reduce_units_tab", "adamw": "k_adamw"}
    out = {
        "metric": METRIC, "value": round(job_bytes / (ms_step * 1e-3) / 1e9, 1), "unit": "GB/s",
        "params_per_s": round(P_total / (ms_step * 1e-3), 1),
        "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms_step, 3), "higher_is_better": True, "scaling": "strong",
        "vs_baseline": None, "dtype": "f32",
        "data": "synthetic: seeded N(0,0.02) fp32 master, N(0,1e-3) bf16 per-rank grads",
        "config": {"workload": wl.name, "N_virtual_ranks": N, "ranks_per_gpu": N // ws,
                   "groups_per_step": len(instances), "params": P_total,
                   "exchange": "pulls over CUDA IPC peer memory (copy-out, reduce-scatter)",
                   "barriers_per_step": 2,
                   "bytes_per_step_per_gpu": dev_bytes,
                   "exchange_bytes_per_step_per_gpu": xbytes,
                   "l2": "inputs larger than L2",
                   "parallelism": f"{ws} GPU(s), {N} virtual ranks, {N // ws} per GPU"},
        "stages": {k: {"ms_per_step": round(stage_ms[k], 3),
                       "GBps": round(sb[k] / (stage_ms[k] * 1e-3) / 1e9, 1)} for k in stage_ms},
        "roofline": {"bound": "hbm", "kernel": kernel_names[dom],
                     "achieved": round(dom_achieved, 1), "peak": peak, "peak_kind": peak_kind,
                     "unit": "GB/s", "frac": round(dom_achieved / peak, 4),
                     "avg_launch_ms": round(stage_ms[dom] / len(instances), 4),
                     "traffic": None},
        "gpu_launches": 4 * len(instances) * args.steps,
        "clocks": clocks, "setup_s": round(setup_s, 1),
    }
    peer.release_all([b for pg in shared for b in pg.buffers()], device)
    return out


def run_peer_pipelined(args, wl, device, rank, ws):
    """The step of run_peer with the devices ordered by CUDA IPC events
    instead of device-draining barriers: one host barrier per step (it waits
    for no device), slots and gradient arenas double buffered by step
    parity, and two streams per device -- the copy-ins and copy-out pulls on
    one, each group's reduce-scatter pulls and AdamW on the other once its
    copy-in has read the master -- so one group's exchange overlaps another
    group's update, and one step's tail overlaps the next step's head (each
    copy-in waits only for its own group's last update)."""
    import torch
    from fully_sharded_shard_b200 import abi
    from fully_sharded_shard_b200 import peer
    from fully_sharded_shard_b200 import workloads as W
    N = wl.N
    if N % ws:
        raise SystemExit(f"--exchange peer needs N = {N} divisible by the {ws} processes")
    s_gather = torch.cuda.Stream(device)
    s_update = torch.cuda.Stream(device)
    t_setup = time.time()
    hp = dict(W.ADAMW_DEFAULTS)
    groups, instances, plans = [], [], []
    max_A, max_LS = 1, 1
    for gi, grp in enumerate(wl.groups):
        first = peer.PipelinedPeerGroup(grp.shapes, N, device=device)
        L, S, A, r0 = first.L, first.S, first.P_arena, first.r0
        g = first.g
        for par in range(2):   # written once: both parities hold the same gradients
            for r in range(r0, r0 + L):
                W.fill_grads_bf16(first.grads[par][r - r0], wl, grp.name, "peer", "pool", 0, r)
                if grp.zero_grad:
                    W.zero_param_ranges(first.grads[par][r - r0], g.arena_off, g.numel,
                                        grp.zero_grad)
        P_local = local_real_elems(grp.shapes, g.chunk_rows, r0, L)
        plans.append((g, L, S, A, P_local))
        full = torch.empty(max(A, 1), dtype=torch.float32, device=device)
        master_full = torch.empty(max(N * S, 1), dtype=torch.float32, device=device)
        for rep_i in range(grp.repeat):
            pg = first if rep_i == 0 else peer.PipelinedPeerGroup(grp.shapes, N, device=device,
                                                                  grads=first)
            W.fill_master(full[:A], wl, grp.name, "peer", "layer", rep_i)
            abi.fsdp_shard_params(g, full, master_full)
            master = master_full[r0 * S:(r0 + L) * S].clone()
            m = torch.zeros(L * S, dtype=torch.float32, device=device)
            v = torch.zeros(L * S, dtype=torch.float32, device=device)
            instances.append((gi, pg, master, m, v))
            if rep_i:
                groups.append(pg)
        groups.append(first)   # closed after the instances sharing its gradients
        del full, master_full
        max_A, max_LS = max(max_A, A), max(max_LS, L * S)
    arenas = [torch.empty(max_A, dtype=torch.bfloat16, device=device) for _ in range(2)]
    reduced = torch.empty(max_LS, dtype=torch.float32, device=device)
    for _, pg, *_ in instances:   # every device's grads are written: record it once
        for par in range(2):
            pg.grads_end(par, s_update)
    torch.cuda.synchronize(device)
    peer.host_barrier()
    setup_s = time.time() - t_setup
    state = {"t": 0}
    n = len(instances)

    def one_step(events=None):
        state["t"] += 1
        t = state["t"]
        par = t % 2

        def timed(name, st, fn):
            if events is None:
                fn()
                return
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(st)
            fn()
            e1.record(st)
            events[name].append((e0, e1))

        # phase A: every group's copy-in, each once its last update is done
        read = []
        for idx, (gi, pg, master, m, v) in enumerate(instances):
            if "updated" in state:
                s_gather.wait_event(state["updated"][idx])
            timed("copy_in", s_gather, lambda: pg.copy_in(par, master, s_gather))
            ev = torch.cuda.Event()
            ev.record(s_gather)
            read.append(ev)
        peer.host_barrier()
        # phase B: the copy-out pulls on one stream, the reduce-scatter pulls
        # and AdamW on the other
        updated = []
        for idx, (gi, pg, master, m, v) in enumerate(instances):
            timed("copy_out", s_gather, lambda: pg.copy_out(par, arenas[idx % 2], s_gather))
            s_update.wait_event(read[idx])
            timed("rs_reduce", s_update, lambda: pg.rs_reduce(par, wl.op, reduced, s_update))
            timed("adamw", s_update, lambda: abi.fsdp_peer_adamw_step(
                pg.pps[par], master, m, v, reduced, step=t, stream=s_update, **hp))
            ev = torch.cuda.Event()
            ev.record(s_update)
            updated.append(ev)
        state["updated"] = updated

    def join():
        """Both streams done: the launching stream waits for the last update."""
        s_gather.wait_event(state["updated"][-1])

    for _ in range(args.warmup):
        one_step()
    join()
    sampler = ClockSampler(device.index if device.index is not None else 0)
    barrier(device)
    torch.cuda.synchronize(device)
    sampler.start()
    e_start = torch.cuda.Event(enable_timing=True)
    e_end = torch.cuda.Event(enable_timing=True)
    e_start.record(s_gather)
    for _ in range(args.steps):
        one_step()
    join()
    e_end.record(s_gather)
    torch.cuda.synchronize(device)
    barrier(device)
    clocks = sampler.stop()
    ms_step = max_over_ranks(e_start.elapsed_time(e_end), device) / args.steps
    events = {k: [] for k in ("copy_in", "copy_out", "rs_reduce", "adamw")}
    one_step(events)
    join()
    torch.cuda.synchronize(device)
    stage_ms = {k: sum(a.elapsed_time(b) for a, b in v) for k, v in events.items()}
    sb = {k: 0 for k in stage_ms}
    xbytes = 0
    P_total = 0
    for gi, pg, master, m, v in instances:
        g, L, S, A, P_local = plans[gi]
        for k, b in peer_stage_bytes(N, S, g.P, L, P_local).items():
            sb[k] += b
        xbytes += peer_exchange_bytes(N, S, L, P_local, ws)
        P_total += g.P
    dev_bytes = sum(sb.values())
    job_bytes = sum_over_ranks(float(dev_bytes), device)
    peak, peak_kind = hbm_peak()
    out = {
        "metric": METRIC, "value": round(job_bytes / (ms_step * 1e-3) / 1e9, 1), "unit": "GB/s",
        "params_per_s": round(P_total / (ms_step * 1e-3), 1),
        "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms_step, 3), "higher_is_better": True, "scaling": "strong",
        "vs_baseline": None, "dtype": "f32",
        "data": "synthetic: seeded N(0,0.02) fp32 master, N(0,1e-3) bf16 per-rank grads",
        "config": {"workload": wl.name, "N_virtual_ranks": N, "ranks_per_gpu": N // ws,
                   "groups_per_step": n, "params": P_total,
                   "exchange": "pulls over CUDA IPC peer memory (copy-out, reduce-scatter)",
                   "ordering": "CUDA IPC events; one host barrier per step, no device sync; "
                               "slots and gradient arenas double buffered by step parity",
                   "bytes_per_step_per_gpu": dev_bytes,
                   "exchange_bytes_per_step_per_gpu": xbytes,
                   "l2": "inputs larger than L2",
                   "parallelism": f"{ws} GPU(s), {N} virtual ranks, {N // ws} per GPU"},
        "stages_in_overlapped_step": {
            k: {"ms_per_step": round(stage_ms[k], 3),
                "GBps": round(sb[k] / (stage_ms[k] * 1e-3) / 1e9, 1)} for k in stage_ms},
        "peak": peak, "peak_kind": peak_kind,
        "gpu_launches": 4 * n * args.steps,
        "clocks": clocks, "setup_s": round(setup_s, 1),
    }
    torch.cuda.synchronize(device)
    for pg in groups:
        pg.close()
    return out


def staged_rs_bytes(N: int, S: int, P: int) -> int:
    """The reduce-scatter with the packed buffer materialised: the pack reads
    every rank's gradients (2 B per real element per rank) and writes the
    fp32 packed buffer [N][N][S]; the reduction reads it back and writes
    [N][S]: (2N + 8N + 4) B per unpadded parameter, the fused path + 8N."""
    Pp = N * S
    return 2 * N * P + 4 * N * Pp + 4 * N * Pp + 4 * Pp


def run_staged(args, model, device, stream):
    """The reduce-scatter of the largest repeated group through the staged
    path (materialised fp32 packed buffer, pack then rank-ordered reduction)
    against the fused path on the same gradients, each under its own byte
    model."""
    import torch
    from fully_sharded_shard_b200 import abi
    gi = max(range(len(model.plans)), key=lambda i: model.wl.groups[i].repeat)
    g = model.plans[gi]
    grads = model.grads[gi][0]
    N = g.N
    packed = torch.empty(N * N * g.S, dtype=torch.float32, device=device)

    def timed(fn):
        with torch.cuda.stream(stream):
            for _ in range(max(1, args.warmup)):
                fn()
        torch.cuda.synchronize(device)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(max(1, args.steps)):
            fn()
        e1.record(stream)
        torch.cuda.synchronize(device)
        return e0.elapsed_time(e1) / max(1, args.steps)

    ms_staged = timed(lambda: abi.fsdp_rs_reduce(g, grads, model.wl.op, model.reduced,
                                                 packed=packed, stream=stream))
    ms_fused = timed(lambda: abi.fsdp_rs_reduce(g, grads, model.wl.op, model.reduced,
                                                stream=stream))
    b_staged = staged_rs_bytes(N, g.S, g.P)
    b_fused = 2 * N * g.P + 4 * N * g.S
    del packed
    return {"group": model.wl.groups[gi].name, "params": g.P,
            "staged_ms": round(ms_staged, 3), "staged_bytes": b_staged,
            "staged_GBps": round(b_staged / (ms_staged * 1e-3) / 1e9, 1),
            "fused_ms": round(ms_fused, 3), "fused_bytes": b_fused,
            "fused_GBps": round(b_fused / (ms_fused * 1e-3) / 1e9, 1),
            "speedup_fused_over_staged": round(ms_staged / ms_fused, 3)}


def run_accumulate(args, model, device, stream, micro: int = 4):
    """Gradient accumulation without sync on the largest repeated group:
    micro - 1 accumulations into fp32 per-rank arenas, then the reduce-scatter
    fused with the last microbatch.  Own byte model: 6 (first) or 10 bytes per
    arena element per accumulation; 6N per real element + 4 per padded
    element for the last microbatch."""
    import torch
    from fully_sharded_shard_b200 import abi
    gi = max(range(len(model.plans)), key=lambda i: model.wl.groups[i].repeat)
    g = model.plans[gi]
    pool = model.grads[gi]
    N = g.N
    acc = torch.empty(N * g.P_arena, dtype=torch.float32, device=device)

    def one():
        for t in range(micro - 1):
            abi.fsdp_grad_accumulate(g, pool[t % len(pool)], acc, first=(t == 0), stream=stream)
        abi.fsdp_rs_reduce_accumulated(g, pool[(micro - 1) % len(pool)], acc, model.wl.op,
                                       model.reduced, stream=stream)

    with torch.cuda.stream(stream):
        for _ in range(max(1, args.warmup)):
            one()
    torch.cuda.synchronize(device)
    reps = max(1, args.steps)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        one()
    e1.record(stream)
    torch.cuda.synchronize(device)
    ms = e0.elapsed_time(e1) / reps
    A = N * g.P_arena
    b = 6 * A + 10 * A * (micro - 2) + 6 * N * g.P + 4 * N * g.S
    del acc
    return {"group": model.wl.groups[gi].name, "microbatches": micro, "params": g.P,
            "ms_per_group_step": round(ms, 3), "bytes": b,
            "value": round(b / (ms * 1e-3) / 1e9, 1), "unit": "GB/s (own byte model)",
            "launches": micro}


def run_fp8(args, model, device, stream):
    """The all-gather half of the step in FP8 (per-parameter scales, E4M3
    copy-in, byte copy-out) against the same half in bf16, over every group
    of the model.  Own byte models: FP8 = 4 B per real element (amax pass) +
    5 B per padded element + 2 B per real element; bf16 = 6 + 4 B."""
    import torch
    from fully_sharded_shard_b200 import abi
    max_NS = max(model.wl.N * g.S for g in model.plans)
    max_A = max(g.P_arena for g in model.plans)
    ag8 = torch.empty(max(max_NS, 1), dtype=torch.uint8, device=device)
    ar8 = torch.empty(max(max_A, 1), dtype=torch.uint8, device=device)
    scales = [torch.empty(max(g.n, 1), dtype=torch.float32, device=device) for g in model.plans]

    def fp8_half():
        for gi, master, m, v, pj in model.instances:
            g = model.plans[gi]
            abi.fsdp_copy_in_fp8(g, master, ag8, scales[gi], stream)
            abi.fsdp_copy_out_fp8(g, ag8, ar8, stream)

    def bf16_half():
        for gi, master, m, v, pj in model.instances:
            g = model.plans[gi]
            abi.fsdp_copy_in(g, master, model.ag, stream)
            abi.fsdp_copy_out(g, model.ag, model.arena, stream)

    def timed(fn):
        with torch.cuda.stream(stream):
            fn()
        torch.cuda.synchronize(device)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(max(1, args.steps)):
            fn()
        e1.record(stream)
        torch.cuda.synchronize(device)
        return e0.elapsed_time(e1) / max(1, args.steps)

    ms8 = timed(fp8_half)
    ms16 = timed(bf16_half)
    N = model.wl.N
    b8 = sum(4 * model.plans[i[0]].P + 5 * N * model.plans[i[0]].S + 2 * model.plans[i[0]].P
             for i in model.instances)
    b16 = sum(6 * N * model.plans[i[0]].S + 2 * N * model.plans[i[0]].S + 2 * model.plans[i[0]].P
              for i in model.instances)
    del ag8, ar8
    return {"fp8_ms_per_step": round(ms8, 3), "fp8_bytes": b8,
            "fp8_GBps": round(b8 / (ms8 * 1e-3) / 1e9, 1),
            "bf16_ms_per_step": round(ms16, 3), "bf16_bytes": b16,
            "bf16_GBps": round(b16 / (ms16 * 1e-3) / 1e9, 1),
            "all_gather_payload_ratio": 0.5,
            "launches_per_step": 2 * len(model.instances) + 3 * len(model.instances)}


def run_latency(device, reps: int = 200, graph_steps: int = 20):
    """The tiny MLP group (4 parameters, N = 2) is launch-bound: report the
    step latency in microseconds, eager (host-side AdamW step count) and as a
    replayed CUDA graph of `graph_steps` whole steps, whose AdamW step count
    lives in device memory so that every step in it is the next training
    step.  One graph holds several steps so that the device time per step is
    measured, not the host's graph-launch rate."""
    import torch
    from fully_sharded_shard_b200 import abi
    from fully_sharded_shard_b200 import workloads as W
    wl = W.tiny_mlp()
    model = Model(wl, device, 1, 0)
    stream = torch.cuda.Stream(device)
    with torch.cuda.stream(stream):
        for _ in range(10):
            model.step(stream)
    torch.cuda.synchronize(device)

    def timed(fn):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize(device)
        return e0.elapsed_time(e1) * 1e3 / reps

    t0 = time.perf_counter()
    eager_us = timed(lambda: model.step(stream))
    host_us = (time.perf_counter() - t0) * 1e6 / reps

    ds = abi.DeviceStep(device)
    hp = dict(W.ADAMW_DEFAULTS)

    def graphed_step():
        abi.fsdp_adamw_prepare(ds, stream=stream, **hp)
        for gi, master, m, v, pj in model.instances:
            g = model.plans[gi]
            abi.fsdp_copy_in(g, master, model.ag, stream)
            abi.fsdp_copy_out(g, model.ag, model.arena, stream)
            abi.fsdp_rs_reduce(g, model.grads[gi][pj], wl.op, model.reduced, stream=stream)
            abi.fsdp_adamw_step_dev(g, master, m, v, model.reduced, ds, stream=stream)

    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for _ in range(graph_steps):
            graphed_step()
    torch.cuda.synchronize(device)
    with torch.cuda.stream(stream):
        graph.replay()
        graph_us = timed(graph.replay) / graph_steps
    del graph

    # the same step through fsdp_group_step: one call per group, and one
    # single-CTA launch for a group this small
    state = {"t": 0}

    def single_call_step():
        state["t"] += 1
        for gi, master, m, v, pj in model.instances:
            g = model.plans[gi]
            abi.fsdp_group_step(g, master, m, v, model.grads[gi][pj], wl.op, step=state["t"],
                                ag=model.ag, arena=model.arena, reduced=model.reduced,
                                stream=stream, **hp)

    for _ in range(10):
        single_call_step()
    t0 = time.perf_counter()
    single_us = timed(single_call_step)
    single_host_us = (time.perf_counter() - t0) * 1e6 / reps

    def graphed_single():
        abi.fsdp_adamw_prepare(ds, stream=stream, **hp)
        for gi, master, m, v, pj in model.instances:
            g = model.plans[gi]
            abi.fsdp_group_step_dev(g, master, m, v, model.grads[gi][pj], wl.op, ds,
                                    ag=model.ag, arena=model.arena, reduced=model.reduced,
                                    stream=stream)

    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for _ in range(graph_steps):
            graphed_single()
    torch.cuda.synchronize(device)
    with torch.cuda.stream(stream):
        graph.replay()
        graph_single_us = timed(graph.replay) / graph_steps
    del graph
    # one call per group that also advances the step counter: one launch per
    # step for a small group, no separate prepare kernel
    ds2 = abi.DeviceStep(device)

    def graphed_one_call():
        for gi, master, m, v, pj in model.instances:
            g = model.plans[gi]
            abi.fsdp_group_step_graph(g, master, m, v, model.grads[gi][pj], wl.op, ds2,
                                      ag=model.ag, arena=model.arena, reduced=model.reduced,
                                      stream=stream, **hp)

    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for _ in range(graph_steps):
            graphed_one_call()
    torch.cuda.synchronize(device)
    with torch.cuda.stream(stream):
        graph.replay()
        graph_one_call_us = timed(graph.replay) / graph_steps
    del graph
    n_small = sum(1 for gi, *_ in model.instances
                  if wl.N * model.plans[gi].S <= abi.FSDP_SMALL_STEP_ELEMS)
    single_launches = sum(1 if wl.N * model.plans[gi].S <= abi.FSDP_SMALL_STEP_ELEMS else 4
                          for gi, *_ in model.instances)
    return {"workload": wl.name, "launches_per_step": model.launches_per_step,
            "eager_us_per_step": round(eager_us, 2), "eager_host_us_per_step": round(host_us, 2),
            "graph_us_per_step": round(graph_us, 2),
            "graph_steps_per_replay": graph_steps,
            "graph_launches_per_step": model.launches_per_step + 1,
            "group_step": {"groups_in_one_launch": n_small,
                           "launches_per_step": single_launches,
                           "eager_us_per_step": round(single_us, 2),
                           "eager_host_us_per_step": round(single_host_us, 2),
                           "graph_us_per_step": round(graph_single_us, 2),
                           "graph_launches_per_step": single_launches + 1},
            "group_step_graph": {"graph_us_per_step": round(graph_one_call_us, 2),
                                 "graph_launches_per_step": sum(
                                     1 if wl.N * model.plans[gi].S <= abi.FSDP_SMALL_STEP_ELEMS
                                     else 5 for gi, *_ in model.instances)}}


def run_e2e(args, model, device, stream, ws):
    """The same step through the public API with the gradients starting in
    pinned host memory: every group's H2D copy (on a copy stream, double
    buffered so group g+1's copy overlaps group g's kernels) and a D2H read
    of the step's last updated parameter are inside the timed region."""
    import torch
    N = model.wl.N
    host = []
    dev = []
    for gi, g in enumerate(model.plans):
        h = torch.empty(N, g.P_arena, dtype=torch.bfloat16, pin_memory=True)
        h.copy_(model.grads[gi][0])
        host.append(h)
        dev.append([torch.empty_like(model.grads[gi][0]) for _ in range(2)])
    copy_stream = torch.cuda.Stream(device)
    result = torch.empty(1, dtype=torch.float32, pin_memory=True)
    n_inst = len(model.instances)
    h2d_bytes = sum(host[gi].numel() * 2 for gi, *_ in model.instances)

    def one_step():
        model.step_count += 1
        ready = [None] * n_inst   # H2D of group idx done (copy stream)
        freed = [None] * n_inst   # group idx's kernels done with its buffer

        def issue(idx):
            gi = model.instances[idx][0]
            buf = dev[gi][idx % 2]
            if idx >= 2:
                copy_stream.wait_event(freed[idx - 2])
            with torch.cuda.stream(copy_stream):
                buf.copy_(host[gi], non_blocking=True)
            ev = torch.cuda.Event()
            ev.record(copy_stream)
            ready[idx] = ev
            return buf

        # the previous step's kernels may still read both buffers
        prev_done = torch.cuda.Event()
        prev_done.record(stream)
        copy_stream.wait_event(prev_done)
        bufs = [None] * n_inst
        for idx in range(min(2, n_inst)):
            bufs[idx] = issue(idx)
        for idx in range(n_inst):
            stream.wait_event(ready[idx])
            model.run_group(idx, stream, model.step_count, grads=bufs[idx])
            ev = torch.cuda.Event()
            ev.record(stream)
            freed[idx] = ev
            if idx + 2 < n_inst:
                bufs[idx + 2] = issue(idx + 2)
        last = model.instances[-1][1]
        with torch.cuda.stream(stream):
            result.copy_(last[:1], non_blocking=True)

    steps = max(1, min(args.steps, args.e2e_steps))
    with torch.cuda.stream(stream):
        one_step()
    torch.cuda.synchronize(device)
    barrier(device)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    with torch.cuda.stream(stream):
        for _ in range(steps):
            one_step()
    e1.record(stream)
    torch.cuda.synchronize(device)
    _ = float(result.item())
    ms = max_over_ranks(e0.elapsed_time(e1) / steps, device)
    return {"value": round(ws * model.bytes_per_step / (ms * 1e-3) / 1e9, 1), "unit": "GB/s",
            "ms_per_step": round(ms, 2), "steps": steps,
            "h2d_bytes_per_step": int(h2d_bytes), "d2h_bytes_per_step": 4}


def workload_summary(args, name, device, rank, ws):
    """Another workload after the headline one (its state freed first): the
    five-stage step on two streams, each stage timed alone (events around
    every launch, one stream), and the fused step, as GB/s and fractions of
    the HBM peak under the same byte models."""
    import argparse as _ap
    import gc
    import torch
    from fully_sharded_shard_b200 import workloads as W
    gc.collect()
    torch.cuda.empty_cache()
    sub = _ap.Namespace(**vars(args))
    for flag in ("no_e2e", "no_accumulate", "no_latency", "no_fp8", "no_staged"):
        setattr(sub, flag, True)
    sub.no_fused = False
    wl = W.by_name(name)
    out, model = run_ours(sub, wl, device, rank, ws)
    del model
    gc.collect()
    torch.cuda.empty_cache()
    peak = out["roofline"]["peak"]
    fused = out["fused_step"]
    return {
        "N_virtual_ranks": wl.N, "reduce_op": W.OP_NAMES[wl.op], "params": out["config"]["params"],
        "groups_per_step": out["config"]["groups_per_step"],
        "value": out["value"], "unit": "GB/s", "ms_per_step": out["ms_per_step"],
        "ms_per_step_median": out["ms_per_step_median"],
        "frac_of_peak": round(out["value"] / ws / peak, 4),
        "stages": out["stages"],
        "fused_step": {
            "ms_per_step": fused["ms_per_step"], "value": fused["value"],
            "frac_of_peak": fused["frac_of_measured_peak"],
            "stages": {k: dict(v, frac_of_peak=round(v["GBps"] / peak, 4))
                       for k, v in fused["stages"].items()},
        },
        "peak": peak, "peak_kind": out["roofline"]["peak_kind"],
        "clocks": out["clocks"],
        "gpu_launches": out["gpu_launches"],
    }


# ---------------------------------------------------------------------------
# the oracle on the host cores (CPU baseline and the reference arm)
# ---------------------------------------------------------------------------
def oracle_sample(wl):
    """One block group of the workload (the unit the step repeats)."""
    from fully_sharded_shard_b200 import workloads as W
    grp = max(wl.groups, key=lambda g: g.repeat)
    return grp


def oracle_pass(O, p, full, grads, wl, state, step):
    """One oracle step over one group: copy-in, copy-out, reduce-scatter
    (direct form), AdamW."""
    master, m, v = state
    ag = O.copy_in(p, master)
    O.copy_out(p, ag)
    red = O.reduce_scatter_direct(p, grads, wl.op)
    O.adamw(master, m, v, red, step=step, lr=3e-4, beta1=0.9, beta2=0.999, eps=1e-8,
            weight_decay=0.01)


def oracle_setup(wl):
    import numpy as np
    import oracle as O
    O.build()
    grp = oracle_sample(wl)
    p = O.plan(grp.shapes, wl.N)
    rng = np.random.default_rng(0)
    full = (rng.standard_normal(p.P_arena, dtype=np.float32) * np.float32(0.02))
    bits = (rng.standard_normal(wl.N * p.P_arena, dtype=np.float32) * np.float32(1e-3)).view(np.uint32)
    grads = O.bf16_bits_from_u32(bits)
    del bits
    master = O.shard(p, full)
    state = (master, np.zeros_like(master), np.zeros_like(master))
    return O, grp, p, full, grads, state


def cpu_model() -> str:
    """The host CPU's model name and logical core count."""
    name = "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    name = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return f"{name} ({os.cpu_count()} logical cores)"


def cpu_baseline(wl, min_seconds: float):
    """The oracle on the host cores: all threads for >= min_seconds, then one
    single-threaded pass; both over one group of the workload, the full-step
    time extrapolated from the per-element rate."""
    O, grp, p, full, grads, state = oracle_setup(wl)
    cores = O.get_threads()
    t0 = time.time()
    passes = 0
    while True:
        passes += 1
        oracle_pass(O, p, full, grads, wl, state, passes)
        if time.time() - t0 >= min_seconds:
            break
    dt = (time.time() - t0) / passes
    O.set_threads(1)
    t1 = time.time()
    oracle_pass(O, p, full, grads, wl, state, passes + 1)
    dt1 = time.time() - t1
    O.set_threads(cores)
    b = group_bytes(wl.N, p.S, p.P)
    step_params = wl.total_params()
    return {"value": round(b / dt / 1e9, 3), "unit": "GB/s", "cores": cores, "kind": "oracle",
            "cpu": cpu_model(),
            "params_per_s": round(p.P / dt, 1),
            "value_1core": round(b / dt1 / 1e9, 3),
            "extrapolated_full_step_s": round(dt * step_params / p.P, 1),
            "extrapolated_full_step_s_1core": round(dt1 * step_params / p.P, 1),
            "sample": f"{passes} oracle pass(es) over one '{grp.name}' group of {wl.name} "
                      f"({p.P} params, N={wl.N}): copy-in, copy-out, reduce-scatter, AdamW; "
                      f"{dt:.2f} s per pass on {cores} threads (OpenMP), {dt1:.2f} s on 1 thread; "
                      f"full step extrapolated by parameter count"}


def run_reference(args, wl):
    O, grp, p, full, grads, state = oracle_setup(wl)
    cores = O.get_threads()
    for k in range(args.warmup):
        oracle_pass(O, p, full, grads, wl, state, k + 1)
    t0 = time.time()
    for k in range(args.steps):
        oracle_pass(O, p, full, grads, wl, state, args.warmup + k + 1)
    dt = (time.time() - t0) / args.steps
    b = group_bytes(wl.N, p.S, p.P)
    val = round(b / dt / 1e9, 3)
    sample = (f"each step: one oracle pass over one '{grp.name}' group of {wl.name} "
              f"({p.P} params, N={wl.N}) on {cores} host threads")
    return {
        "impl": "reference", "metric": METRIC, "value": val, "unit": "GB/s",
        "params_per_s": round(p.P / dt, 1), "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(dt * 1e3, 2), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic: seeded N(0,0.02) fp32 master, N(0,1e-3) bf16 per-rank grads",
        "config": {"workload": wl.name, "N_virtual_ranks": wl.N,
                   "sample_group": grp.name, "params_per_sample": p.P},
        "cpu_baseline": {"value": val, "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "cpu": cpu_model(), "sample": sample},
        "e2e": {"value": val, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# ---------------------------------------------------------------------------
def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="llama7b")
    ap.add_argument("--grad-pool", type=int, default=8)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-fused", action="store_true")
    ap.add_argument("--no-accumulate", action="store_true")
    ap.add_argument("--no-latency", action="store_true")
    ap.add_argument("--no-fp8", action="store_true")
    ap.add_argument("--no-staged", action="store_true")
    ap.add_argument("--one-stream", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--extra-workloads", default="uneven,moe,small_params",
                    help="comma-separated workloads timed after the headline one (per-stage "
                         "GB/s of the five-stage and the fused step); empty for none")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--exchange", choices=["replicas", "peer"], default="replicas",
                    help="replicas: one full N-rank replica per GPU (weak scaling); peer: one "
                         "model whose N ranks are spread over the GPUs, exchanged as pulls "
                         "over peer memory (strong scaling)")
    ap.add_argument("--peer-sync", choices=["barriers", "events"], default="events",
                    help="--exchange peer: order the devices by CUDA IPC events with one host "
                         "barrier per step (events), or by two device-draining barriers per "
                         "step (barriers)")
    ap.add_argument("--backend", choices=["nccl", "gloo"], default="nccl",
                    help="process-group backend for N > 1 (gloo lets several processes share "
                         "one GPU, to exercise --exchange peer without several GPUs)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)

    from fully_sharded_shard_b200 import workloads as W
    wl = W.by_name(args.workload)
    ws, rank, local = dist_env()

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, wl)), flush=True)
        return 0

    import torch
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    device = torch.device("cuda", local % torch.cuda.device_count())
    torch.cuda.set_device(device)
    if ws > 1:
        init_dist(args.backend)
    if args.exchange == "peer":
        if args.peer_sync == "events":
            out = run_peer_pipelined(args, wl, device, rank, ws)
        else:
            out = run_peer(args, wl, device, rank, ws)
        if rank == 0:
            print(json.dumps(out), flush=True)
        if ws > 1:
            import torch.distributed as dist
            barrier(device)
            dist.destroy_process_group()
        return 0
    out, model = run_ours(args, wl, device, rank, ws)
    del model
    extra = [w for w in args.extra_workloads.split(",") if w and w != wl.name]
    if extra:
        out["workloads"] = {}
        for name in extra:
            out["workloads"][name] = workload_summary(args, name, device, rank, ws)
    if rank == 0 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(wl, args.cpu_seconds)
    if rank == 0:
        print(json.dumps(out), flush=True)
    if ws > 1:
        import torch.distributed as dist
        barrier(device)
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
