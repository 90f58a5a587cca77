"""Helpers for the GPU parity tests: run one parameter group through the
C-ABI kernels and through the CPU oracle on identical seeded inputs, and
compare (bit-exact for data movement and reduction, 1e-6 * (1 + |x|) for
AdamW).

Buffers are allocated with guard bands on both sides, filled with a
sentinel and checked after every call, so an out-of-range write shows up
as a failure.
"""
from __future__ import annotations

import json
import os

import numpy as np
import torch

import oracle
from fully_sharded_shard_b200 import abi
from fully_sharded_shard_b200 import workloads as W

GUARD = 64  # elements on each side (a multiple of 16 bytes for every dtype here)
ADAM_TOL = 1e-6


def log_parity(path: str, wl: W.Workload, group: W.Group, g: abi.Group, **rec) -> None:
    """One JSON line per passed parity case, appended to $FSDPK_PARITY_LOG
    when it is set: the case, the stages compared bit for bit and the largest
    AdamW difference as a fraction of the tolerance."""
    out = os.environ.get("FSDPK_PARITY_LOG")
    if not out:
        return
    rec = {"path": path, "workload": wl.name, "group": group.name, "N": wl.N, "n_params": g.n,
           "S": g.S, "P": g.P, **rec}
    with open(out, "a") as f:
        f.write(json.dumps(rec) + "\n")


class Guarded:
    """A device buffer with sentinel guard bands before and after it."""

    def __init__(self, n: int, dtype, device="cuda", fill=None):
        self.n = n
        self.full = torch.empty(n + 2 * GUARD, dtype=dtype, device=device)
        if dtype == torch.float32:
            self.full.fill_(-12345.5)
        elif dtype == torch.uint8:
            self.full.fill_(0x5A)
        else:
            self.full.view(torch.int16).fill_(0x3BEF)
        self.t = self.full[GUARD:GUARD + n]
        if fill is not None:
            self.t.copy_(fill)

    def guards_intact(self) -> bool:
        if self.full.dtype == torch.float32:
            s = torch.tensor(-12345.5, dtype=torch.float32, device=self.full.device)
            lo, hi = self.full[:GUARD], self.full[GUARD + self.n:]
            return bool((lo == s).all() and (hi == s).all())
        if self.full.dtype == torch.uint8:
            return bool((self.full[:GUARD] == 0x5A).all() and (self.full[GUARD + self.n:] == 0x5A).all())
        v = self.full.view(torch.int16)
        return bool((v[:GUARD] == 0x3BEF).all() and (v[GUARD + self.n:] == 0x3BEF).all())


def u16(t: torch.Tensor) -> np.ndarray:
    return t.detach().view(torch.int16).cpu().numpy().view(np.uint16).reshape(-1)


def f32(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy().reshape(-1)


def bits_equal(a: np.ndarray, b: np.ndarray) -> bool:
    a = np.asarray(a)
    b = np.asarray(b)
    if a.dtype == np.float32:
        a = a.view(np.uint32)
    if b.dtype == np.float32:
        b = b.view(np.uint32)
    return a.shape == b.shape and bool(np.array_equal(a, b))


def first_mismatch(a, b) -> str:
    a = np.asarray(a).reshape(-1)
    b = np.asarray(b).reshape(-1)
    if a.dtype == np.float32:
        a, b = a.view(np.uint32), b.view(np.uint32)
    bad = np.nonzero(a != b)[0]
    if bad.size == 0:
        return "no mismatch"
    k = int(bad[0])
    return f"{bad.size} mismatches, first at {k}: gpu={a[k]:#x} oracle={b[k]:#x}"


def _nan_mask(a: np.ndarray, kind: str) -> np.ndarray:
    if kind == "bf16":
        return ((a & 0x7F80) == 0x7F80) & ((a & 0x007F) != 0)
    if kind == "f32":
        return ((a & 0x7F800000) == 0x7F800000) & ((a & 0x007FFFFF) != 0)
    if kind == "e4m3":
        return (a & 0x7F) == 0x7F
    raise ValueError(kind)


def equal_nan_class(a, b, kind: str) -> bool:
    """Bit-exact equality of two bit-pattern arrays (uint16 bf16, uint32 /
    float32 binary32, uint8 E4M3) where any NaN matches any NaN: the pages fix
    no NaN encoding, so a NaN is compared as a class; every other pattern,
    signed zeros and infinities included, must match bit for bit."""
    a = np.asarray(a).reshape(-1)
    b = np.asarray(b).reshape(-1)
    if a.dtype == np.float32:
        a = a.view(np.uint32)
    if b.dtype == np.float32:
        b = b.view(np.uint32)
    if a.shape != b.shape:
        return False
    na, nb = _nan_mask(a, kind), _nan_mask(b, kind)
    return bool(np.array_equal(na, nb) and np.array_equal(a[~na], b[~nb]))


def adam_close_special(gpu: np.ndarray, ref: np.ndarray, tol: float = ADAM_TOL):
    """The AdamW bar max |gpu - ref| <= tol * (1 + |ref|) on finite values;
    infinities must be equal and NaN must meet NaN."""
    g = gpu.astype(np.float64).reshape(-1)
    r = ref.astype(np.float64).reshape(-1)
    gn, rn = np.isnan(g), np.isnan(r)
    if not np.array_equal(gn, rn):
        return False, float("inf")
    gi, ri = np.isinf(g), np.isinf(r)
    if not np.array_equal(gi, ri) or not np.array_equal(g[gi], r[ri]):
        return False, float("inf")
    fin = ~(gn | gi)
    return adam_close(g[fin].astype(np.float32), r[fin].astype(np.float32), tol)


def adamw_from_state(p, m, v, g, step: int, hp: dict):
    """The oracle's AdamW applied to copies of a given pre-step state."""
    p, m, v = p.copy(), m.copy(), v.copy()
    oracle.adamw(p, m, v, g, step=step, **hp)
    return p, m, v


def adam_close(gpu: np.ndarray, ref: np.ndarray, tol: float = ADAM_TOL):
    d = np.abs(gpu.astype(np.float64) - ref.astype(np.float64))
    lim = tol * (1.0 + np.abs(ref.astype(np.float64)))
    ok = bool(np.all(d <= lim))
    return ok, float(np.max(d / lim)) if d.size else 0.0


def check_plan(g: abi.Group, p: oracle.Plan) -> None:
    assert abi.fsdp_group_check(g) == 0, "the plan's work tables are inconsistent"
    assert (g.S, g.P, g.P_arena) == (p.S, p.P, p.P_arena)
    assert list(g.shard_off) == [int(x) for x in p.shard_off]
    assert list(g.arena_off) == [int(x) for x in p.arena_off]
    assert list(g.chunk_rows) == [int(x) for x in p.chunk_rows]


def make_grads(g: abi.Group, wl: W.Workload, group: W.Group, step: int, tag=()) -> torch.Tensor:
    """Per-rank bf16 gradients [N][P_arena] on the device, seeded per rank."""
    grads = torch.empty(g.N, g.P_arena, dtype=torch.bfloat16, device="cuda")
    for r in range(g.N):
        W.fill_grads_bf16(grads[r], wl, group.name, *tag, step, r)
        if group.zero_grad:
            W.zero_param_ranges(grads[r], g.arena_off, g.numel, group.zero_grad)
    return grads


def _initial_master(g, p, wl, group, tag, full_init):
    """The full fp32 parameters (seeded, or `full_init` in the arena layout),
    sharded on the GPU and in the oracle; the two must agree bit for bit."""
    NS = g.N * g.S
    full = torch.empty(max(g.P_arena, 1), dtype=torch.float32, device="cuda")
    if full_init is None:
        W.fill_master(full, wl, group.name, *tag)
    else:
        full.zero_()
        full[:g.P_arena].copy_(torch.from_numpy(np.ascontiguousarray(full_init, np.float32)))
    master = Guarded(NS, torch.float32)
    abi.fsdp_shard_params(g, full, master.t)
    torch.cuda.synchronize()
    assert master.guards_intact(), "shard wrote outside master"
    master_o = oracle.shard(p, f32(full)[:p.P_arena] if p.P_arena else np.zeros(0, np.float32))
    assert bits_equal(f32(master.t), master_o), "shard: " + first_mismatch(f32(master.t), master_o)
    return master, master_o


def _grads_for(g, wl, group, step, tag, grads_init):
    if grads_init is None:
        return make_grads(g, wl, group, step, tag)
    h = np.ascontiguousarray(grads_init(step), np.uint16).reshape(g.N, g.P_arena)
    return torch.from_numpy(h.view(np.int16)).to("cuda").view(torch.bfloat16)


def _adam_check(report, what, step, gpu_state, ref_state):
    for name, gbuf, obuf in zip(("master", "m", "v"), gpu_state, ref_state):
        ok, ratio = adam_close_special(gbuf, obuf)
        report["adam_max_ratio"] = max(report["adam_max_ratio"], ratio)
        assert ok, f"{what} {name} step {step}: max |d|/tol = {ratio}"


def run_group(wl: W.Workload, group: W.Group, *, steps: int = 1, ops=None, staged: bool = True,
              direct_oracle: bool = False, tag=(), full_init=None, grads_init=None) -> dict:
    """Run shard -> copy-in -> copy-out -> reduce-scatter -> AdamW on the GPU and
    in the oracle for `steps` steps; assert parity at every stage.

    Every stage is checked against the oracle applied to the GPU's own inputs
    at that stage: copy-in from the GPU's master, copy-out from the GPU's
    all-gather buffer, AdamW from the GPU's pre-step master, m and v and its
    reduced gradient (data movement and reduction bit for bit, NaN compared
    as a class where arithmetic makes it; AdamW within 1e-6 * (1 + |x|)).
    Over several steps the GPU's AdamW state is also held to the oracle's own
    trajectory within that bar.  full_init (fp32, arena layout) and
    grads_init (step -> uint16 [N][P_arena]) replace the seeded inputs.
    Returns a small report."""
    N = wl.N
    g = abi.fsdp_plan_group(group.shapes, N)
    p = oracle.plan(group.shapes, N)
    check_plan(g, p)
    NS = N * g.S
    report = {"S": g.S, "P": g.P, "N": N, "adam_max_ratio": 0.0}
    ops = [wl.op] if ops is None else list(ops)
    master, master_o = _initial_master(g, p, wl, group, tag, full_init)
    m = Guarded(NS, torch.float32, fill=torch.zeros(NS))
    v = Guarded(NS, torch.float32, fill=torch.zeros(NS))
    m_o = np.zeros(NS, np.float32)
    v_o = np.zeros(NS, np.float32)
    hp = dict(W.ADAMW_DEFAULTS)

    for step in range(1, steps + 1):
        pre = (f32(master.t), f32(m.t), f32(v.t))
        # stage 1: copy-in, against the oracle's copy-in of the GPU's master
        ag = Guarded(NS, torch.bfloat16)
        abi.fsdp_copy_in(g, master.t, ag.t)
        torch.cuda.synchronize()
        assert ag.guards_intact(), "copy-in wrote outside ag"
        ag_h = u16(ag.t)
        ag_o = oracle.copy_in(p, pre[0])
        assert equal_nan_class(ag_h, ag_o, "bf16"), "copy-in: " + first_mismatch(ag_h, ag_o)

        # stage 2: copy-out of the GPU's buffer (a bit move: NaN bits too;
        # gaps keep their sentinel on both sides)
        arena = Guarded(g.P_arena, torch.bfloat16)
        abi.fsdp_copy_out(g, ag.t, arena.t)
        torch.cuda.synchronize()
        assert arena.guards_intact(), "copy-out wrote outside the arena"
        arena_o = oracle.copy_out(p, ag_h, np.full(p.P_arena, 0x3BEF, np.uint16))
        arena_h = u16(arena.t)
        assert bits_equal(arena_h, arena_o), "copy-out: " + first_mismatch(arena_h, arena_o)
        del ag, arena

        # stages 3 + 4: reduce-scatter (the same gradients on both sides)
        grads = _grads_for(g, wl, group, step, tag, grads_init)
        grads_h = u16(grads)
        red = None
        for op in ops:
            red = Guarded(NS, torch.float32)
            abi.fsdp_rs_reduce(g, grads, op, red.t)
            torch.cuda.synchronize()
            assert red.guards_intact(), "reduce wrote outside reduced"
            if direct_oracle:
                red_o = oracle.reduce_scatter_direct(p, grads_h, op)
            else:
                red_o = oracle.reduce_scatter(p, grads_h, op)
            assert equal_nan_class(f32(red.t), red_o, "f32"), \
                f"rs fused {W.OP_NAMES[op]}: " + first_mismatch(f32(red.t), red_o)
            if staged:
                packed = Guarded(N * NS, torch.float32)
                red2 = Guarded(NS, torch.float32)
                abi.fsdp_rs_reduce(g, grads, op, red2.t, packed=packed.t)
                torch.cuda.synchronize()
                assert packed.guards_intact() and red2.guards_intact()
                packed_o = oracle.pack(p, grads_h)
                assert bits_equal(f32(packed.t), packed_o), "pack: " + first_mismatch(f32(packed.t), packed_o)
                assert equal_nan_class(f32(red2.t), red_o, "f32"), \
                    f"rs staged {W.OP_NAMES[op]}: " + first_mismatch(f32(red2.t), red_o)
                del packed, red2
        del grads

        # stage 5: AdamW on the last op's reduced gradient, against the oracle
        # from the GPU's own pre-step state, then against the oracle's own
        # trajectory (both sides start from the seeded master at step 1)
        red_h = f32(red.t)
        abi.fsdp_adamw_step(g, master.t, m.t, v.t, red.t, step=step, **hp)
        torch.cuda.synchronize()
        assert master.guards_intact() and m.guards_intact() and v.guards_intact()
        post = (f32(master.t), f32(m.t), f32(v.t))
        _adam_check(report, "adamw", step, post, adamw_from_state(*pre, red_h, step, hp))
        oracle.adamw(master_o, m_o, v_o, red_o, step=step, **hp)
        _adam_check(report, "adamw trajectory", step, post, (master_o, m_o, v_o))
    log_parity("stages", wl, group, g, steps=steps, ops=[W.OP_NAMES[o] for o in ops],
               bit_exact=["shard", "copy_in", "copy_out", "rs_fused"] + (["pack", "rs_staged"] if staged else []),
               inputs="gpu_state_each_stage",
               adam_max_ratio=report["adam_max_ratio"])
    g.destroy()
    return report


def run_group_fused(wl: W.Workload, group: W.Group, *, steps: int = 1, op=None,
                    direct_oracle: bool = False, tag=(), full_init=None,
                    grads_init=None) -> dict:
    """The fused reduce-scatter + AdamW + next copy-in against (a) the three
    separate GPU stages on a copy of the same state (bit for bit) and (b) the
    oracle's composition reduce_scatter -> adamw -> copy_in applied to the
    GPU's own pre-step state: reduced gradient bit for bit, AdamW within the
    tolerance, and the bf16 next all-gather input bit for bit against the
    oracle's copy-in of the GPU's updated master.  Over several steps the
    AdamW state is also held to the oracle's own trajectory."""
    N = wl.N
    op = wl.op if op is None else op
    g = abi.fsdp_plan_group(group.shapes, N)
    p = oracle.plan(group.shapes, N)
    check_plan(g, p)
    NS = N * g.S
    master, master_o = _initial_master(g, p, wl, group, tag, full_init)
    m = Guarded(NS, torch.float32, fill=torch.zeros(NS))
    v = Guarded(NS, torch.float32, fill=torch.zeros(NS))
    # the unfused GPU path on a copy of the same state
    mu, vu = torch.zeros(NS, device="cuda"), torch.zeros(NS, device="cuda")
    masteru = master.t.clone()
    m_o = np.zeros(NS, np.float32)
    v_o = np.zeros(NS, np.float32)
    hp = dict(W.ADAMW_DEFAULTS)
    report = {"adam_max_ratio": 0.0}
    for step in range(1, steps + 1):
        pre = (f32(master.t), f32(m.t), f32(v.t))
        grads = _grads_for(g, wl, group, step, tag, grads_init)
        grads_h = u16(grads)
        ag = Guarded(NS, torch.bfloat16)
        red = Guarded(NS, torch.float32)
        abi.fsdp_rs_adamw_step(g, grads, op, master.t, m.t, v.t, step=step, ag_next=ag.t,
                               reduced=red.t, **hp)
        # unfused GPU stages
        redu = torch.empty(NS, device="cuda")
        agu = torch.empty(NS, dtype=torch.bfloat16, device="cuda")
        abi.fsdp_rs_reduce(g, grads, op, redu)
        abi.fsdp_adamw_step(g, masteru, mu, vu, redu, step=step, **hp)
        abi.fsdp_copy_in(g, masteru, agu)
        torch.cuda.synchronize()
        for buf in (master, m, v, ag, red):
            assert buf.guards_intact(), "fused kernel wrote outside a buffer"
        for name, a, b in (("master", master.t, masteru), ("m", m.t, mu), ("v", v.t, vu),
                           ("reduced", red.t, redu)):
            assert torch.equal(a.view(torch.int32), b.view(torch.int32)), f"fused != unfused {name}"
        assert torch.equal(ag.t.view(torch.int16), agu.view(torch.int16)), "fused != unfused ag"
        # the oracle on the GPU's own inputs
        red_o = (oracle.reduce_scatter_direct if direct_oracle else oracle.reduce_scatter)(p, grads_h, op)
        red_h = f32(red.t)
        assert equal_nan_class(red_h, red_o, "f32"), "fused reduced: " + first_mismatch(red_h, red_o)
        post = (f32(master.t), f32(m.t), f32(v.t))
        _adam_check(report, "fused adamw", step, post, adamw_from_state(*pre, red_h, step, hp))
        ag_h = u16(ag.t)
        ag_o = oracle.copy_in(p, post[0])
        assert equal_nan_class(ag_h, ag_o, "bf16"), "fused next copy-in: " + first_mismatch(ag_h, ag_o)
        # the oracle's own trajectory
        oracle.adamw(master_o, m_o, v_o, red_o, step=step, **hp)
        _adam_check(report, "fused adamw trajectory", step, post, (master_o, m_o, v_o))
        del grads, ag, red, redu, agu
    log_parity("fused", wl, group, g, steps=steps, ops=[W.OP_NAMES[op]],
               bit_exact=["fused_vs_stages", "rs_vs_oracle", "next_copy_in_vs_oracle"],
               inputs="gpu_state_each_step",
               adam_max_ratio=report["adam_max_ratio"])
    g.destroy()
    return report


def run_group_fused_fp8(wl: W.Workload, group: W.Group, *, steps: int = 2, op=None,
                        tag=(), full_init=None, grads_init=None) -> dict:
    """The fused reduce-scatter + AdamW + FP8 next copy-in (delayed scaling)
    against (a) the separate GPU stages rs_reduce -> adamw -> copy_in_fp8_scaled
    with the previous scales, plus copy_in_fp8 for the next scales, on a copy of
    the same state (bit for bit) and (b) the oracle applied to the GPU's own
    inputs: reduced gradient bit for bit; AdamW from the GPU's pre-step state
    within the tolerance; the E4M3 codes bit for bit against the oracle's FP8
    copy-in of the GPU's updated master with the GPU's previous scales; the
    next scales bit for bit against the oracle's scales of that master.  Over
    several steps the AdamW state is also held to the oracle's own
    trajectory within the tolerance."""
    N = wl.N
    op = wl.op if op is None else op
    g = abi.fsdp_plan_group(group.shapes, N)
    p = oracle.plan(group.shapes, N)
    check_plan(g, p)
    NS = N * g.S
    n = max(g.n, 1)
    master, master_o = _initial_master(g, p, wl, group, tag, full_init)
    m = Guarded(NS, torch.float32, fill=torch.zeros(NS))
    v = Guarded(NS, torch.float32, fill=torch.zeros(NS))
    mu, vu = torch.zeros(NS, device="cuda"), torch.zeros(NS, device="cuda")
    masteru = master.t.clone()
    m_o = np.zeros(NS, np.float32)
    v_o = np.zeros(NS, np.float32)
    hp = dict(W.ADAMW_DEFAULTS)
    # step 0: dynamic scales of the initial master start the delayed chain
    scales_prev = torch.empty(n, device="cuda")
    abi.fsdp_copy_in_fp8(g, master.t, torch.empty(max(NS, 1), dtype=torch.uint8, device="cuda"),
                         scales_prev)
    torch.cuda.synchronize()
    assert bits_equal(f32(scales_prev)[:g.n], oracle.fp8_scales(p, f32(master.t)))
    report = {"adam_max_ratio": 0.0, "saturated": 0}
    for step in range(1, steps + 1):
        pre = (f32(master.t), f32(m.t), f32(v.t))
        sp = f32(scales_prev)[:g.n]
        grads = _grads_for(g, wl, group, step, tag, grads_init)
        grads_h = u16(grads)
        ag8 = Guarded(NS, torch.uint8)
        red = Guarded(NS, torch.float32)
        scales_next = Guarded(g.n, torch.float32)
        abi.fsdp_rs_adamw_step_fp8(g, grads, op, master.t, m.t, v.t, step=step,
                                   scales_prev=scales_prev, ag8_next=ag8.t,
                                   scales_next=scales_next.t, reduced=red.t, **hp)
        # the separate GPU stages
        redu = torch.empty(NS, device="cuda")
        ag8u = torch.empty(NS, dtype=torch.uint8, device="cuda")
        dyn = torch.empty(n, device="cuda")
        abi.fsdp_rs_reduce(g, grads, op, redu)
        abi.fsdp_adamw_step(g, masteru, mu, vu, redu, step=step, **hp)
        abi.fsdp_copy_in_fp8_scaled(g, masteru, scales_prev, ag8u)
        abi.fsdp_copy_in_fp8(g, masteru, torch.empty(max(NS, 1), dtype=torch.uint8,
                                                      device="cuda"), dyn)
        torch.cuda.synchronize()
        for buf in (master, m, v, ag8, red, scales_next):
            assert buf.guards_intact(), "fused FP8 kernel wrote outside a buffer"
        for name, a, b in (("master", master.t, masteru), ("m", m.t, mu), ("v", v.t, vu),
                           ("reduced", red.t, redu), ("scales", scales_next.t, dyn[:g.n])):
            assert torch.equal(a.view(torch.int32), b.view(torch.int32)), f"fused != unfused {name}"
        assert torch.equal(ag8.t, ag8u), "fused != unfused ag8"
        # the oracle on the GPU's own inputs
        red_o = oracle.reduce_scatter(p, grads_h, op)
        red_h = f32(red.t)
        assert equal_nan_class(red_h, red_o, "f32"), "fused reduced: " + first_mismatch(red_h, red_o)
        post = (f32(master.t), f32(m.t), f32(v.t))
        _adam_check(report, "fused fp8 adamw", step, post, adamw_from_state(*pre, red_h, step, hp))
        got = ag8.t.cpu().numpy()
        ag8_o = oracle.copy_in_fp8(p, post[0], sp)
        assert equal_nan_class(got, ag8_o, "e4m3"), \
            f"fused fp8 codes: {int(np.sum(got != ag8_o))} differ from the oracle's"
        for i in range(g.n):                     # quantiser inputs the clamp saturated
            for r in range(N):
                o0 = r * g.S + int(p.shard_off[i])
                x = post[0][o0:o0 + int(p.valid_rows(i, r)) * int(p.cols[i])].astype(np.float64)
                with np.errstate(invalid="ignore"):    # Inf * 0 where the scale is 0
                    report["saturated"] += int(np.sum(np.abs(x * float(sp[i])) > 448.0))
        sn = f32(scales_next.t)
        sn_o = oracle.fp8_scales(p, post[0])
        assert bits_equal(sn, sn_o), "fused fp8 next scales: " + first_mismatch(sn, sn_o)
        # the oracle's own trajectory
        oracle.adamw(master_o, m_o, v_o, red_o, step=step, **hp)
        _adam_check(report, "fused fp8 adamw trajectory", step, post, (master_o, m_o, v_o))
        scales_prev = scales_next.t.clone() if g.n else scales_prev
        del grads, ag8, red, redu, ag8u
    log_parity("fused_fp8", wl, group, g, steps=steps, ops=[W.OP_NAMES[op]],
               bit_exact=["fused_vs_stages", "rs_vs_oracle", "fp8_codes_vs_oracle",
                          "next_scales_vs_oracle"],
               inputs="gpu_state_each_step",
               adam_max_ratio=report["adam_max_ratio"])
    g.destroy()
    return report


def run_group_accumulate(wl: W.Workload, group: W.Group, *, micro: int = 3, op=None,
                         tag=(), grads_init=None) -> None:
    """Gradient accumulation without sync over `micro` microbatches: the
    accumulated fp32 arenas after every microbatch and the final reduce-scatter
    (fused with the last microbatch, and from the accumulated arenas alone)
    against the oracle, bit for bit."""
    assert micro >= 2, "one microbatch needs no accumulation: use fsdp_rs_reduce"
    N = wl.N
    op = wl.op if op is None else op
    g = abi.fsdp_plan_group(group.shapes, N)
    p = oracle.plan(group.shapes, N)
    check_plan(g, p)
    n = N * g.P_arena
    acc = Guarded(n, torch.float32)
    acc_o = np.zeros(n, np.float32)
    for t in range(1, micro):
        grads = _grads_for(g, wl, group, t, ("micro",) + tuple(tag), grads_init)
        abi.fsdp_grad_accumulate(g, grads, acc.t, first=(t == 1))
        torch.cuda.synchronize()
        assert acc.guards_intact()
        oracle.accumulate(acc_o, u16(grads), first=(t == 1))
        assert equal_nan_class(f32(acc.t), acc_o, "f32"), f"accumulate {t}: " + first_mismatch(f32(acc.t), acc_o)
    last = _grads_for(g, wl, group, micro, ("micro",) + tuple(tag), grads_init)
    red = Guarded(N * g.S, torch.float32)
    abi.fsdp_rs_reduce_accumulated(g, last, acc.t, op, red.t)
    torch.cuda.synchronize()
    assert red.guards_intact() and acc.guards_intact()
    oracle.accumulate(acc_o, u16(last), first=False)
    red_o = oracle.reduce_scatter_f32(p, acc_o, op)
    assert equal_nan_class(f32(red.t), red_o, "f32"), "rs accumulated: " + first_mismatch(f32(red.t), red_o)
    # the same through an explicit last accumulation and a reduce of acc alone
    abi.fsdp_grad_accumulate(g, last, acc.t, first=False)
    red2 = torch.empty(N * g.S, device="cuda")
    abi.fsdp_rs_reduce_accumulated(g, None, acc.t, op, red2)
    torch.cuda.synchronize()
    assert equal_nan_class(f32(red2), red_o, "f32")
    log_parity("accumulate", wl, group, g, microbatches=micro, ops=[W.OP_NAMES[op]],
               bit_exact=["accumulate", "rs_accumulated", "rs_accumulated_no_last"])
    g.destroy()


def run_group_fp8(wl: W.Workload, group: W.Group, tag=(), full_init=None) -> None:
    """FP8 all-gather: scales, the E4M3 copy-in and the byte copy-out against
    the oracle, bit for bit, with guard bands."""
    N = wl.N
    g = abi.fsdp_plan_group(group.shapes, N)
    p = oracle.plan(group.shapes, N)
    check_plan(g, p)
    NS = N * g.S
    full = torch.empty(max(g.P_arena, 1), dtype=torch.float32, device="cuda")
    if full_init is None:
        W.fill_master(full, wl, group.name, *tag)
    else:
        full.zero_()
        full[:g.P_arena].copy_(torch.from_numpy(np.ascontiguousarray(full_init, np.float32)))
    master = torch.empty(max(NS, 1), dtype=torch.float32, device="cuda")
    abi.fsdp_shard_params(g, full, master)
    G8 = 4 * GUARD  # guard bytes on each side (a multiple of 16)
    ag8 = torch.full((NS + 2 * G8,), 0x5A, dtype=torch.uint8, device="cuda")
    ag8_t = ag8[G8:G8 + NS]
    scales = torch.full((max(g.n, 1) + 2,), -3.0, dtype=torch.float32, device="cuda")
    abi.fsdp_copy_in_fp8(g, master[:NS], ag8_t, scales[1:1 + g.n] if g.n else scales[1:1])
    arena8 = torch.full((g.P_arena + 2 * G8,), 0xA5, dtype=torch.uint8, device="cuda")
    arena8_t = arena8[G8:G8 + g.P_arena]
    abi.fsdp_copy_out_fp8(g, ag8_t, arena8_t)
    torch.cuda.synchronize()
    host_ag8 = ag8.cpu().numpy()
    assert np.all(host_ag8[:G8] == 0x5A) and np.all(host_ag8[G8 + NS:] == 0x5A)
    host_ar = arena8.cpu().numpy()
    assert np.all(host_ar[:G8] == 0xA5) and np.all(host_ar[G8 + g.P_arena:] == 0xA5)
    sc = scales.cpu().numpy()
    assert sc[0] == -3.0 and sc[1 + g.n] == -3.0
    master_o = oracle.shard(p, f32(full)[:p.P_arena] if p.P_arena else np.zeros(0, np.float32))
    assert bits_equal(f32(master[:NS]), master_o)
    scales_o = oracle.fp8_scales(p, master_o)
    assert bits_equal(sc[1:1 + g.n], scales_o), "fp8 scales: " + first_mismatch(sc[1:1 + g.n], scales_o)
    ag8_o = oracle.copy_in_fp8(p, master_o, scales_o)
    got = host_ag8[G8:G8 + NS]
    assert equal_nan_class(got, ag8_o, "e4m3"), f"fp8 copy-in: {int(np.sum(got != ag8_o))} mismatches"
    # the byte copy-out of the GPU's own codes (a bit move)
    arena_o = oracle.copy_out_fp8(p, got, np.full(p.P_arena, 0xA5, np.uint8))
    got = host_ar[G8:G8 + g.P_arena]
    assert np.array_equal(got, arena_o), f"fp8 copy-out: {int(np.sum(got != arena_o))} mismatches"
    log_parity("fp8", wl, group, g, bit_exact=["scales", "fp8_copy_in", "fp8_copy_out"])
    g.destroy()
