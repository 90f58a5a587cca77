"""The several-device exchange on one GPU: per-rank pointer tables and CUDA
IPC, against the single-device path bit for bit.

* In one process, D "devices" are D disjoint sets of buffers (each with its
  own slot and gradient arenas) and D peer plans; the pulls of the copy-out
  and of the reductions read across those allocations exactly as they read
  peers' memory, and every result equals the single-device group's rows.
* Across processes, D processes on the one GPU map each other's buffers with
  CUDA IPC (fully_sharded_shard_b200.peer.PeerGroup) and run two fused steps;
  gloo barriers order the phases on the host (no kernel waits on another).

Every result of every device is also checked against the CPU oracle applied
to the GPU's own inputs: each device's copy-out against the oracle's
copy-out of the slots, each device's reduced rows against the oracle's
reduce-scatter, its AdamW state against the oracle's AdamW from its pre-step
state (within 1e-6 * (1 + |x|)), and the slots its fused update wrote against
the oracle's copy-in (bf16 or E4M3 with the previous scales) of the updated
master, with the next FP8 scales against the oracle's scales of that master.
"""
import os
import socket

import numpy as np
import pytest
import torch

import fully_sharded_shard_b200.workloads as W

pytestmark = pytest.mark.gpu


def _wl(name, shapes, N, op=W.AVG, zero=()):
    g = W.Group(name, [tuple(s) for s in shapes], [f"p{i}" for i in range(len(shapes))],
                zero_grad=list(zero))
    return W.Workload(name, N, [g], op, 0, "normal", 0.02, 1e-3, steps=2)


@pytest.fixture(scope="module")
def H():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    from tests import _harness
    return _harness


def run_group_peer(H, wl, grp, D, *, steps=2, direct_oracle=False, tag=(), full_init=None,
                   grads_init=None):
    """Every stage of D emulated devices against the single-device group and
    against the oracle on the GPU's own inputs.  full_init / grads_init
    replace the seeded inputs as in the harness."""
    from fully_sharded_shard_b200 import abi
    from fully_sharded_shard_b200.peer import rank_pointer_tables
    import oracle
    N, op = wl.N, wl.op
    L = N // D
    g = abi.fsdp_plan_group(grp.shapes, N)
    S, A = g.S, g.P_arena
    full = torch.empty(max(A, 1), device="cuda")
    if full_init is None:
        W.fill_master(full, wl, grp.name, *tag)
    else:
        full.zero_()
        full[:A].copy_(torch.from_numpy(np.ascontiguousarray(full_init, np.float32)))
    master = torch.empty(max(N * S, 1), device="cuda")
    abi.fsdp_shard_params(g, full, master)
    ref = {"p": master[:N * S].clone(), "m": torch.zeros(N * S, device="cuda"),
           "v": torch.zeros(N * S, device="cuda")}
    pps = [abi.fsdp_peer_plan(g, D, d) for d in range(D)]
    assert [(pp.L, pp.r0) for pp in pps] == [(L, d * L) for d in range(D)]
    slots = [H.Guarded(L * S, torch.bfloat16) for _ in range(D)]
    gbufs = [H.Guarded(L * A, torch.bfloat16) for _ in range(D)]
    ag_ptrs, gr_ptrs = rank_pointer_tables([s.t.data_ptr() for s in slots],
                                           [b.t.data_ptr() for b in gbufs], L, S, A)
    for pp in pps:
        abi.fsdp_peer_set_sources(pp, ag_ptrs, gr_ptrs)
    dev = [{"p": ref["p"][d * L * S:(d + 1) * L * S].clone(),
            "m": torch.zeros(L * S, device="cuda"), "v": torch.zeros(L * S, device="cuda")}
           for d in range(D)]
    hp = dict(W.ADAMW_DEFAULTS)
    sentinel = 0x3BEF
    p = oracle.plan(grp.shapes, N)
    rs_oracle = oracle.reduce_scatter_direct if direct_oracle else oracle.reduce_scatter

    def slot_rows(d):
        return slice(d * L * S, (d + 1) * L * S)

    def gathered_and_copied_out(ag_ref):
        """Copy-out on every device from the slots; the reference copy-out of
        the single-device all-gather buffer; compare."""
        arena_ref = torch.full((max(A, 1),), sentinel, dtype=torch.int16, device="cuda")
        abi.fsdp_copy_out(g, ag_ref, arena_ref.view(torch.bfloat16)[:A] if A else arena_ref.view(torch.bfloat16))
        got = torch.cat([s.t.view(torch.int16) for s in slots]) if S else None
        if S:
            assert torch.equal(got, ag_ref.view(torch.int16)[:N * S]), "slots != all-gather buffer"
        slots_h = H.u16(got) if S else np.zeros(0, np.uint16)
        arena_o = oracle.copy_out(p, slots_h, np.full(A, sentinel, np.uint16))
        assert H.bits_equal(H.u16(arena_ref[:A]), arena_o), "copy-out vs oracle"
        for d in range(D):
            arena = H.Guarded(A, torch.bfloat16)
            arena.t.view(torch.int16).fill_(sentinel)
            abi.fsdp_peer_copy_out(pps[d], arena.t)
            torch.cuda.synchronize()
            assert arena.guards_intact()
            assert torch.equal(arena.t.view(torch.int16), arena_ref[:A]), f"device {d} copy-out"

    # step 0: copy-in on every device, then the pulls of the copy-out
    for d in range(D):
        abi.fsdp_peer_copy_in(pps[d], dev[d]["p"], slots[d].t)
    ag_ref = torch.empty(max(N * S, 1), dtype=torch.bfloat16, device="cuda")
    abi.fsdp_copy_in(g, ref["p"], ag_ref)
    torch.cuda.synchronize()
    gathered_and_copied_out(ag_ref)
    for step in range(1, steps + 1):
        grads = H._grads_for(g, wl, grp, step, tag, grads_init)
        for d in range(D):
            gbufs[d].t.copy_(grads[d * L:(d + 1) * L].reshape(-1))
        # the reduce-scatter pulls
        red_ref = torch.empty(max(N * S, 1), device="cuda")
        abi.fsdp_rs_reduce(g, grads, op, red_ref)
        reds = [H.Guarded(L * S, torch.float32) for _ in range(D)]
        for d in range(D):
            abi.fsdp_peer_rs_reduce(pps[d], op, reds[d].t)
        torch.cuda.synchronize()
        for d in range(D):
            assert reds[d].guards_intact()
            assert torch.equal(reds[d].t.view(torch.int32),
                               red_ref[d * L * S:(d + 1) * L * S].view(torch.int32)), \
                f"device {d} reduce-scatter, step {step}"
        red_o = rs_oracle(p, H.u16(grads), op)
        for d in range(D):
            assert H.equal_nan_class(H.f32(reds[d].t), red_o[slot_rows(d)], "f32"), \
                f"device {d} reduce-scatter vs oracle, step {step}"
        # the unfused AdamW of the local shards, on copies of the state
        full_cp = {k: t.clone() for k, t in ref.items()}
        abi.fsdp_adamw_step(g, full_cp["p"], full_cp["m"], full_cp["v"], red_ref[:N * S],
                            step=step, **hp)
        pre = [tuple(H.f32(dev[d][k]) for k in ("p", "m", "v")) for d in range(D)]
        for d in range(D):
            cp = {k: t.clone() for k, t in dev[d].items()}
            abi.fsdp_peer_adamw_step(pps[d], cp["p"], cp["m"], cp["v"], reds[d].t, step=step, **hp)
            torch.cuda.synchronize()
            for k in ("p", "m", "v"):
                assert torch.equal(cp[k].view(torch.int32),
                                   full_cp[k][d * L * S:(d + 1) * L * S].view(torch.int32)), \
                    f"device {d} adamw {k}"
            want = H.adamw_from_state(*pre[d], H.f32(reds[d].t), step, hp)
            for k, w in zip(("p", "m", "v"), want):
                ok, ratio = H.adam_close_special(H.f32(cp[k]), w)
                assert ok, f"device {d} adamw {k} vs oracle: {ratio}"
        del full_cp
        # the fused update with the next copy-in into each device's own slot
        red2 = [H.Guarded(L * S, torch.float32) for _ in range(D)]
        for d in range(D):
            abi.fsdp_peer_rs_adamw_step(pps[d], op, dev[d]["p"], dev[d]["m"], dev[d]["v"],
                                        step=step, ag_next=slots[d].t, reduced=red2[d].t, **hp)
        red2_ref = torch.empty(max(N * S, 1), device="cuda")
        abi.fsdp_rs_adamw_step(g, grads, op, ref["p"], ref["m"], ref["v"], step=step,
                               ag_next=ag_ref, reduced=red2_ref, **hp)
        torch.cuda.synchronize()
        for d in range(D):
            assert slots[d].guards_intact() and red2[d].guards_intact()
            rows = slice(d * L * S, (d + 1) * L * S)
            for k in ("p", "m", "v"):
                assert torch.equal(dev[d][k].view(torch.int32), ref[k][rows].view(torch.int32)), \
                    f"device {d} fused {k}, step {step}"
            assert torch.equal(red2[d].t.view(torch.int32), red2_ref[rows].view(torch.int32))
            assert H.equal_nan_class(H.f32(red2[d].t), red_o[rows], "f32")
            want = H.adamw_from_state(*pre[d], H.f32(red2[d].t), step, hp)
            for k, w in zip(("p", "m", "v"), want):
                ok, ratio = H.adam_close_special(H.f32(dev[d][k]), w)
                assert ok, f"device {d} fused {k} vs oracle: {ratio}"
        if S:
            post = np.concatenate([H.f32(dev[d]["p"]) for d in range(D)])
            ag_o = oracle.copy_in(p, post)
            for d in range(D):
                assert H.equal_nan_class(H.u16(slots[d].t), ag_o[slot_rows(d)], "bf16"), \
                    f"device {d} next copy-in vs oracle, step {step}"
        # the next step's all-gather: pulls of the slots the fused update wrote
        gathered_and_copied_out(ag_ref)
        del grads
    for pp in pps:
        pp.destroy()
    g.destroy()


def run_group_peer_fp8(H, wl, grp, D, *, steps=2, tag=()):
    """The FP8 all-gather over D emulated devices (delayed scaling): slots,
    partial amax arrays, next scales, the byte copy-out pulls and the state
    against fsdp_rs_adamw_step_fp8 / fsdp_copy_out_fp8 of the single-device
    group, bit for bit, and against the oracle on the GPU's own inputs."""
    from fully_sharded_shard_b200 import abi
    from fully_sharded_shard_b200.peer import rank_pointer_tables
    import oracle
    N, op = wl.N, wl.op
    L = N // D
    g = abi.fsdp_plan_group(grp.shapes, N)
    S, A, n = g.S, g.P_arena, g.n
    full = torch.empty(max(A, 1), device="cuda")
    W.fill_master(full, wl, grp.name, *tag)
    master = torch.empty(max(N * S, 1), device="cuda")
    abi.fsdp_shard_params(g, full, master)
    ref = {"p": master[:N * S].clone(), "m": torch.zeros(N * S, device="cuda"),
           "v": torch.zeros(N * S, device="cuda")}
    pps = [abi.fsdp_peer_plan(g, D, d) for d in range(D)]
    slots = [H.Guarded(L * S, torch.bfloat16) for _ in range(D)]
    slots8 = [H.Guarded(L * S, torch.uint8) for _ in range(D)]
    gbufs = [H.Guarded(L * A, torch.bfloat16) for _ in range(D)]
    amax = [torch.empty(max(n, 1), dtype=torch.int32, device="cuda") for _ in range(D)]
    ag_ptrs, gr_ptrs = rank_pointer_tables([s.t.data_ptr() for s in slots],
                                           [b.t.data_ptr() for b in gbufs], L, S, A)
    ag8_ptrs = [slots8[r // L].t.data_ptr() + S * (r % L) for r in range(N)]
    for pp in pps:
        abi.fsdp_peer_set_sources(pp, ag_ptrs, gr_ptrs)
        abi.fsdp_peer_set_fp8_sources(pp, ag8_ptrs, [a.data_ptr() for a in amax])
    dev = [{k: t[d * L * S:(d + 1) * L * S].clone() for k, t in ref.items()} for d in range(D)]
    hp = dict(W.ADAMW_DEFAULTS)
    p = oracle.plan(grp.shapes, N)
    # step 0: dynamic scales of the initial master, the scaled copy-in on every device
    scales = torch.empty(max(n, 1), device="cuda")
    ag8_ref = torch.empty(max(N * S, 1), dtype=torch.uint8, device="cuda")
    abi.fsdp_copy_in_fp8(g, ref["p"], ag8_ref, scales)
    for d in range(D):
        abi.fsdp_peer_copy_in_fp8_scaled(pps[d], dev[d]["p"], scales, slots8[d].t)

    def pulls_equal_reference():
        torch.cuda.synchronize()
        if S:
            got = torch.cat([s.t for s in slots8])
            assert torch.equal(got, ag8_ref[:N * S]), "E4M3 slots != single-device buffer"
        ar_ref = torch.full((max(A, 1),), 0xA5, dtype=torch.uint8, device="cuda")
        abi.fsdp_copy_out_fp8(g, ag8_ref, ar_ref)
        slots_h = torch.cat([s.t for s in slots8]).cpu().numpy() if S else np.zeros(0, np.uint8)
        ar_o = oracle.copy_out_fp8(p, slots_h, np.full(A, 0xA5, np.uint8))
        for d in range(D):
            ar = H.Guarded(A, torch.uint8)
            ar.t.fill_(0xA5)
            abi.fsdp_peer_copy_out_fp8(pps[d], ar.t)
            torch.cuda.synchronize()
            assert ar.guards_intact()
            assert torch.equal(ar.t, ar_ref[:A]), f"device {d} FP8 copy-out"
            assert np.array_equal(ar.t.cpu().numpy(), ar_o), f"device {d} FP8 copy-out vs oracle"

    pulls_equal_reference()
    for step in range(1, steps + 1):
        grads = H.make_grads(g, wl, grp, step, tag)
        for d in range(D):
            gbufs[d].t.copy_(grads[d * L:(d + 1) * L].reshape(-1))
        pre = [tuple(H.f32(dev[d][k]) for k in ("p", "m", "v")) for d in range(D)]
        red_o = oracle.reduce_scatter(p, H.u16(grads), op)
        nxt_ref = torch.empty(max(n, 1), device="cuda")
        abi.fsdp_rs_adamw_step_fp8(g, grads, op, ref["p"], ref["m"], ref["v"], step=step,
                                   scales_prev=scales, ag8_next=ag8_ref, scales_next=nxt_ref, **hp)
        for d in range(D):
            abi.fsdp_peer_rs_adamw_step_fp8(pps[d], op, dev[d]["p"], dev[d]["m"], dev[d]["v"],
                                            step=step, scales_prev=scales, ag8_next=slots8[d].t,
                                            amax_local=amax[d], **hp)
        torch.cuda.synchronize()  # every device's partial amax is complete
        nxt = [torch.empty(max(n, 1), device="cuda") for _ in range(D)]
        for d in range(D):
            abi.fsdp_peer_fp8_scales(pps[d], nxt[d])
        torch.cuda.synchronize()
        for d in range(D):
            assert slots8[d].guards_intact()
            assert torch.equal(nxt[d][:n].view(torch.int32), nxt_ref[:n].view(torch.int32)), \
                f"device {d} next scales, step {step}"
            rows = slice(d * L * S, (d + 1) * L * S)
            for k in ("p", "m", "v"):
                assert torch.equal(dev[d][k].view(torch.int32), ref[k][rows].view(torch.int32))
            want = H.adamw_from_state(*pre[d], red_o[rows], step, hp)
            for k, w in zip(("p", "m", "v"), want):
                ok, ratio = H.adam_close_special(H.f32(dev[d][k]), w)
                assert ok, f"device {d} fused FP8 {k} vs oracle: {ratio}"
        if S:
            post = np.concatenate([H.f32(dev[d]["p"]) for d in range(D)])
            sp = H.f32(scales)[:n]
            ag8_o = oracle.copy_in_fp8(p, post, sp)
            for d in range(D):
                rows = slice(d * L * S, (d + 1) * L * S)
                assert H.equal_nan_class(slots8[d].t.cpu().numpy(), ag8_o[rows], "e4m3"), \
                    f"device {d} E4M3 slot vs oracle, step {step}"
            assert H.bits_equal(H.f32(nxt[0])[:n], oracle.fp8_scales(p, post)), \
                f"next scales vs oracle, step {step}"
        pulls_equal_reference()
        scales = nxt_ref
        del grads
    for pp in pps:
        pp.destroy()
    g.destroy()


PEER = [
    (_wl("peer_ragged_n4", [(7, 3), (5,), (1, 32), (1,), (0, 4), (13, 9), (2, 2)], 4, op=W.SUM), (1, 2, 4)),
    (_wl("peer_n6_odd", [(1001, 3), (17,), (3, 4099), (8191, 1)], 6, op=W.SUM_THEN_DIV), (2, 3, 6)),
    (_wl("peer_n12", [(37, 100), (6,), (1999, 31)], 12), (3, 4, 12)),
    (_wl("peer_n2_shift", [(3,), (9001, 5), (7, 1), (16385,)], 2, zero=[1]), (1, 2)),
    (_wl("peer_n64", [(129, 7), (64,), (1, 5), (300,)], 64), (8, 64)),
    (W.tiny_mlp(), (2,)),
    (W.uneven(8), (2, 3, 6)),
    (W.moe(8), (2, 8)),
]


@pytest.mark.parametrize("case", PEER, ids=[c[0].name for c in PEER])
def test_peer_pulls_equal_single_device(H, case):
    wl, Ds = case
    for grp in wl.groups:
        for D in Ds:
            run_group_peer(H, wl, grp, D, steps=2)


@pytest.mark.parametrize("case", PEER, ids=[c[0].name for c in PEER])
def test_peer_fp8_all_gather_equals_single_device(H, case):
    wl, Ds = case
    for grp in wl.groups:
        for D in Ds:
            run_group_peer_fp8(H, wl, grp, D, steps=2)


def test_peer_full_size_llama7b_block_eight_devices(H):
    wl = W.llama7b()
    run_group_peer(H, wl, wl.groups[0], 8, steps=1, direct_oracle=True)


def test_peer_plan_rejects_bad_splits(H):
    from fully_sharded_shard_b200 import abi
    g = abi.fsdp_plan_group([(10, 3)], 6)
    for D, d in ((4, 0), (0, 0), (3, 3), (3, -1)):
        with pytest.raises(abi.FsdpError) as e:
            abi.fsdp_peer_plan(g, D, d)
        assert e.value.status == abi.FSDP_EINVAL
    big = abi.fsdp_plan_group([(10, 3)], 128)
    with pytest.raises(abi.FsdpError):
        abi.fsdp_peer_plan(big, 2, 0)  # more ranks than a table holds
    pp = abi.fsdp_peer_plan(g, 3, 1)
    arena = torch.empty(g.P_arena, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(abi.FsdpError) as e:
        abi.fsdp_peer_copy_out(pp, arena)  # no tables yet
    assert e.value.status == abi.FSDP_ESTATE
    buf = torch.empty(64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(abi.FsdpError) as e:  # a gradient arena must be 16-byte aligned
        abi.fsdp_peer_set_sources(pp, None, [buf.data_ptr() + 2] * 6)
    assert e.value.status == abi.FSDP_EALIGN
    pp.destroy()
    g.destroy()
    big.destroy()


# ---------------------------------------------------------------------------
# several processes on the one GPU, CUDA IPC between them
# ---------------------------------------------------------------------------
def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _ipc_worker(rank, port, D, case_name, result_dir):
    import datetime
    import torch.distributed as dist
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=D, timeout=datetime.timedelta(seconds=120))
    msg = "ok"
    try:
        torch.cuda.set_device(0)
        from fully_sharded_shard_b200 import abi
        from fully_sharded_shard_b200.peer import PeerGroup
        from tests import _harness as H
        import oracle
        wl = {"uneven": W.uneven(16), "tiny": W.tiny_mlp(), "moe": W.moe(16)}[case_name]
        grp = wl.groups[0]
        N, op = wl.N, wl.op
        p = oracle.plan(grp.shapes, N)
        pgrp = PeerGroup(grp.shapes, N, device="cuda:0")
        g, S, A, L, r0 = pgrp.g, pgrp.S, pgrp.P_arena, pgrp.L, pgrp.r0
        rows = slice(r0 * S, (r0 + L) * S)
        full = torch.empty(max(A, 1), device="cuda")
        W.fill_master(full, wl, grp.name)
        master = torch.empty(max(N * S, 1), device="cuda")
        abi.fsdp_shard_params(g, full, master)
        ref = {"p": master[:N * S].clone(), "m": torch.zeros(N * S, device="cuda"),
               "v": torch.zeros(N * S, device="cuda")}
        mine = {k: t[rows].clone() for k, t in ref.items()}
        hp = dict(W.ADAMW_DEFAULTS)
        ag_ref = torch.empty(max(N * S, 1), dtype=torch.bfloat16, device="cuda")
        abi.fsdp_copy_in(g, ref["p"], ag_ref)
        pgrp.copy_in(mine["p"])
        for step in range(1, 3):
            pgrp.barrier()                       # every slot written
            arena = torch.full((max(A, 1),), 0x3BEF, dtype=torch.int16, device="cuda")
            pgrp.copy_out(arena.view(torch.bfloat16)[:A])
            arena_ref = torch.full((max(A, 1),), 0x3BEF, dtype=torch.int16, device="cuda")
            abi.fsdp_copy_out(g, ag_ref, arena_ref.view(torch.bfloat16)[:A])
            torch.cuda.synchronize()
            arena_o = oracle.copy_out(p, H.u16(ag_ref)[:N * S], np.full(A, 0x3BEF, np.uint16))
            grads = H.make_grads(g, wl, grp, step)
            pgrp.grads.copy_(grads[r0:r0 + L])
            pgrp.barrier()                       # every copy-out done, every gradient written
            pre = tuple(H.f32(mine[k]) for k in ("p", "m", "v"))
            red = torch.empty(max(L * S, 1), device="cuda")
            pgrp.rs_adamw_step(op, mine["p"], mine["m"], mine["v"], reduced=red, step=step, **hp)
            red_ref = torch.empty(max(N * S, 1), device="cuda")
            abi.fsdp_rs_adamw_step(g, grads, op, ref["p"], ref["m"], ref["v"], step=step,
                                   ag_next=ag_ref, reduced=red_ref, **hp)
            torch.cuda.synchronize()
            if not torch.equal(arena, arena_ref):
                msg = f"copy-out differs at step {step}"
                break
            bad = [k for k in ("p", "m", "v")
                   if not torch.equal(mine[k].view(torch.int32), ref[k][rows].view(torch.int32))]
            if bad or not torch.equal(red[:L * S].view(torch.int32), red_ref[rows].view(torch.int32)):
                msg = f"fused update differs at step {step}: {bad or 'reduced'}"
                break
            if not torch.equal(pgrp.ag_slot.view(torch.int16), ag_ref[rows].view(torch.int16)):
                msg = f"next copy-in differs at step {step}"
                break
            # the oracle on this process's own inputs
            red_o = oracle.reduce_scatter(p, H.u16(grads), op)[rows]
            want = H.adamw_from_state(*pre, red_o, step, hp)
            if not H.bits_equal(H.u16(arena.view(torch.bfloat16))[:A], arena_o):
                msg = f"copy-out differs from the oracle at step {step}"
                break
            if not H.equal_nan_class(H.f32(red)[:L * S], red_o, "f32"):
                msg = f"reduced rows differ from the oracle at step {step}"
                break
            if not all(H.adam_close_special(H.f32(mine[k]), w)[0]
                       for k, w in zip(("p", "m", "v"), want)):
                msg = f"AdamW differs from the oracle at step {step}"
                break
            if not H.equal_nan_class(H.u16(pgrp.ag_slot), oracle.copy_in(p, H.f32(ref["p"]))[rows],
                                     "bf16"):
                msg = f"next copy-in differs from the oracle at step {step}"
                break
        pgrp.close()
    except Exception as e:  # reported through the result file
        msg = f"error: {type(e).__name__}: {e}"
    finally:
        with open(os.path.join(result_dir, f"r{rank}.txt"), "w") as f:
            f.write(msg + "\n")
        dist.destroy_process_group()


@pytest.mark.parametrize("D,case", [(2, "tiny"), (2, "uneven"), (3, "uneven"), (4, "moe")])
def test_peer_group_over_cuda_ipc_processes(H, tmp_path, D, case):
    import torch.multiprocessing as mp
    mp.spawn(_ipc_worker, args=(_free_port(), D, case, str(tmp_path)), nprocs=D, join=True)
    for r in range(D):
        assert open(tmp_path / f"r{r}.txt").read().strip() == "ok", f"process {r}"


def _ipc_fp8_worker(rank, port, D, case_name, result_dir):
    import datetime
    import torch.distributed as dist
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=D, timeout=datetime.timedelta(seconds=120))
    msg = "ok"
    try:
        torch.cuda.set_device(0)
        from fully_sharded_shard_b200 import abi
        from fully_sharded_shard_b200.peer import PeerGroup
        from tests import _harness as H
        wl = {"uneven": W.uneven(16), "moe": W.moe(16)}[case_name]
        grp = wl.groups[0]
        N, op = wl.N, wl.op
        pgrp = PeerGroup(grp.shapes, N, device="cuda:0", fp8=True)
        g, S, A, L, r0, n = pgrp.g, pgrp.S, pgrp.P_arena, pgrp.L, pgrp.r0, pgrp.g.n
        rows = slice(r0 * S, (r0 + L) * S)
        full = torch.empty(max(A, 1), device="cuda")
        W.fill_master(full, wl, grp.name)
        master = torch.empty(max(N * S, 1), device="cuda")
        abi.fsdp_shard_params(g, full, master)
        ref = {"p": master[:N * S].clone(), "m": torch.zeros(N * S, device="cuda"),
               "v": torch.zeros(N * S, device="cuda")}
        mine = {k: t[rows].clone() for k, t in ref.items()}
        hp = dict(W.ADAMW_DEFAULTS)
        scales = torch.empty(max(n, 1), device="cuda")
        ag8_ref = torch.empty(max(N * S, 1), dtype=torch.uint8, device="cuda")
        abi.fsdp_copy_in_fp8(g, ref["p"], ag8_ref, scales)
        pgrp.copy_in_fp8(mine["p"], scales)
        for step in range(1, 3):
            pgrp.barrier()                       # every E4M3 slot written
            ar = torch.full((max(A, 1),), 0xA5, dtype=torch.uint8, device="cuda")
            pgrp.copy_out_fp8(ar[:A])
            ar_ref = torch.full((max(A, 1),), 0xA5, dtype=torch.uint8, device="cuda")
            abi.fsdp_copy_out_fp8(g, ag8_ref, ar_ref[:A])
            grads = H.make_grads(g, wl, grp, step)
            pgrp.grads.copy_(grads[r0:r0 + L])
            pgrp.barrier()                       # copy-outs done, gradients written
            pgrp.rs_adamw_step_fp8(op, mine["p"], mine["m"], mine["v"], scales_prev=scales,
                                   step=step, **hp)
            nxt_ref = torch.empty(max(n, 1), device="cuda")
            abi.fsdp_rs_adamw_step_fp8(g, grads, op, ref["p"], ref["m"], ref["v"], step=step,
                                       scales_prev=scales, ag8_next=ag8_ref,
                                       scales_next=nxt_ref, **hp)
            pgrp.barrier()                       # every partial amax complete
            nxt = torch.empty(max(n, 1), device="cuda")
            pgrp.fp8_scales(nxt)
            torch.cuda.synchronize()
            if not torch.equal(ar, ar_ref):
                msg = f"FP8 copy-out differs at step {step}"
                break
            if not torch.equal(nxt[:n].view(torch.int32), nxt_ref[:n].view(torch.int32)):
                msg = f"next scales differ at step {step}"
                break
            if not torch.equal(pgrp.ag8_slot, ag8_ref[rows]):
                msg = f"E4M3 slot differs at step {step}"
                break
            bad = [k for k in ("p", "m", "v")
                   if not torch.equal(mine[k].view(torch.int32), ref[k][rows].view(torch.int32))]
            if bad:
                msg = f"fused FP8 update differs at step {step}: {bad}"
                break
            scales = nxt_ref
        pgrp.close()
    except Exception as e:  # reported through the result file
        msg = f"error: {type(e).__name__}: {e}"
    finally:
        with open(os.path.join(result_dir, f"r{rank}.txt"), "w") as f:
            f.write(msg + "\n")
        dist.destroy_process_group()


@pytest.mark.parametrize("D,case", [(2, "uneven"), (4, "moe")])
def test_peer_fp8_group_over_cuda_ipc_processes(H, tmp_path, D, case):
    import torch.multiprocessing as mp
    mp.spawn(_ipc_fp8_worker, args=(_free_port(), D, case, str(tmp_path)), nprocs=D, join=True)
    for r in range(D):
        assert open(tmp_path / f"r{r}.txt").read().strip() == "ok", f"process {r}"


# ---------------------------------------------------------------------------
# several processes on the one GPU, ordered by CUDA IPC events (one host
# barrier per step, no device synchronisation inside the steps)
# ---------------------------------------------------------------------------
def _ipc_pipelined_worker(rank, port, D, case_name, steps, result_dir):
    import datetime
    import torch.distributed as dist
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=D, timeout=datetime.timedelta(seconds=120))
    msg = "ok"
    try:
        torch.cuda.set_device(0)
        from fully_sharded_shard_b200 import abi
        from fully_sharded_shard_b200.peer import PipelinedPeerGroup, host_barrier
        from tests import _harness as H
        import oracle
        wl = {"uneven": W.uneven(16), "tiny": W.tiny_mlp(), "moe": W.moe(16)}[case_name]
        grp = wl.groups[0]
        N, op = wl.N, wl.op
        p = oracle.plan(grp.shapes, N)
        pgrp = PipelinedPeerGroup(grp.shapes, N, device="cuda:0")
        g, S, A, L, r0 = pgrp.g, pgrp.S, pgrp.P_arena, pgrp.L, pgrp.r0
        rows = slice(r0 * S, (r0 + L) * S)
        full = torch.empty(max(A, 1), device="cuda")
        W.fill_master(full, wl, grp.name)
        master = torch.empty(max(N * S, 1), device="cuda")
        abi.fsdp_shard_params(g, full, master)
        hp = dict(W.ADAMW_DEFAULTS)
        grads = [H.make_grads(g, wl, grp, t) for t in range(1, steps + 1)]
        # the single-device references of every step, computed first
        ref = {"p": master[:N * S].clone(), "m": torch.zeros(N * S, device="cuda"),
               "v": torch.zeros(N * S, device="cuda")}
        mine = {k: t[rows].clone() for k, t in ref.items()}
        ag_ref = torch.empty(max(N * S, 1), dtype=torch.bfloat16, device="cuda")
        abi.fsdp_copy_in(g, ref["p"], ag_ref)
        arena_ref, red_ref, pre = [], [], []
        for t in range(1, steps + 1):
            a = torch.full((max(A, 1),), 0x3BEF, dtype=torch.int16, device="cuda")
            abi.fsdp_copy_out(g, ag_ref, a.view(torch.bfloat16)[:A])
            arena_ref.append(a)
            pre.append(tuple(H.f32(ref[k][rows]) for k in ("p", "m", "v")))
            r = torch.empty(max(N * S, 1), device="cuda")
            abi.fsdp_rs_adamw_step(g, grads[t - 1], op, ref["p"], ref["m"], ref["v"], step=t,
                                   ag_next=ag_ref, reduced=r, **hp)
            red_ref.append(r)
        torch.cuda.synchronize()
        # the pipelined run: two streams, events between the processes
        sg, su = torch.cuda.Stream(), torch.cuda.Stream()
        arenas = [torch.full((max(A, 1),), 0x3BEF, dtype=torch.int16, device="cuda")
                  for _ in range(steps)]
        reds = [torch.empty(max(L * S, 1), device="cuda") for _ in range(steps)]
        host_barrier()
        for t in range(1, steps + 1):
            par = t % 2
            # phase A: the first step's copy-in; this step's gradients
            if t == 1:
                pgrp.copy_in(par, mine["p"], sg)
                read = torch.cuda.Event()
                read.record(sg)
                su.wait_event(read)          # the update rewrites the master it read
            buf = pgrp.grads_begin(par, su)
            with torch.cuda.stream(su):
                buf.copy_(grads[t - 1][r0:r0 + L])
            pgrp.grads_end(par, su)
            host_barrier()
            # phase B: the all-gather pulls and the fused update (which writes
            # the next step's slot)
            pgrp.copy_out(par, arenas[t - 1].view(torch.bfloat16)[:A], sg)
            pgrp.rs_adamw_step(par, op, mine["p"], mine["m"], mine["v"], stream=su,
                               reduced=reds[t - 1], step=t, **hp)
        torch.cuda.synchronize()
        host_barrier()
        for t in range(1, steps + 1):
            if not torch.equal(arenas[t - 1], arena_ref[t - 1]):
                msg = f"copy-out differs at step {t}"
                break
            if not torch.equal(reds[t - 1][:L * S].view(torch.int32),
                               red_ref[t - 1][rows].view(torch.int32)):
                msg = f"reduced rows differ at step {t}"
                break
            red_o = oracle.reduce_scatter(p, H.u16(grads[t - 1]), op)[rows]
            if not H.equal_nan_class(H.f32(reds[t - 1])[:L * S], red_o, "f32"):
                msg = f"reduced rows differ from the oracle at step {t}"
                break
        if msg == "ok":
            bad = [k for k in ("p", "m", "v")
                   if not torch.equal(mine[k].view(torch.int32), ref[k][rows].view(torch.int32))]
            if bad:
                msg = f"state differs after {steps} steps: {bad}"
            elif not torch.equal(pgrp.ag_slots[(steps + 1) % 2].view(torch.int16),
                                 ag_ref[rows].view(torch.int16)):
                msg = "next slot differs"
            else:
                want = H.adamw_from_state(*pre[-1], H.f32(reds[-1])[:L * S], steps, hp)
                if not all(H.adam_close_special(H.f32(mine[k]), w)[0]
                           for k, w in zip(("p", "m", "v"), want)):
                    msg = "AdamW differs from the oracle at the last step"
        pgrp.close()
    except Exception as e:  # reported through the result file
        msg = f"error: {type(e).__name__}: {e}"
    finally:
        with open(os.path.join(result_dir, f"r{rank}.txt"), "w") as f:
            f.write(msg + "\n")
        dist.destroy_process_group()


@pytest.mark.parametrize("D,case", [(2, "tiny"), (2, "uneven"), (3, "uneven"), (4, "moe")])
def test_pipelined_peer_group_over_cuda_ipc_events(H, tmp_path, D, case):
    import torch.multiprocessing as mp
    mp.spawn(_ipc_pipelined_worker, args=(_free_port(), D, case, 4, str(tmp_path)), nprocs=D,
             join=True)
    for r in range(D):
        assert open(tmp_path / f"r{r}.txt").read().strip() == "ok", f"process {r}"


def _ipc_pipelined_fp8_worker(rank, port, D, case_name, steps, result_dir):
    """The FP8 all-gather (delayed scaling) over D processes, event-ordered:
    E4M3 slot rows and partial amax arrays double buffered, each step's
    scales computed in the next step's phase B."""
    import datetime
    import torch.distributed as dist
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=D, timeout=datetime.timedelta(seconds=120))
    msg = "ok"
    try:
        torch.cuda.set_device(0)
        from fully_sharded_shard_b200 import abi
        from fully_sharded_shard_b200.peer import PipelinedPeerGroup, host_barrier
        from tests import _harness as H
        import oracle
        wl = {"uneven": W.uneven(16), "moe": W.moe(16)}[case_name]
        grp = wl.groups[0]
        N, op = wl.N, wl.op
        p = oracle.plan(grp.shapes, N)
        pgrp = PipelinedPeerGroup(grp.shapes, N, device="cuda:0", fp8=True)
        g, S, A, L, r0, n = pgrp.g, pgrp.S, pgrp.P_arena, pgrp.L, pgrp.r0, pgrp.g.n
        rows = slice(r0 * S, (r0 + L) * S)
        full = torch.empty(max(A, 1), device="cuda")
        W.fill_master(full, wl, grp.name)
        master = torch.empty(max(N * S, 1), device="cuda")
        abi.fsdp_shard_params(g, full, master)
        hp = dict(W.ADAMW_DEFAULTS)
        grads = [H.make_grads(g, wl, grp, t) for t in range(1, steps + 1)]
        # single-device references of every step
        ref = {"p": master[:N * S].clone(), "m": torch.zeros(N * S, device="cuda"),
               "v": torch.zeros(N * S, device="cuda")}
        mine = {k: t[rows].clone() for k, t in ref.items()}
        ag8_ref = torch.empty(max(N * S, 1), dtype=torch.uint8, device="cuda")
        scales_ref = [torch.empty(max(n, 1), device="cuda")]
        abi.fsdp_copy_in_fp8(g, ref["p"], ag8_ref, scales_ref[0])
        ar_ref = []
        for t in range(1, steps + 1):
            a8 = torch.full((max(A, 1),), 0xA5, dtype=torch.uint8, device="cuda")
            abi.fsdp_copy_out_fp8(g, ag8_ref, a8[:A])
            ar_ref.append(a8)
            nxt = torch.empty(max(n, 1), device="cuda")
            abi.fsdp_rs_adamw_step_fp8(g, grads[t - 1], op, ref["p"], ref["m"], ref["v"], step=t,
                                       scales_prev=scales_ref[-1], ag8_next=ag8_ref,
                                       scales_next=nxt, **hp)
            scales_ref.append(nxt)
        torch.cuda.synchronize()
        # the pipelined run
        sg, su = torch.cuda.Stream(), torch.cuda.Stream()
        scales = [scales_ref[0].clone()] + [torch.full((max(n, 1),), -1.0, device="cuda")
                                           for _ in range(steps)]
        ar = [torch.full((max(A, 1),), 0xA5, dtype=torch.uint8, device="cuda")
              for _ in range(steps)]
        torch.cuda.synchronize()
        host_barrier()
        for t in range(1, steps + 1):
            par = t % 2
            if t == 1:
                pgrp.copy_in_fp8(par, mine["p"], scales[0], sg)
                read = torch.cuda.Event()
                read.record(sg)
                su.wait_event(read)
            buf = pgrp.grads_begin(par, su)
            with torch.cuda.stream(su):
                buf.copy_(grads[t - 1][r0:r0 + L])
            pgrp.grads_end(par, su)
            host_barrier()
            if t > 1:   # the previous step's scales, from every device's partial amax
                pgrp.fp8_scales(1 - par, scales[t - 1], su)
            pgrp.copy_out_fp8(par, ar[t - 1][:A], sg)
            pgrp.rs_adamw_step_fp8(par, op, mine["p"], mine["m"], mine["v"],
                                   scales_prev=scales[t - 1], stream=su, step=t, **hp)
        host_barrier()
        pgrp.fp8_scales(steps % 2, scales[steps], su)
        torch.cuda.synchronize()
        host_barrier()
        for t in range(1, steps + 1):
            if not torch.equal(ar[t - 1], ar_ref[t - 1]):
                msg = f"FP8 copy-out differs at step {t}"
                break
            if not torch.equal(scales[t][:n].view(torch.int32), scales_ref[t][:n].view(torch.int32)):
                msg = f"scales of step {t} differ"
                break
        if msg == "ok":
            bad = [k for k in ("p", "m", "v")
                   if not torch.equal(mine[k].view(torch.int32), ref[k][rows].view(torch.int32))]
            if bad:
                msg = f"state differs after {steps} steps: {bad}"
            elif not torch.equal(pgrp.ag8_slots[(steps + 1) % 2], ag8_ref[rows]):
                msg = "next E4M3 slot differs"
            elif n and not H.bits_equal(H.f32(scales[steps])[:n],
                                        oracle.fp8_scales(p, H.f32(ref["p"]))):
                msg = "last scales differ from the oracle's"
        pgrp.close()
    except Exception as e:  # reported through the result file
        msg = f"error: {type(e).__name__}: {e}"
    finally:
        with open(os.path.join(result_dir, f"r{rank}.txt"), "w") as f:
            f.write(msg + "\n")
        dist.destroy_process_group()


@pytest.mark.parametrize("D,case", [(2, "uneven"), (4, "moe")])
def test_pipelined_peer_fp8_over_cuda_ipc_events(H, tmp_path, D, case):
    import torch.multiprocessing as mp
    mp.spawn(_ipc_pipelined_fp8_worker, args=(_free_port(), D, case, 4, str(tmp_path)),
             nprocs=D, join=True)
    for r in range(D):
        assert open(tmp_path / f"r{r}.txt").read().strip() == "ok", f"process {r}"
