"""Child-process driver of tests/test_gpu_debug_build.py (run with
FSDPK_DEBUG=1, so the binding loads libfsdpk_debug.so).

  python tests/_debug_run.py grid     every stage over the brute-force grid,
                                      40 random groups, the emulated
                                      several-device pulls and groups of many
                                      small parameters (the flat paths);
                                      prints the error words (all zero expected)
  python tests/_debug_run.py shrink   the copy-out and the fused reduce-scatter
                                      (and, for a group of many small
                                      parameters, the flat copy-out,
                                      reduce-scatter and fused update) with
                                      every extent narrowed by one element;
                                      prints the error words and whether the
                                      skipped units were left untouched
"""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

from fully_sharded_shard_b200 import abi  # noqa: E402
from fully_sharded_shard_b200 import workloads as W  # noqa: E402


def grid() -> dict:
    from tests import _harness as H
    from tests.test_gpu_parity import FLAT, GRID, RANDOM, _wl
    from tests.test_gpu_peer import run_group_peer
    words = torch.zeros(4, dtype=torch.int32, device="cuda")
    abi.fsdp_debug_set_error_words(words)
    ops = [W.SUM, W.AVG, W.SUM_THEN_DIV]
    cases = 0
    for wl in GRID + RANDOM:
        grp = wl.groups[0]
        H.run_group(wl, grp, steps=2, ops=ops, staged=True)
        H.run_group_fused(wl, grp, steps=1)
        H.run_group_fp8(wl, grp)
        H.run_group_fused_fp8(wl, grp, steps=1)
        H.run_group_accumulate(wl, grp, micro=2)
        cases += 1
    for wl, D in ((_wl("dbg_peer", [(7, 3), (5,), (1, 32), (1001, 3)], 4), 2),
                  (W.uneven(16), 3)):
        run_group_peer(H, wl, wl.groups[0], D, steps=1)
        cases += 1
    # groups of many small parameters: the flat copy-out, reduce-scatter and
    # update (N = 8, 3 with a partial last vector, 11 on the any-N kernels),
    # and the packed FP8 paths
    flat = [W.small_params()] + [w for w in FLAT if w.name in ("flat_n3", "flat_n11")]
    for wl in flat:
        H.run_group(wl, wl.groups[0], steps=1, ops=ops, staged=True)
        H.run_group_fused(wl, wl.groups[0], steps=1)
        H.run_group_fused_fp8(wl, wl.groups[0], steps=1)
        cases += 1
    torch.cuda.synchronize()
    abi.fsdp_debug_set_error_words(None)
    return {"words": [int(x) for x in words.cpu()], "cases": cases}


def shrink() -> dict:
    shapes, N = [(7, 3), (5,), (1001, 3), (16386,)], 3   # rank 2 ends the [N][S] space
    g = abi.fsdp_plan_group(shapes, N)
    words = torch.zeros(4, dtype=torch.int32, device="cuda")
    abi.fsdp_debug_set_error_words(words, shrink=1)
    ag = torch.ones(N * g.S, dtype=torch.bfloat16, device="cuda")
    arena = torch.full((g.P_arena,), 7.0, dtype=torch.bfloat16, device="cuda")
    abi.fsdp_copy_out(g, ag, arena)
    torch.cuda.synchronize()
    copy_out = [int(x) for x in words.cpu()]
    # the last parameter's last rows were skipped: they keep the fill
    tail_kept = bool((arena[-8:].float() == 7.0).all())
    words.zero_()
    grads = torch.ones(N, g.P_arena, dtype=torch.bfloat16, device="cuda")
    red = torch.full((N * g.S,), -3.0, device="cuda")
    abi.fsdp_rs_reduce(g, grads, W.AVG, red)
    torch.cuda.synchronize()
    reduce = [int(x) for x in words.cpu()]
    g.destroy()
    out = {"copy_out": copy_out, "tail_kept": tail_kept, "reduce": reduce}
    # a group of many small parameters (the flat path), the same last parameter
    shapes = [(3 + k % 23, 1 + k % 5) for k in range(800)] + [(16386,)]
    g = abi.fsdp_plan_group(shapes, N)
    assert abi.fsdp_group_flat(g)[:2] == (True, True)
    NS = N * g.S
    last = int(g.arena_off[-1]) + 16385          # the last real element of the arena
    words.zero_()
    ag = torch.ones(NS, dtype=torch.bfloat16, device="cuda")
    arena = torch.full((g.P_arena,), 7.0, dtype=torch.bfloat16, device="cuda")
    abi.fsdp_copy_out(g, ag, arena)
    torch.cuda.synchronize()
    out["flat_copy_out"] = [int(x) for x in words.cpu()]
    out["flat_tail_kept"] = bool(arena[last].item() == 7.0 and arena[last - 1].item() == 1.0)
    words.zero_()
    grads = torch.ones(N, g.P_arena, dtype=torch.bfloat16, device="cuda")
    red = torch.full((NS,), -3.0, device="cuda")
    abi.fsdp_rs_reduce(g, grads, W.AVG, red)
    torch.cuda.synchronize()
    out["flat_reduce"] = [int(x) for x in words.cpu()]
    out["flat_reduce_kept"] = bool(red[-1].item() == -3.0 and red[0].item() == 1.0)
    words.zero_()
    master = torch.full((NS,), 0.5, device="cuda")
    m = torch.zeros(NS, device="cuda")
    v = torch.zeros(NS, device="cuda")
    abi.fsdp_rs_adamw_step(g, grads, W.AVG, master, m, v, step=1, **W.ADAMW_DEFAULTS)
    torch.cuda.synchronize()
    out["flat_update"] = [int(x) for x in words.cpu()]
    out["flat_update_kept"] = bool(master[-1].item() == 0.5 and master[0].item() != 0.5)
    abi.fsdp_debug_set_error_words(None)
    g.destroy()
    return out


if __name__ == "__main__":
    assert abi.fsdp_debug_build(), "not the debug library (set FSDPK_DEBUG=1)"
    torch.cuda.set_device(0)
    out = {"grid": grid, "shrink": shrink}[sys.argv[1]]()
    print("RESULT " + json.dumps(out), flush=True)
