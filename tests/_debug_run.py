"""Child-process driver of tests/test_gpu_debug_build.py (run with
FSDPK_DEBUG=1, so the binding loads libfsdpk_debug.so).

  python tests/_debug_run.py grid     every stage over the brute-force grid,
                                      40 random groups, the emulated
                                      several-device pulls and a group of 3000
                                      small parameters (the packed paths);
                                      prints the error words (all zero expected)
  python tests/_debug_run.py shrink   the copy-out and the fused reduce-scatter
                                      with every extent narrowed by one
                                      element; prints the error words and
                                      whether the skipped units were left
                                      untouched
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
    from tests.test_gpu_parity import GRID, RANDOM, _wl
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
    wl = W.small_params()          # the packed copy-out, reduce-scatter and update paths
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
    abi.fsdp_debug_set_error_words(None)
    g.destroy()
    return {"copy_out": copy_out, "tail_kept": tail_kept, "reduce": reduce}


if __name__ == "__main__":
    assert abi.fsdp_debug_build(), "not the debug library (set FSDPK_DEBUG=1)"
    torch.cuda.set_device(0)
    out = {"grid": grid, "shrink": shrink}[sys.argv[1]]()
    print("RESULT " + json.dumps(out), flush=True)
