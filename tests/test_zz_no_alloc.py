"""fsdp_rs_reduce_noalloc: the reduce-scatter for callers that cannot
allocate device memory (a memory pool that owns the whole device, code that
must not call cudaMalloc).  Its work table lives in a fixed array inside the
library instead of a plan's cudaMalloc'd table.

Checked through the C ABI against the planned entry point fsdp_rs_reduce on
the same inputs, bit for bit (the reduction's tolerance), on calls in a row
whose tables differ in size, so a stale table from the previous call would
show.  This file is collected last on purpose.
"""
import ctypes

import pytest
import torch

from fully_sharded_shard_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _grads(N, P_arena, seed):
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    x = torch.randn(N, P_arena, generator=g, device="cuda") * 1e-3
    return x.to(torch.bfloat16)


def _both(abi, shapes, N, op, seed):
    grp = abi.fsdp_plan_group(shapes, N)
    grads = _grads(N, grp.P_arena, seed)
    want = torch.full((N * grp.S,), -7.0, device="cuda")
    got = torch.full((N * grp.S,), -9.0, device="cuda")
    abi.fsdp_rs_reduce(grp, grads, op, want)
    abi.fsdp_rs_reduce_noalloc(shapes, N, grads, op, got, P_arena=grp.P_arena, S=grp.S)
    torch.cuda.synchronize()
    grp.destroy()
    return got, want


def test_noalloc_matches_planned_reduce_on_consecutive_calls():
    assert torch.cuda.is_available()
    from fully_sharded_shard_b200 import abi
    cases = [
        (W.uneven(8).groups[0].shapes, 6, W.SUM_THEN_DIV, 1),     # pads, shifted runs
        ([(7, 3), (5,), (1001, 3), (1, 32)], 3, W.AVG, 2),        # small table after a big one
        (W.llama_block(16).groups[0].shapes, 8, W.SUM, 3),        # larger again
        ([(9, 5), (3,)], 12, W.AVG, 4),                          # any-N path
    ]
    for shapes, N, op, seed in cases:
        got, want = _both(abi, shapes, N, op, seed)
        assert torch.equal(got.view(torch.int32), want.view(torch.int32)), (N, op)


def test_noalloc_rejects_a_table_beyond_its_limit():
    from fully_sharded_shard_b200 import abi
    n = abi.FSDP_NOALLOC_MAX_UNITS + 10           # one table entry per 1-element parameter
    shapes = [(1,)] * n
    grp = abi.fsdp_plan_group(shapes, 1)
    grads = torch.zeros(grp.P_arena, dtype=torch.bfloat16, device="cuda")
    out = torch.full((grp.S,), 3.0, device="cuda")
    _, arr = abi._descs(shapes)
    st = abi.lib().fsdp_rs_reduce_noalloc(
        arr, n, 1, ctypes.c_void_p(grads.data_ptr()), W.AVG, ctypes.c_void_p(out.data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == abi.FSDP_EINVAL
    torch.cuda.synchronize()
    assert bool((out == 3.0).all())                # nothing was enqueued
    grp.destroy()
