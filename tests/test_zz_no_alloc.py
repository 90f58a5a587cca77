"""fsdp_rs_reduce_noalloc: the reduce-scatter for callers that cannot
allocate device memory (a memory pool that owns the whole device, code that
must not call cudaMalloc).  Its work table lives in a fixed array inside the
library instead of a plan's cudaMalloc'd table.

Checked through the C ABI, bit for bit (the reduction is exact), against the
CPU oracle and against the planned entry point fsdp_rs_reduce on the same
inputs, on calls in a row whose tables differ in size, so a stale table from
the previous call would show: once with a synchronisation after each call,
then with every call queued back to back on one non-default stream while
the device's free memory is watched.  This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from fully_sharded_shard_b200 import workloads as W

pytestmark = pytest.mark.gpu

CASES = [
    (W.uneven(8).groups[0].shapes, 6, W.SUM_THEN_DIV, 1),     # pads, shifted runs
    ([(7, 3), (5,), (1001, 3), (1, 32)], 3, W.AVG, 2),        # small table after a big one
    (W.llama_block(16).groups[0].shapes, 8, W.SUM, 3),        # larger again
    ([(9, 5), (3,)], 12, W.AVG, 4),                          # any-N path
]


def _grads(N, P_arena, seed):
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    x = torch.randn(N, max(P_arena, 1), generator=g, device="cuda") * 1e-3
    return x.to(torch.bfloat16)


def _bits(t):
    return t.detach().cpu().numpy().reshape(-1).view(np.uint32)


@pytest.fixture(scope="module")
def prepared():
    """Per case: the gradients, the oracle's reduced shards and the planned
    entry point's result (made before any no-alloc call)."""
    assert torch.cuda.is_available()
    oracle.build()
    from fully_sharded_shard_b200 import abi
    out = []
    for shapes, N, op, seed in CASES:
        grp = abi.fsdp_plan_group(shapes, N)
        p = oracle.plan(shapes, N)
        grads = _grads(N, grp.P_arena, seed)
        want = torch.full((N * grp.S,), -7.0, device="cuda")
        abi.fsdp_rs_reduce(grp, grads, op, want)
        torch.cuda.synchronize()
        grads_h = grads[:, :p.P_arena].contiguous().view(torch.int16).cpu().numpy() \
            .view(np.uint16).reshape(-1)
        red_o = oracle.reduce_scatter_direct(p, grads_h, op)
        assert np.array_equal(_bits(want), red_o.view(np.uint32)), "planned reduce != oracle"
        out.append(dict(shapes=shapes, N=N, op=op, grads=grads, want=want,
                        red_o=red_o.view(np.uint32), NS=N * grp.S))
        grp.destroy()
    return abi, out


def test_noalloc_matches_oracle_and_planned_reduce_on_consecutive_calls(prepared):
    abi, cases = prepared
    for c in cases:
        got = torch.full((c["NS"],), -9.0, device="cuda")
        abi.fsdp_rs_reduce_noalloc(c["shapes"], c["N"], c["grads"], c["op"], got)
        torch.cuda.synchronize()
        assert np.array_equal(_bits(got), c["red_o"]), (c["N"], c["op"], "vs oracle")
        assert torch.equal(got.view(torch.int32), c["want"].view(torch.int32))


def test_noalloc_back_to_back_on_one_stream_allocates_nothing(prepared):
    abi, cases = prepared
    s = torch.cuda.Stream()
    # warm-up: every kernel variant these calls use has run once on this device
    for c in cases:
        abi.fsdp_rs_reduce_noalloc(c["shapes"], c["N"], c["grads"], c["op"],
                                   torch.empty(c["NS"], device="cuda"), stream=s)
    outs = [torch.full((c["NS"],), -5.0, device="cuda") for c in cases]
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for rep in range(2):
        for c, got in zip(cases, outs):   # different tables, no sync in between
            abi.fsdp_rs_reduce_noalloc(c["shapes"], c["N"], c["grads"], c["op"], got, stream=s)
    s.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0, f"free device memory changed by {free0 - free1} bytes"
    for c, got in zip(cases, outs):
        assert np.array_equal(_bits(got), c["red_o"]), (c["N"], c["op"])


def test_noalloc_refuses_a_capturing_stream(prepared):
    abi, cases = prepared
    c = cases[1]
    got = torch.full((c["NS"],), 3.0, device="cuda")
    x = torch.zeros(1, device="cuda")
    s = torch.cuda.Stream()
    graph = torch.cuda.CUDAGraph()
    torch.cuda.synchronize()
    with torch.cuda.graph(graph, stream=s):
        x.add_(1.0)
        with pytest.raises(abi.FsdpError) as err:
            abi.fsdp_rs_reduce_noalloc(c["shapes"], c["N"], c["grads"], c["op"], got)
    assert err.value.status == abi.FSDP_ESTATE
    torch.cuda.synchronize()
    assert bool((got == 3.0).all())                # nothing was enqueued
    del graph


def test_noalloc_rejects_a_table_beyond_its_limit(prepared):
    abi, _ = prepared
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
