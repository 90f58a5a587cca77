"""Pins for gradient accumulation without sync.

"Sharded Training: FSDP2, DTensor, Tensor and Pipeline Parallelism", Other
controls paragraph: set_requires_gradient_sync(False) accumulates the
unsharded gradients and skips the reduce-scatter.  Reading: each rank keeps
its unsharded gradient in reduce_dtype fp32, a left fold over microbatches;
the last microbatch reduce-scatters the fp32 sum.

Pins: the accumulation against torch's fp32 adds (a library routine); the
fp32 reduce-scatter against an independent torch all-reduce of the
accumulated per-parameter gradients (RS + AG == AR); with one microbatch the
fp32 path equals the bf16 reduce-scatter bit for bit; and a case where the
microbatch order of the fold decides the result.
"""
import numpy as np
import pytest
import torch

from fully_sharded_shard_b200 import workloads as W

GROUPS = [
    ("ragged", [(7, 3), (5,), (1, 32), (1,), (0, 4), (13, 9), (2, 2)], 4),
    ("n3", [(1001, 3), (17,)], 3),
    ("block_div64", W.llama_block(64).groups[0].shapes, 8),
]


def _bf16(shape, gen):
    return torch.randn(shape, generator=gen).to(torch.bfloat16)


def _u16(t):
    return t.view(torch.int16).numpy().view(np.uint16).reshape(-1)


def test_accumulate_matches_torch_fp32_adds(oracle):
    gen = torch.Generator().manual_seed(3)
    micro = [_bf16((4, 1001), gen) for _ in range(5)]
    acc = np.empty(4 * 1001, np.float32)
    want = None
    for t, g in enumerate(micro):
        oracle.accumulate(acc, _u16(g), first=(t == 0))
        want = g.float() if want is None else want + g.float()
        assert np.array_equal(acc.view(np.uint32), want.reshape(-1).numpy().view(np.uint32))


def test_accumulation_order_is_microbatch_order(oracle):
    # 2^24 + 1 - 2^24 over three microbatches: the left fold gives 0
    vals = [2.0 ** 24, 1.0, -(2.0 ** 24)]
    acc = np.empty(8, np.float32)
    for t, x in enumerate(vals):
        oracle.accumulate(acc, _u16(torch.full((8,), x).to(torch.bfloat16)), first=(t == 0))
    assert np.all(acc == 0.0)


@pytest.mark.parametrize("op", [W.SUM, W.AVG, W.SUM_THEN_DIV], ids=["SUM", "AVG", "SUM_THEN_DIV"])
@pytest.mark.parametrize("name,shapes,N", GROUPS, ids=[g[0] for g in GROUPS])
def test_fp32_reduce_scatter_then_all_gather_equals_all_reduce(oracle, name, shapes, N, op):
    p = oracle.plan(shapes, N)
    gen = torch.Generator().manual_seed(4)
    M = 3
    # per-rank, per-parameter microbatch gradients
    g = [[[_bf16(int(np.prod(s)) if len(s) else 1, gen) for s in shapes] for _ in range(N)]
         for _ in range(M)]
    acc = np.zeros(N * p.P_arena, np.float32)
    for t in range(M):
        arena = np.zeros((N, p.P_arena), np.uint16)
        for r in range(N):
            for i in range(p.n):
                x = g[t][r][i]
                arena[r, p.arena_off[i]:p.arena_off[i] + x.numel()] = _u16(x)
        oracle.accumulate(acc, arena.reshape(-1), first=(t == 0))
    red = oracle.reduce_scatter_f32(p, acc, op)
    for i in range(p.n):
        # independent all-reduce: per rank, microbatch fold in fp32; then rank fold
        per_rank = []
        for r in range(N):
            a = g[0][r][i].float()
            for t in range(1, M):
                a = a + g[t][r][i].float()
            per_rank.append(a)
        ar = per_rank[0]
        for r in range(1, N):
            ar = ar + per_rank[r]
        if op != W.SUM:
            ar = ar / float(N)
        parts = []
        for j in range(N):
            lo = j * p.S + int(p.shard_off[i])
            parts.append(red[lo:lo + p.valid_rows(i, j) * int(p.cols[i])])
        assert np.array_equal(np.concatenate(parts).view(np.uint32), ar.numpy().view(np.uint32))


@pytest.mark.parametrize("name,shapes,N", GROUPS, ids=[g[0] for g in GROUPS])
def test_single_microbatch_equals_bf16_reduce_scatter(oracle, name, shapes, N):
    p = oracle.plan(shapes, N)
    gen = torch.Generator().manual_seed(5)
    grads = _u16(_bf16(N * p.P_arena, gen))
    acc = np.empty(N * p.P_arena, np.float32)
    oracle.accumulate(acc, grads, first=True)
    for op in (W.SUM, W.AVG):
        a = oracle.reduce_scatter_f32(p, acc, op)
        b = oracle.reduce_scatter_direct(p, grads, op)
        assert np.array_equal(a.view(np.uint32), b.view(np.uint32))
