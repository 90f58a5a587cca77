"""Pins for the oracle's reduce-scatter: packing and the rank-ordered fold.

Sources: "Introduction to PyTorch FSDP2 Backend Features", Working Principle
(All-Reduce decomposes into Reduce-Scatter + All-Gather) and Mixed Precision
(gradients cast to fp32 for the reduction); "Sharded Training: FSDP2,
DTensor, Tensor and Pipeline Parallelism", ZeRO paragraph (a ring all-reduce
is a reduce-scatter plus an all-gather), Mixed precision paragraph
(reduce_dtype fp32), Other controls and The bug Adam hid (AVG vs SUM plus
FSDP's own division by the world size).

Pins: reduce-scatter then all-gather equals an independent all-reduce (a
torch left fold over per-parameter tensors); AVG == SUM / N; SUM_THEN_DIV ==
AVG; SUM / AVG == N for power-of-two N; identity at N = 1; a brute-force
step-by-step rounded fold; and a case where only the left fold from rank 0
gives the stated result.
"""
import numpy as np
import pytest
import torch

from fully_sharded_shard_b200 import workloads as W

GROUPS = [
    ("tiny_mlp", [(32, 16), (32,), (4, 32), (4,)], 2),
    ("ragged", [(7, 3), (5,), (1, 32), (1,), (0, 4), (13, 9), (2, 2)], 4),
    ("one_rank", [(5, 3), (4,)], 1),
    ("nine_ranks", [(3, 5), (9,), (17, 2)], 9),
    ("block_div64", W.llama_block(64).groups[0].shapes, 8),
    ("uneven_div64", W.uneven(64).groups[0].shapes, 6),
    ("moe_div32", W.moe(32, experts=8, zero_experts=2).groups[0].shapes, 8),
]


def _numel(s):
    return int(np.prod(s)) if len(s) else 1


def _rank_grads(shapes, N, seed):
    """Per-rank, per-parameter bf16 gradients (torch), and the arena copy."""
    g = torch.Generator().manual_seed(seed)
    return [[torch.randn(_numel(s), generator=g).to(torch.bfloat16) for s in shapes]
            for _ in range(N)]


def _arena(p, grads):
    N = len(grads)
    a = np.zeros((N, p.P_arena), np.uint16)
    for r in range(N):
        for i, x in enumerate(grads[r]):
            a[r, p.arena_off[i]:p.arena_off[i] + x.numel()] = x.view(torch.int16).numpy().view(np.uint16)
    return a.reshape(-1)


def _allreduce(grads, i, op):
    """Independent all-reduce of parameter i: left fold in torch fp32."""
    acc = grads[0][i].float()
    for r in range(1, len(grads)):
        acc = acc + grads[r][i].float()
    if op != W.SUM:
        acc = acc / float(len(grads))
    return acc


def _gather_reduced(p, red, i):
    """all-gather of the reduced shards of parameter i, padding stripped."""
    parts = []
    for j in range(p.N):
        lo = j * p.S + int(p.shard_off[i])
        parts.append(red[lo:lo + p.valid_rows(i, j) * int(p.cols[i])])
    return np.concatenate(parts)


@pytest.mark.parametrize("form", ["packed", "direct"])
@pytest.mark.parametrize("op", [W.SUM, W.AVG, W.SUM_THEN_DIV], ids=["SUM", "AVG", "SUM_THEN_DIV"])
@pytest.mark.parametrize("name,shapes,N", GROUPS, ids=[g[0] for g in GROUPS])
def test_reduce_scatter_then_all_gather_equals_all_reduce(oracle, name, shapes, N, op, form):
    p = oracle.plan(shapes, N)
    grads = _rank_grads(shapes, N, seed=11)
    rs = oracle.reduce_scatter if form == "packed" else oracle.reduce_scatter_direct
    red = rs(p, _arena(p, grads), op)
    for i in range(p.n):
        want = _allreduce(grads, i, op).numpy()
        got = _gather_reduced(p, red, i)
        assert np.array_equal(got.view(np.uint32), want.view(np.uint32)), (name, i)
    # every pad element of the reduced shards is +0
    for j in range(N):
        for i in range(p.n):
            lo = j * p.S + int(p.shard_off[i]) + p.valid_rows(i, j) * int(p.cols[i])
            hi = j * p.S + int(p.shard_off[i]) + int(p.shard_size[i])
            assert np.all(red[lo:hi].view(np.uint32) == 0)


@pytest.mark.parametrize("name,shapes,N", GROUPS, ids=[g[0] for g in GROUPS])
def test_avg_sum_relations(oracle, name, shapes, N):
    p = oracle.plan(shapes, N)
    a = _arena(p, _rank_grads(shapes, N, seed=12))
    s = oracle.reduce_scatter(p, a, W.SUM)
    avg = oracle.reduce_scatter(p, a, W.AVG)
    std = oracle.reduce_scatter(p, a, W.SUM_THEN_DIV)
    # AVG == SUM / N (one binary32 division), and SUM-then-divide == AVG
    assert np.array_equal(avg.view(np.uint32), (s / np.float32(N)).astype(np.float32).view(np.uint32))
    assert np.array_equal(std.view(np.uint32), avg.view(np.uint32))
    if N & (N - 1) == 0:
        # division by a power of two is exact here: SUM is exactly N x AVG,
        # the "gradients exactly 2x" signature at world size 2
        assert np.array_equal(s.view(np.uint32), (avg * np.float32(N)).view(np.uint32))
    if N == 1:
        assert np.array_equal(s.view(np.uint32), avg.view(np.uint32))


@pytest.mark.parametrize("op", [W.SUM, W.AVG, W.SUM_THEN_DIV], ids=["SUM", "AVG", "SUM_THEN_DIV"])
@pytest.mark.parametrize("name,shapes,N", GROUPS, ids=[g[0] for g in GROUPS])
def test_direct_form_equals_packed_form(oracle, name, shapes, N, op):
    p = oracle.plan(shapes, N)
    a = _arena(p, _rank_grads(shapes, N, seed=15))
    x = oracle.reduce_scatter(p, a, op)
    y = oracle.reduce_scatter_direct(p, a, op)
    assert np.array_equal(x.view(np.uint32), y.view(np.uint32))


def test_world_size_one_is_a_cast(oracle):
    shapes = [(5, 3), (4,)]
    p = oracle.plan(shapes, 1)
    grads = _rank_grads(shapes, 1, seed=13)
    red = oracle.reduce_scatter(p, _arena(p, grads), W.AVG)
    want = torch.cat([x.float() for x in grads[0]]).numpy()
    assert np.array_equal(red.view(np.uint32), want.view(np.uint32))


def test_brute_force_stepwise_rounded_fold(oracle):
    """Each add is one binary32 RN add: compare with an exact binary64 add of
    the two operands (exact for these magnitudes) rounded to binary32."""
    rng = np.random.default_rng(0)
    for N in range(1, 10):
        shapes = [(int(rng.integers(1, 9)), int(rng.integers(1, 4))) for _ in range(3)]
        p = oracle.plan(shapes, N)
        a = _arena(p, _rank_grads(shapes, N, seed=100 + N))
        packed = oracle.pack(p, a).reshape(N, N * p.S)
        red = oracle.reduce_packed(p, packed.reshape(-1), W.SUM)
        for k in range(N * p.S):
            acc = np.float32(packed[0, k])
            for r in range(1, N):
                acc = np.float32(np.float64(acc) + np.float64(packed[r, k]))
            assert acc.view(np.uint32) == red[k].view(np.uint32)


def test_fold_order_is_rank_order(oracle):
    """2^24 + 1 - 2^24: the left fold from rank 0 gives 0, other orders 1."""
    shapes, N = [(3,)], 3
    p = oracle.plan(shapes, N)
    vals = [2.0 ** 24, 1.0, -(2.0 ** 24)]
    grads = [[torch.full((3,), v).to(torch.bfloat16)] for v in vals]
    red = oracle.reduce_scatter(p, _arena(p, grads), W.SUM)
    for j in range(N):
        lo = j * p.S
        assert np.all(red[lo:lo + p.valid_rows(0, j)] == 0.0)


def test_pack_layout_is_reduce_scatter_input(oracle):
    """packed[r] is rank r's reduce-scatter input: N destination chunks of S,
    each the padded shard slot of the destination rank."""
    shapes, N = [(7, 3), (5,), (1, 2)], 4
    p = oracle.plan(shapes, N)
    grads = _rank_grads(shapes, N, seed=14)
    packed = oracle.pack(p, _arena(p, grads)).reshape(N, N, p.S)
    for r in range(N):
        for j in range(N):
            for i, s in enumerate(shapes):
                x = grads[r][i].float().reshape(s[0], -1)
                ch = torch.chunk(x, N, 0)
                piece = ch[j].reshape(-1) if j < len(ch) else torch.zeros(0)
                lo = int(p.shard_off[i])
                seg = packed[r, j, lo:lo + int(p.shard_size[i])]
                assert np.array_equal(seg[:piece.numel()], piece.numpy())
                assert np.all(seg[piece.numel():].view(np.uint32) == 0)
