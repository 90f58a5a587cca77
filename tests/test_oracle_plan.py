"""Pins for the oracle's plan: torch.chunk rows, padded shard sizes, offsets.

The plan follows the fully_shard paragraph of "Sharded Training: FSDP2,
DTensor, Tensor and Pipeline Parallelism": rank r keeps chunk r of
torch.chunk(param, world, dim=0), padded when rows do not divide evenly.
It is pinned to torch.chunk itself (a library routine), to brute force, and
to the worked shapes the pages print (tests/golden/worked_examples.json).
"""
import numpy as np
import pytest
import torch

from fully_sharded_shard_b200 import workloads as W


def _torch_rows(d0, N):
    """Rows per rank as torch.chunk hands them out (missing chunks -> 0)."""
    t = torch.empty(d0, 1)
    chunks = torch.chunk(t, N, dim=0)
    rows = [c.shape[0] for c in chunks] + [0] * (N - len(chunks))
    return rows[:N]


def test_chunk_rows_brute_force(oracle):
    for N in range(1, 10):
        for d0 in range(0, 65):
            rows = _torch_rows(d0, N)
            c = oracle.chunk_rows(d0, N)
            # the padded shard height is the largest chunk torch hands out
            assert c == max(rows), (d0, N)
            for r in range(N):
                assert oracle.valid_rows(d0, N, r) == rows[r], (d0, N, r)
            assert sum(oracle.valid_rows(d0, N, r) for r in range(N)) == d0


@pytest.mark.parametrize("wl", [W.tiny_mlp(), W.llama_block(), W.uneven(),
                                W.moe(), W.llama7b()], ids=lambda w: w.name)
def test_plan_matches_torch_chunk_on_every_config_shape(oracle, wl):
    for g in wl.groups:
        p = oracle.plan(g.shapes, wl.N)
        S = 0
        for i, shp in enumerate(g.shapes):
            rows = _torch_rows(shp[0], wl.N)
            cols = int(np.prod(shp[1:])) if len(shp) > 1 else 1
            assert p.chunk_rows[i] == max(rows)
            assert p.shard_size[i] == max(rows) * cols
            assert p.shard_off[i] == S
            S += max(rows) * cols
            assert p.arena_off[i] % 8 == 0
            for r in range(wl.N):
                assert p.valid_rows(i, r) == rows[r]
        assert p.S == S
        assert p.P == sum(int(np.prod(s)) for s in g.shapes)
        # arena: parameters in order, no overlap, starts on 8-element bounds
        ends = p.arena_off + p.d0 * p.cols
        assert np.all(p.arena_off[1:] >= ends[:-1])
        assert p.P_arena >= int(ends[-1]) and p.P_arena % 8 == 0


def test_worked_shapes_from_the_pages(oracle, golden):
    for ex in golden["shard_shapes"]:
        shp, N = ex["shape"], ex["N"]
        p = oracle.plan([tuple(shp)], N)
        if "local_shape_every_rank" in ex:
            loc = ex["local_shape_every_rank"]
            for r in range(N):
                assert p.valid_rows(0, r) == loc[0]
            assert p.chunk_rows[0] == loc[0]
            assert p.cols[0] == int(np.prod(loc[1:]))
        if "local_rows_per_rank" in ex:
            assert [p.valid_rows(0, r) for r in range(N)] == ex["local_rows_per_rank"]
        if "rank_rows" in ex:
            # the rows of the logical tensor that each rank holds
            c = int(p.chunk_rows[0])
            for r, rows in enumerate(ex["rank_rows"]):
                got = list(range(r * c, r * c + p.valid_rows(0, r)))
                assert got == rows


def test_tiny_mlp_sizes_and_zero1_contrast(oracle, golden):
    t = golden["tiny_mlp"]
    shapes = [tuple(s) for s in t["shapes"]]
    assert [int(np.prod(s)) for s in shapes] == t["numel"]
    p = oracle.plan(shapes, 2)
    # FSDP2: every parameter is split along dim 0 -> equal padded shards
    assert list(p.shard_size) == [256, 16, 64, 2]
    assert p.S == 338 and p.P == 676
    per_rank_real = [sum(p.valid_rows(i, r) * int(p.cols[i]) for i in range(p.n))
                     for r in range(2)]
    assert per_rank_real == [338, 338]
    ratio = per_rank_real[0] / p.P
    lo, hi = t["lab_shard_ratio_bounds"]
    assert lo <= ratio <= hi
    # ZeroRedundancyOptimizer partitions whole tensors: 1,024 vs 328 Adam
    # elements (2 moments each) -- far outside the same bounds.
    z0, z1 = t["zero1_adam_elements_rank0"], t["zero1_adam_elements_rank1"]
    assert z0 == 2 * t["numel"][0] and z1 == 2 * sum(t["numel"][1:])
    assert not (lo <= z0 / (z0 + z1) <= hi)


def test_uneven_config_really_pads(oracle):
    wl = W.uneven()
    p = oracle.plan(wl.groups[0].shapes, wl.N)
    # [32003, 4096] over 6 ranks: c = 5334, rank 5 holds 5333 rows
    assert p.chunk_rows[0] == 5334 and p.valid_rows(0, 5) == 5333
    # [4096] over 6 ranks: c = 683, rank 5 holds 681 rows
    assert p.chunk_rows[2] == 683 and p.valid_rows(2, 5) == 681
    assert wl.N * p.S > p.P


def test_llama7b_has_no_padding_and_its_sizes(oracle):
    wl = W.llama7b()
    blk, root = wl.groups
    pb = oracle.plan(blk.shapes, 8)
    pr = oracle.plan(root.shapes, 8)
    assert pb.S == 25_297_920 and pr.S == 32_768_512
    assert 8 * pb.S == pb.P and 8 * pr.S == pr.P
    assert blk.repeat * pb.P + pr.P == 6_738_415_616 == wl.total_params()


def test_empty_and_degenerate_parameters(oracle):
    # d0 = 0 parameters and N = 1 are legal
    p = oracle.plan([(0, 5), (3,), (0,)], 4)
    assert list(p.chunk_rows) == [0, 1, 0]
    assert p.S == 1
    p1 = oracle.plan([(7, 3)], 1)
    assert p1.S == 21 and p1.valid_rows(0, 0) == 7
