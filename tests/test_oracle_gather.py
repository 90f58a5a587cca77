"""Pins for the oracle's shard, all-gather copy-in and copy-out.

"Introduction to PyTorch FSDP2 Backend Features", Working Principle: the
all-gather turns the shards back into the full parameters before compute.
"Sharded Training: FSDP2, DTensor, Tensor and Pipeline Parallelism",
fully_shard paragraph (chunk r of torch.chunk, internal padding) and Mixed
precision paragraph (bf16 copies are gathered).

The expected buffers are built here from torch library routines
(torch.chunk, zero-row padding by torch.cat, .to(torch.bfloat16)), and the
round trip all_gather(shard(x)) == bf16(x) is checked as an invariant.
"""
import numpy as np
import pytest
import torch

from fully_sharded_shard_b200 import workloads as W

SMALL_GROUPS = [
    ("tiny_mlp", [(32, 16), (32,), (4, 32), (4,)], 2),
    ("ragged", [(7, 3), (5,), (1, 32), (1,), (0, 4), (13, 9), (2, 2)], 4),
    ("one_rank", [(5, 3), (4,)], 1),
    ("many_ranks", [(3, 5), (9,), (17, 2)], 9),
    ("block_div64", W.llama_block(64).groups[0].shapes, 8),
    ("uneven_div64", W.uneven(64).groups[0].shapes, 6),
]


def _cols(shape):
    return int(np.prod(shape[1:])) if len(shape) > 1 else 1


def _full_params(shapes, seed):
    g = torch.Generator().manual_seed(seed)
    return [torch.randn(*s, generator=g) if len(s) else torch.randn(1, generator=g)
            for s in shapes]


def _arena_of(p, params, dtype=np.float32):
    a = np.zeros(p.P_arena, dtype)
    for i, x in enumerate(params):
        flat = x.reshape(-1).numpy()
        a[p.arena_off[i]:p.arena_off[i] + flat.size] = flat
    return a


def _torch_shard_rank(x, N, r):
    """Rank r's padded Shard(0) piece, built with torch.chunk + zero rows."""
    x2 = x.reshape(x.shape[0], _cols(tuple(x.shape)))
    chunks = torch.chunk(x2, N, dim=0)
    c = chunks[0].shape[0] if len(chunks) else 0
    piece = chunks[r] if r < len(chunks) else x2[:0]
    pad = torch.zeros(c - piece.shape[0], x2.shape[1], dtype=x2.dtype)
    return torch.cat([piece, pad], 0).reshape(-1)


@pytest.mark.parametrize("name,shapes,N", SMALL_GROUPS, ids=[g[0] for g in SMALL_GROUPS])
def test_shard_and_copy_in_match_torch_chunk(oracle, name, shapes, N):
    p = oracle.plan(shapes, N)
    params = _full_params(shapes, seed=3)
    master = oracle.shard(p, _arena_of(p, params))
    ag = oracle.copy_in(p, master)
    for r in range(N):
        slot = torch.cat([_torch_shard_rank(x, N, r) for x in params]) if params else torch.zeros(0)
        assert slot.numel() == p.S
        got_master = master[r * p.S:(r + 1) * p.S]
        assert np.array_equal(got_master.view(np.uint32), slot.numpy().view(np.uint32))
        want_ag = slot.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        assert np.array_equal(ag[r * p.S:(r + 1) * p.S], want_ag)


@pytest.mark.parametrize("name,shapes,N", SMALL_GROUPS, ids=[g[0] for g in SMALL_GROUPS])
def test_all_gather_of_shard_is_identity(oracle, name, shapes, N):
    """all-gather(shard(x)) == x, in bf16 (param_dtype) here."""
    p = oracle.plan(shapes, N)
    params = _full_params(shapes, seed=5)
    master = oracle.shard(p, _arena_of(p, params))
    sentinel = np.uint16(0xBEEF)
    arena = np.full(p.P_arena, sentinel, np.uint16)
    out = oracle.copy_out(p, oracle.copy_in(p, master), arena)
    covered = np.zeros(p.P_arena, bool)
    for i, x in enumerate(params):
        want = x.reshape(-1).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        a = p.arena_off[i]
        assert np.array_equal(out[a:a + want.size], want)
        covered[a:a + want.size] = True
    # alignment gaps between parameters are never written
    assert np.all(out[~covered] == sentinel)


def test_pad_rows_are_zero_even_if_master_pad_is_not(oracle):
    """The copy-in writes +0 into every pad row regardless of master bytes."""
    shapes, N = [(5, 3), (3,)], 4
    p = oracle.plan(shapes, N)
    master = np.full(N * p.S, -7.5, np.float32)
    ag = oracle.copy_in(p, master)
    for r in range(N):
        for i in range(p.n):
            v = p.valid_rows(i, r) * int(p.cols[i])
            lo = r * p.S + int(p.shard_off[i])
            assert np.all(ag[lo:lo + v] == 0xC0F0)          # bf16(-7.5)
            assert np.all(ag[lo + v:lo + int(p.shard_size[i])] == 0)


def test_shard_pads_are_positive_zero(oracle):
    shapes, N = [(13, 9), (2,)], 4
    p = oracle.plan(shapes, N)
    arena = np.full(p.P_arena, -1.0, np.float32)
    master = oracle.shard(p, arena)
    for r in range(N):
        for i in range(p.n):
            v = p.valid_rows(i, r) * int(p.cols[i])
            lo = r * p.S + int(p.shard_off[i])
            assert np.all(master[lo:lo + v] == -1.0)
            assert np.all(master[lo + v:lo + int(p.shard_size[i])].view(np.uint32) == 0)
