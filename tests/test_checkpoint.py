"""Checkpoint round trip of a group's sharded state (CPU tensors here; the
GPU resume test is in test_gpu_parity.py)."""
import numpy as np
import pytest
import torch

from fully_sharded_shard_b200 import checkpoint as C


def test_round_trip_and_layout_checks(tmp_path):
    shapes, N, S = [(7, 3), (5,)], 4, 8
    g = torch.Generator().manual_seed(0)
    bufs = [torch.randn(N * S + 3, generator=g) for _ in range(3)]
    C.save_group_state(str(tmp_path), shapes, N, S, 7, *bufs)
    out = [torch.zeros(N * S) for _ in range(3)]
    assert C.load_group_state(str(tmp_path), shapes, N, S, *out) == 7
    for a, b in zip(bufs, out):
        assert torch.equal(a[:N * S], b)
    with pytest.raises(ValueError):
        C.load_group_state(str(tmp_path), shapes, 2, S, *out)
    with pytest.raises(ValueError):
        C.load_group_state(str(tmp_path), [(7, 3)], N, S, *out)
