"""The 2 + 2 + 12 bytes-per-parameter accounting and the layout's sizes.

Printed figures (tests/golden/worked_examples.json): 16 bytes/param, a 7 B
model needs 112 GB (104.3 GiB) and ZeRO-3 over 8 ranks 14 GB ("Sharded
Training: FSDP2, DTensor, Tensor and Pipeline Parallelism", opening
paragraph and Fence 1); 70 B needs 140 + 140 + 560 + 280 = 1,120 GB against an
80 GB H100 ("PyTorch FSDP2 Guide: Distributed LLM Training with DTensor", The
Hidden Memory Tax of Legacy FSDP1).  The oracle's plan must reproduce the
per-rank share: fp32 master + m + v is 12 bytes per padded element, split
into N equal shards.
"""
import numpy as np

from fully_sharded_shard_b200 import workloads as W


def _zero_bytes(P, n, stage):
    """Per-rank bytes under ZeRO stage `stage` (0 = DDP): the optimizer state
    (12 B/param) is divided by n from stage 1, gradients (2 B) from stage 2,
    parameters (2 B) from stage 3."""
    opt = 12 * P / (n if stage >= 1 else 1)
    grads = 2 * P / (n if stage >= 2 else 1)
    params = 2 * P / (n if stage >= 3 else 1)
    return params + grads + opt


def test_printed_figures(golden):
    a = golden["accounting"]
    bpp = a["bytes_per_param"]
    assert bpp["bf16_weights"] + bpp["bf16_grads"] + bpp["fp32_master_m_v"] == bpp["total"] == 16
    assert a["P_7b"] * 16 == a["bytes_7b"]
    assert round(a["bytes_7b"] / 2 ** 30, 1) == a["gib_7b"]
    assert _zero_bytes(a["P_7b"], 64, 0) == a["bytes_7b"]
    assert _zero_bytes(a["P_7b"], 8, 3) == a["zero3_n8_bytes_7b"] == 16 * a["P_7b"] / 8
    for n in (1, 8, 64):
        row = [_zero_bytes(a["P_7b"], n, s) for s in range(4)]
        assert all(x >= y for x, y in zip(row, row[1:]))
    parts = a["parts_70b_gb"]
    P70 = a["P_70b"]
    assert parts["weights_bf16"] == 2 * P70 / 1e9 and parts["grads_bf16"] == 2 * P70 / 1e9
    assert parts["adam_m_v_fp32"] == 8 * P70 / 1e9 and parts["master_fp32"] == 4 * P70 / 1e9
    assert sum(parts.values()) == a["total_70b_gb"] == 16 * P70 / 1e9 > a["h100_gb"]


def test_sharded_state_is_twelve_bytes_per_element_over_n_ranks(oracle):
    wl = W.llama7b()
    total_padded = 0
    for g in wl.groups:
        p = oracle.plan(g.shapes, wl.N)
        total_padded += g.repeat * wl.N * p.S
    P = wl.total_params()
    assert total_padded == P == 6_738_415_616    # no padding at N = 8
    state = 12 * total_padded
    assert abs(state / 1e9 - 80.86) < 0.01        # fp32 master + m + v
    assert state / wl.N == _zero_bytes(P, wl.N, 3) - 4 * P / wl.N
