"""Pins for the oracle's binary32 -> bfloat16 round-to-nearest-even.

The cast is the MixedPrecisionPolicy(param_dtype=torch.bfloat16) step of the
all-gather copy-in ("Sharded Training: FSDP2, DTensor, Tensor and Pipeline
Parallelism", Mixed precision paragraph; "Introduction to PyTorch FSDP2
Backend Features", Mixed Precision).  The oracle computes it from the bit
pattern; here it is checked against torch's own CPU conversion over every one
of the 2^32 binary32 bit patterns, and against hand-worked special values.
NaN payloads are not part of the contract: any NaN must map to a NaN.
"""
import numpy as np
import pytest
import torch


def _torch_bf16_bits(u32: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(u32.view(np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def test_special_values(oracle):
    cases = {
        0x00000000: 0x0000,   # +0
        0x80000000: 0x8000,   # -0
        0x7F800000: 0x7F80,   # +Inf
        0xFF800000: 0xFF80,   # -Inf
        0x3F800000: 0x3F80,   # 1.0
        0x3F808000: 0x3F80,   # 1 + half ulp, tie -> even (down)
        0x3F818000: 0x3F82,   # tie with odd lsb -> up
        0x3F808001: 0x3F81,   # just above the tie -> up
        0x3F807FFF: 0x3F80,   # just below the tie -> down
        0x7F7FFFFF: 0x7F80,   # max finite rounds to +Inf
        0x7F7F7FFF: 0x7F7F,   # stays finite
        0x00000001: 0x0000,   # smallest subnormal rounds to +0
        0x00008000: 0x0000,   # subnormal tie, even -> down
        0x00018000: 0x0002,   # subnormal tie, odd -> up
        0x007FFFFF: 0x0080,   # largest subnormal rounds up to min normal
    }
    for x, want in cases.items():
        assert oracle.lib().or_bf16_rne_bits(x) == want, hex(x)
    for nan in (0x7FC00000, 0xFFC00000, 0x7F800001, 0xFF800001, 0x7FFFFFFF):
        h = oracle.lib().or_bf16_rne_bits(nan)
        assert (h & 0x7F80) == 0x7F80 and (h & 0x7F) != 0, hex(nan)


def test_exhaustive_against_torch(oracle):
    step = 1 << 24
    base = np.arange(step, dtype=np.uint32)
    for hi in range(0, 1 << 32, step):
        u = base + np.uint32(hi)
        got = oracle.bf16_bits_from_u32(u)
        want = _torch_bf16_bits(u)
        isnan = np.isnan(u.view(np.float32))
        bad = (got != want) & ~isnan
        assert not bad.any(), hex(int(u[np.argmax(bad)]))
        g_nan = got[isnan]
        assert np.all(((g_nan & 0x7F80) == 0x7F80) & ((g_nan & 0x7F) != 0))


def test_bf16_to_f32_is_exact_widening(oracle):
    h = np.arange(1 << 16, dtype=np.uint16)
    f = oracle.bf16_to_f32(h)
    want = torch.from_numpy(h.view(np.int16)).view(torch.bfloat16).float().numpy()
    same = (f.view(np.uint32) == want.view(np.uint32)) | (np.isnan(f) & np.isnan(want))
    assert same.all()
