"""Pins for the oracle's FP8 (E4M3) all-gather copy-in and copy-out.

"PyTorch FSDP2 Guide: Distributed LLM Training with DTensor", Deep Dive
section "2. Native FP8 Training with Float8Tensor": parameters in FP8 E4M3,
the all-gather moves raw FP8 bytes (half the bf16 traffic).  The pages do not
fix the scaling; the reading is per-parameter tensorwise dynamic scaling
(scale = 448 / max(amax, 1e-12) in binary32, clamp to +-448, round to nearest
even).

Pins: the E4M3 rounding against torch's float8_e4m3fn cast over every binary32
pattern with exponent in [-12, 8] (all mantissas, both signs) plus zeros, the
largest finite value, ties and NaN; the scales against numpy's max|x|; the
copy-in against torch (x * scale, clamp, cast) laid out with torch.chunk and
zero pad rows; the copy-out as the round trip all-gather(shard(q)) == q.
"""
import numpy as np
import torch

from fully_sharded_shard_b200 import workloads as W


def _torch_e4m3(x: np.ndarray) -> np.ndarray:
    return torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_e4m3_rounding_against_torch(oracle):
    base = np.arange(1 << 23, dtype=np.uint32)
    for sign in (0, 1):
        for e in range(-12, 9):
            bits = base | np.uint32(((e + 127) << 23) | (sign << 31))
            x = bits.view(np.float32)
            x = x[np.abs(x) <= 448.0]
            got = oracle.e4m3_bits(x)
            want = _torch_e4m3(x)
            bad = got != want
            assert not bad.any(), (e, sign, float(x[np.argmax(bad)]))


def test_e4m3_special_values(oracle):
    L = oracle.lib()
    cases = [(0.0, 0x00), (-0.0, 0x80), (448.0, 0x7E), (-448.0, 0xFE), (2.0 ** -6, 0x08),
             (2.0 ** -9, 0x01), (2.0 ** -10, 0x00), (3 * 2.0 ** -11, 0x01), (1.0, 0x38),
             (1.0625, 0x38), (1.1875, 0x3A), (240.0, 0x77), (256.0, 0x78)]
    for x, want in cases:
        assert L.or_e4m3_bits(x) == want, (x, hex(L.or_e4m3_bits(x)))
    assert L.or_e4m3_bits(float("nan")) & 0x7F == 0x7F
    # the clamp keeps everything finite: x * scale beyond 448 maps to 448
    assert L.or_fp8_quant_input(1e9, 1.0) == 448.0 and L.or_fp8_quant_input(-464.0, 1.0) == -448.0
    assert L.or_fp8_scale(0.0) == np.float32(448.0) / np.float32(1e-12)


def _group(shapes, N, seed):
    g = torch.Generator().manual_seed(seed)
    params = [torch.randn(*s, generator=g) * 0.02 for s in shapes]
    return params


def test_scales_and_copy_in_against_torch(oracle):
    shapes, N = [(7, 3), (5,), (1, 32), (13, 9), (2, 2), (0, 4)], 4
    params = _group(shapes, N, 1)
    params[4] = torch.zeros(2, 2)               # an all-zero parameter: amax floor
    params[1][2] = 1e6                          # saturates nothing: scale shrinks
    p = oracle.plan(shapes, N)
    arena = np.zeros(p.P_arena, np.float32)
    for i, x in enumerate(params):
        arena[p.arena_off[i]:p.arena_off[i] + x.numel()] = x.reshape(-1).numpy()
    master = oracle.shard(p, arena)
    scales = oracle.fp8_scales(p, master)
    for i, x in enumerate(params):
        amax = np.float32(np.max(np.abs(x.numpy()))) if x.numel() else np.float32(0)
        want = np.float32(448.0) / np.maximum(amax, np.float32(1e-12))
        assert scales[i].view(np.uint32) == np.float32(want).view(np.uint32)
    ag8 = oracle.copy_in_fp8(p, master, scales)
    for r in range(N):
        parts = []
        for i, x in enumerate(params):
            x2 = x.reshape(x.shape[0], int(np.prod(x.shape[1:])) if x.dim() > 1 else 1)
            ch = torch.chunk(x2, N, 0)
            c = int(p.chunk_rows[i])
            piece = ch[r] if r < len(ch) else x2[:0]
            y = (piece * torch.tensor(scales[i])).clamp(-448.0, 448.0)
            q = y.to(torch.float8_e4m3fn).view(torch.uint8).reshape(-1)
            parts.append(torch.cat([q, torch.zeros((c - piece.shape[0]) * x2.shape[1], dtype=torch.uint8)]))
        want = torch.cat(parts).numpy()
        assert np.array_equal(ag8[r * p.S:(r + 1) * p.S], want), r


def test_copy_out_round_trip(oracle):
    shapes, N = W.uneven(64).groups[0].shapes, 6
    p = oracle.plan(shapes, N)
    rng = np.random.default_rng(2)
    arena = rng.normal(0, 0.02, p.P_arena).astype(np.float32)
    master = oracle.shard(p, arena)
    scales = oracle.fp8_scales(p, master)
    ag8 = oracle.copy_in_fp8(p, master, scales)
    out = oracle.copy_out_fp8(p, ag8, np.full(p.P_arena, 0xA5, np.uint8))
    for i in range(p.n):
        n = int(p.d0[i] * p.cols[i])
        a = p.arena_off[i]
        x = arena[a:a + n]
        want = oracle.e4m3_bits(np.clip(x * scales[i], -448, 448).astype(np.float32))
        assert np.array_equal(out[a:a + n], want)
