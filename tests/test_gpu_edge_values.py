"""GPU parity on the values where hardware conversions and the pages'
definitions can part: every stage, through the C ABI, on a hand-built group
whose masters and per-rank gradients hold the special values, against the
CPU oracle applied to the GPU's own inputs.

The group (N = 3, 8 and 12 ranks, so the 3-rank, 8-rank and any-N kernels
all run):
  p0 [6, 7]    masters: quiet and signalling NaN with payloads, +-Inf, +-0,
               the largest finite binary32 (rounds to +Inf in bf16), exact
               bf16 round-to-nearest-even ties on both parities (normal,
               subnormal, next to the largest finite), subnormals;
               gradients per rank (the fold): 2^24, 1, -2^24 in three orders
               (a left fold from rank 0 is the only order that gives these
               bits), -0 on every rank, -0 / +0 mixes, +Inf + -Inf, NaN,
               the largest finite bf16 summed into overflow and back,
               bf16 subnormals, and reduced gradients beyond 5.8e20 where
               (1 - b2) g^2 overflows binary32 in AdamW;
  p1 [11]      a NaN beside finite values (the FP8 amax must skip it);
  p2 [5, 4]    amax 448, so the FP8 scale is exactly 1: E4M3 ties on both
               parities, E4M3 subnormals and their ties, +-0, +-448;
  p3 [4, 3]    an amax whose scaled value rounds above 448 (the clamp
               saturates it), and a gradient that pushes it further under the
               delayed scale of the fused update;
  p4 [1000, 3] seeded values with the fold triples again at the head, over
               several work units with pad rows;
  p5 [7]       seeded values.
Data movement is bit-exact (NaN payloads included); arithmetic outputs are
bit-exact with NaN compared as a class (the pages fix no NaN encoding);
AdamW is within 1e-6 * (1 + |x|), infinities equal and NaN meeting NaN.
"""
import numpy as np
import pytest
import torch

from fully_sharded_shard_b200 import workloads as W

pytestmark = pytest.mark.gpu

ALL_OPS = [W.SUM, W.AVG, W.SUM_THEN_DIV]
SHAPES = [(6, 7), (11,), (5, 4), (4, 3), (1000, 3), (7,)]

MASTER_P0 = [0x7FC00000, 0xFFC00001, 0x7F800001, 0x7F800000, 0xFF800000, 0x00000000,
             0x80000000, 0x7F7FFFFF, 0xFF7FFFFF, 0x7F7F7FFF, 0x7F7F8000, 0x7F7E8000,
             0x00000001, 0x00008000, 0x00018000, 0x00017FFF, 0x007FFFFF, 0x80008001,
             0x00800000, 0x3F808000, 0x3F818000, 0x3F807FFF, 0x3F808001, 0xBF818000,
             0x3F800000]
NAN32 = float(np.uint32(0x7FC00000).view(np.float32))
MASTER_P1 = [0.5, -0.75, NAN32, 0.25, 1.5, -1.25, 0.1, -NAN32, 0.0, -0.0, 1e-3]
MASTER_P2 = [448.0, 1.0625, 1.1875, 2 ** -10, 3 * 2 ** -10, -1.0625, -2 ** -10, 0.0, -0.0,
             232.0, 240.0, 248.0, 2 ** -7, 2 ** -6, 2 ** -6 - 2 ** -10, 1e-3, -447.0, 300.0,
             1.0, -448.0]
AMAX_P3 = 0.1024751216173172      # 448 / amax, times amax, rounds above 448 in binary32
MASTER_P3 = [AMAX_P3, -AMAX_P3, 0.1, 0.05, -0.0125, 0.001]

# bf16 bit patterns
B_2P24, B_M2P24, B_ONE, B_MZERO, B_PZERO = 0x4B80, 0xCB80, 0x3F80, 0x8000, 0x0000
B_INF, B_MINF, B_NAN, B_MAX, B_MMAX = 0x7F80, 0xFF80, 0x7FC1, 0x7F7F, 0xFF7F
B_SUB, B_MSUB, B_1E25, B_M1E25, B_1E20, B_3E19 = 0x0001, 0x8001, 0x6904, 0xE904, 0x60AD, 0x5FD0
# (ranks 0, 1, 2 ...), value of the ranks beyond the list
FOLD = [
    ((B_2P24, B_ONE, B_M2P24), B_PZERO),     # (2^24 + 1) - 2^24 = 0 in binary32
    ((B_2P24, B_M2P24, B_ONE), B_PZERO),     # 0 + 1 = 1
    ((B_ONE, B_2P24, B_M2P24), B_PZERO),     # (1 + 2^24) - 2^24 = 0
    ((B_MZERO, B_MZERO, B_MZERO), B_MZERO),  # -0 throughout
    ((B_MZERO, B_PZERO, B_MZERO), B_MZERO),  # +0 once makes it +0
    ((B_INF, B_MINF, B_ONE), B_PZERO),       # NaN
    ((B_INF, B_ONE, B_ONE), B_ONE),          # +Inf
    ((B_NAN, B_ONE, B_ONE), B_PZERO),        # NaN from a NaN input
    ((B_ONE, B_NAN, B_MINF), B_PZERO),
    ((B_MAX, B_MAX, B_MMAX), B_PZERO),       # overflow, then +Inf stays
    ((B_MAX, B_MMAX, B_MAX), B_PZERO),       # the largest finite bf16 again
    ((B_SUB, B_SUB, B_MSUB), B_PZERO),       # bf16 subnormals, exact in binary32
    ((B_1E25, B_PZERO, B_PZERO), B_PZERO),   # AdamW: (1 - b2) g^2 overflows binary32
    ((B_M1E25, B_1E20, B_PZERO), B_PZERO),
    ((B_3E19, B_3E19, B_PZERO), B_PZERO),    # large, g^2 still finite
]


def _u16_of(x: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.bfloat16) \
        .view(torch.int16).numpy().view(np.uint16)


# The edge group followed by 800 small parameters: at least 2048 short and
# pad runs at every N here, so the copy-out, the fused reduce-scatter and the
# fused update take the flat path (fixed tiles, one code per 8 elements).
FLAT_SHAPES = SHAPES + [(3 + k % 23, 1 + k % 5) for k in range(800)]


def _layout(N, shapes=SHAPES):
    import oracle
    return oracle.plan(shapes, N)


def full_init(N: int, shapes=SHAPES) -> np.ndarray:
    """The full fp32 parameters in the arena layout: seeded N(0, 0.02), the
    listed values at the head of each parameter."""
    p = _layout(N, shapes)
    rng = np.random.default_rng(11)
    full = (rng.standard_normal(p.P_arena) * 0.02).astype(np.float32)
    u = [int(x) for x in p.arena_off]
    full[u[0]:u[0] + len(MASTER_P0)] = np.array(MASTER_P0, np.uint32).view(np.float32)
    full[u[1]:u[1] + len(MASTER_P1)] = np.array(MASTER_P1, np.float32)
    full[u[2]:u[2] + len(MASTER_P2)] = np.array(MASTER_P2, np.float32)
    p3 = rng.uniform(-0.09, 0.09, 12).astype(np.float32)
    p3[:len(MASTER_P3)] = np.array(MASTER_P3, np.float32)
    full[u[3]:u[3] + 12] = p3
    return full


def grads_init(N: int, shapes=SHAPES):
    """step -> bf16 bit patterns [N][P_arena]: seeded N(0, 1e-3), the fold
    cases at the heads of p0 and p4, and a negative gradient on the amax
    elements of p2 and p3."""
    p = _layout(N, shapes)
    u = [int(x) for x in p.arena_off]

    def make(step: int) -> np.ndarray:
        rng = np.random.default_rng(1000 + step)
        g = _u16_of(rng.standard_normal((N, p.P_arena)) * 1e-3).reshape(N, p.P_arena)
        for base in (u[0], u[4]):
            for k, (head, rest) in enumerate(FOLD):
                for r in range(N):
                    g[r, base + k] = head[r] if r < len(head) else rest
        g[:, u[2]] = _u16_of(np.full(N, -1.0))      # 448 grows past 448
        g[:, u[3]] = _u16_of(np.full(N, -1.0))      # the amax of p3 too
        return g
    return make


def _wl(N, op, shapes=SHAPES):
    g = W.Group("edge", list(shapes), [f"p{i}" for i in range(len(shapes))])
    return W.Workload(f"edge_n{N}", N, [g], op, 0, "normal", 0.02, 1e-3, steps=2)


@pytest.fixture(scope="module")
def H():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from tests import _harness
    return _harness


NS = [3, 8, 12]


def test_edge_inputs_hold_what_they_claim():
    """The inputs really contain the cases (checked on the host)."""
    full = full_init(3)
    assert np.isnan(full).sum() >= 4 and np.isinf(full).sum() >= 2
    assert np.array_equal(_u16_of(np.array([1e25, -1e25, 1e20, 3e19])),
                          [B_1E25, B_M1E25, B_1E20, B_3E19])
    amax = np.float32(AMAX_P3)
    assert amax * (np.float32(448.0) / amax) > np.float32(448.0)


@pytest.mark.parametrize("N", NS)
def test_edge_values_through_the_five_stages(H, N):
    wl = _wl(N, W.AVG)
    H.run_group(wl, wl.groups[0], steps=2, ops=ALL_OPS, staged=True,
                full_init=full_init(N), grads_init=grads_init(N))


@pytest.mark.parametrize("N", NS)
def test_edge_values_through_the_flat_path(H, N):
    """The same values in a group of many small parameters: the flat
    copy-out, fused reduce-scatter (all ops) and fused update."""
    from fully_sharded_shard_b200 import abi
    g = abi.fsdp_plan_group(FLAT_SHAPES, N)
    flat, flat_copy_out, mixed_shard, mixed_arena = abi.fsdp_group_flat(g)
    g.destroy()
    assert flat and flat_copy_out and mixed_shard > 0 and mixed_arena > 0
    fi, gi = full_init(N, FLAT_SHAPES), grads_init(N, FLAT_SHAPES)
    wl = _wl(N, W.AVG, FLAT_SHAPES)
    H.run_group(wl, wl.groups[0], steps=2, ops=ALL_OPS, staged=False, full_init=fi,
                grads_init=gi)
    for op in ALL_OPS:
        wl = _wl(N, op, FLAT_SHAPES)
        H.run_group_fused(wl, wl.groups[0], steps=2, full_init=fi, grads_init=gi)


@pytest.mark.parametrize("N", NS)
@pytest.mark.parametrize("op", ALL_OPS, ids=["sum", "avg", "sum_then_div"])
def test_edge_values_through_the_fused_update(H, N, op):
    wl = _wl(N, op)
    H.run_group_fused(wl, wl.groups[0], steps=2, full_init=full_init(N),
                      grads_init=grads_init(N))


@pytest.mark.parametrize("N", NS)
def test_edge_values_through_the_fused_fp8_update(H, N):
    wl = _wl(N, W.AVG)
    rep = H.run_group_fused_fp8(wl, wl.groups[0], steps=2, full_init=full_init(N),
                                grads_init=grads_init(N))
    assert rep["saturated"] > 0, "no quantiser input went past 448 under the delayed scale"


@pytest.mark.parametrize("N", NS)
def test_edge_values_fp8_all_gather(H, N):
    wl = _wl(N, W.AVG)
    H.run_group_fp8(wl, wl.groups[0], full_init=full_init(N))


@pytest.mark.parametrize("N", NS)
def test_edge_values_gradient_accumulation(H, N):
    wl = _wl(N, W.SUM_THEN_DIV)
    for op in ALL_OPS:
        H.run_group_accumulate(wl, wl.groups[0], micro=3, op=op, grads_init=grads_init(N))


@pytest.mark.parametrize("N", [3, 8])
def test_edge_values_single_launch_group_step(H, N):
    """The whole step in one call (a single launch when the group is small)."""
    from tests.test_gpu_parity import _group_step_case
    shapes = SHAPES[:4] + [(40, 3)]                 # small enough for one CTA
    g = W.Group("edge_small", shapes, [f"p{i}" for i in range(len(shapes))])
    wl = W.Workload(f"edge_small_n{N}", N, [g], W.AVG, 0, "normal", 0.02, 1e-3, steps=2)
    import oracle
    p = oracle.plan(shapes, N)
    big = full_init(N)
    pb = _layout(N)
    full = np.zeros(p.P_arena, np.float32)
    for i in range(len(shapes)):
        n = shapes[i][0] * (shapes[i][1] if len(shapes[i]) > 1 else 1)
        full[int(p.arena_off[i]):int(p.arena_off[i]) + n] = \
            big[int(pb.arena_off[i]):int(pb.arena_off[i]) + n]
    mk = grads_init(N)

    def gi(step):
        gb = mk(step)
        out = np.zeros((N, p.P_arena), np.uint16)
        for i in range(len(shapes)):
            n = shapes[i][0] * (shapes[i][1] if len(shapes[i]) > 1 else 1)
            out[:, int(p.arena_off[i]):int(p.arena_off[i]) + n] = \
                gb[:, int(pb.arena_off[i]):int(pb.arena_off[i]) + n]
        return out
    _group_step_case(H, wl, g, steps=2, graph=False, full_init=full, grads_init=gi)


@pytest.mark.parametrize("N,D", [(3, 3), (8, 2), (12, 4)])
def test_edge_values_through_the_peer_pulls(H, N, D):
    """The several-device pulls (copy-out, reduce-scatter, fused update) on
    the special values, against the single-device path and the oracle."""
    from tests.test_gpu_peer import run_group_peer
    wl = _wl(N, W.AVG)
    run_group_peer(H, wl, wl.groups[0], D, steps=2, full_init=full_init(N),
                   grads_init=grads_init(N))
