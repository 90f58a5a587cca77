"""GPU parity: the C-ABI kernels against the CPU oracle on seeded inputs.

Bit-exact for the Shard(0) placement, copy-in, copy-out, packing and the
rank-ordered reduction; max |gpu - oracle| <= 1e-6 * (1 + |x|) for AdamW on
parameters and both moments.  Every buffer carries guard bands that must
survive each call.

Small cases span several units and tiles with ragged heads and tails and
misaligned segments; the full-size cases are the five workloads at their
real shapes, in the same launch configuration the benchmark times (the 7B
model's 32 block groups share one plan, so one block group plus the root
group covers every launch it makes).
"""
import numpy as np
import pytest
import torch

from fully_sharded_shard_b200 import workloads as W

pytestmark = pytest.mark.gpu

ALL_OPS = [W.SUM, W.AVG, W.SUM_THEN_DIV]


@pytest.fixture(scope="module")
def H():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from tests import _harness
    return _harness


def _wl(name, shapes, N, op=W.AVG, steps=2, dist="normal", scale=0.02, sigma=1e-3, zero=()):
    g = W.Group(name, [tuple(s) for s in shapes], [f"p{i}" for i in range(len(shapes))],
                zero_grad=list(zero))
    return W.Workload(name, N, [g], op, 0, dist, scale, sigma, steps=steps)


SMALL = [
    _wl("ragged_n4", [(7, 3), (5,), (1, 32), (1,), (0, 4), (13, 9), (2, 2)], 4),
    _wl("one_rank", [(5, 3), (4,), (1000, 7)], 1),
    _wl("n3_odd", [(1001, 3), (17,), (3, 4099), (8191, 1)], 3),
    _wl("n9_generic", [(3, 5), (9,), (17, 2), (4000, 13), (123, 77)], 9),
    _wl("n12_generic", [(37, 100), (6,), (1999, 31)], 12),
    _wl("n2_shift", [(3,), (9001, 5), (7, 1), (16385,)], 2, zero=[1]),
    _wl("n8_tiny_rows", [(3, 1), (1, 1), (7, 8), (5, 3)], 8),
    _wl("empty_params", [(0, 5), (0,)], 4),
    _wl("no_params", [], 3),
]


@pytest.mark.parametrize("wl", SMALL, ids=[w.name for w in SMALL])
def test_small_groups_all_ops_two_steps(H, wl):
    H.run_group(wl, wl.groups[0], steps=2, ops=ALL_OPS, staged=True)


def test_tiny_mlp_three_steps(H):
    wl = W.tiny_mlp()
    rep = H.run_group(wl, wl.groups[0], steps=wl.steps, ops=ALL_OPS, staged=True)
    assert rep["S"] == 338


SCALED = [W.llama_block(16), W.uneven(8), W.moe(8), W.llama7b(16, layers=1)]


@pytest.mark.parametrize("wl", SCALED, ids=[w.name for w in SCALED])
def test_scaled_workloads(H, wl):
    for g in wl.groups:
        H.run_group(wl, g, steps=2, ops=ALL_OPS, staged=True)


def test_toy_llm_block_and_root(H):
    """The DTensor guide's demo transformer at N = 8 (SwiGLU rows 1364 and
    256 x 682: the gate/up projection pads its last rank): every stage and
    op, the fused update and the FP8 all-gather, for the block and the root
    group."""
    wl = W.toy_llm()
    for g in wl.groups:
        H.run_group(wl, g, steps=2, ops=ALL_OPS, staged=True)
        H.run_group_fused(wl, g, steps=2)
        H.run_group_fp8(wl, g)


FULL = [W.tiny_mlp(), W.llama_block(), W.uneven(), W.moe()]


@pytest.mark.parametrize("wl", FULL, ids=[w.name for w in FULL])
def test_full_size_workloads(H, wl):
    for g in wl.groups:
        H.run_group(wl, g, steps=1, ops=[wl.op], staged=False, direct_oracle=True)


def test_full_size_llama7b_block_and_root(H):
    wl = W.llama7b()
    for g in wl.groups:
        H.run_group(wl, g, steps=1, ops=[wl.op], staged=False, direct_oracle=True)


FUSED = [
    _wl("fused_ragged_n4", [(7, 3), (5,), (1, 32), (1,), (0, 4), (13, 9), (2, 2)], 4, op=W.SUM),
    _wl("fused_n3_odd", [(1001, 3), (17,), (3, 4099), (8191, 1)], 3, op=W.SUM_THEN_DIV),
    _wl("fused_n12", [(37, 100), (6,), (1999, 31)], 12),
    _wl("fused_n2_shift", [(3,), (9001, 5), (7, 1), (16385,)], 2, zero=[1]),
]


@pytest.mark.parametrize("wl", FUSED + [W.tiny_mlp(), W.uneven(8), W.moe(8)],
                         ids=[w.name for w in FUSED] + ["tiny_mlp", "uneven_div8", "moe_div8"])
def test_fused_rs_adamw_copy_in(H, wl):
    for g in wl.groups:
        H.run_group_fused(wl, g, steps=3)


def test_fused_full_size_llama7b_block(H):
    wl = W.llama7b()
    H.run_group_fused(wl, wl.groups[0], steps=1, direct_oracle=True)


@pytest.mark.parametrize("wl", FUSED + [W.tiny_mlp(), W.uneven(8), W.moe(8)],
                         ids=[w.name for w in FUSED] + ["tiny_mlp", "uneven_div8", "moe_div8"])
def test_fused_rs_adamw_fp8_delayed_scaling(H, wl):
    for g in wl.groups:
        H.run_group_fused_fp8(wl, g, steps=3)


def test_fused_fp8_full_size_llama7b_block(H):
    wl = W.llama7b()
    H.run_group_fused_fp8(wl, wl.groups[0], steps=1)


ACCUM = SMALL[:4] + [W.tiny_mlp(), W.uneven(8), W.moe(16), W.llama7b(16, layers=1)]


@pytest.mark.parametrize("wl", ACCUM, ids=[w.name for w in ACCUM])
def test_gradient_accumulation_without_sync(H, wl):
    for g in wl.groups:
        for op in ALL_OPS:
            H.run_group_accumulate(wl, g, micro=3, op=op)


def test_gradient_accumulation_two_microbatches(H):
    wl = W.uneven(16)
    H.run_group_accumulate(wl, wl.groups[0], micro=2)


FP8 = SMALL + [W.tiny_mlp(), W.uneven(8), W.moe(8), W.llama7b(8, layers=1)]


@pytest.mark.parametrize("wl", FP8, ids=[w.name for w in FP8])
def test_fp8_all_gather_copy_in_and_out(H, wl):
    for g in wl.groups:
        H.run_group_fp8(wl, g)


def test_fp8_full_size_llama7b_root(H):
    wl = W.llama7b()
    H.run_group_fp8(wl, wl.groups[1])


def test_fused_and_staged_reduce_are_deterministic(H):
    from fully_sharded_shard_b200 import abi
    wl = W.uneven(8)
    grp = wl.groups[0]
    g = abi.fsdp_plan_group(grp.shapes, wl.N)
    grads = H.make_grads(g, wl, grp, 1)
    outs = []
    for packed in (None, torch.empty(wl.N * wl.N * g.S, device="cuda")):
        for _ in range(2):
            red = torch.empty(wl.N * g.S, device="cuda")
            abi.fsdp_rs_reduce(g, grads, W.SUM_THEN_DIV, red, packed=packed)
            outs.append(red)
    torch.cuda.synchronize()
    for o in outs[1:]:
        assert torch.equal(o.view(torch.int32), outs[0].view(torch.int32))


def test_host_validation_rejects_before_launch(H):
    from fully_sharded_shard_b200 import abi
    g = abi.fsdp_plan_group([(33, 5), (7,)], 4)
    NS = g.N * g.S
    buf = torch.zeros(NS + 8, device="cuda")
    ag = torch.zeros(NS + 16, dtype=torch.bfloat16, device="cuda")
    L = abi.lib()
    import ctypes
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    p = lambda t, off=0: ctypes.c_void_p(t.data_ptr() + off)
    # misaligned pointers
    assert L.fsdp_copy_in(g.handle, p(buf, 4), p(ag), s) == abi.FSDP_EALIGN
    assert L.fsdp_copy_out(g.handle, p(ag, 2), p(ag), s) == abi.FSDP_EALIGN
    # null pointers, bad op, bad hyper-parameters
    assert L.fsdp_copy_in(g.handle, None, p(ag), s) == abi.FSDP_EINVAL
    assert L.fsdp_rs_reduce(g.handle, p(ag), 7, None, p(buf), s) == abi.FSDP_EINVAL
    hp = abi.AdamWHparams(1e-3, 0.9, 0.999, 1e-8, 0.0, 0)   # step 0
    assert L.fsdp_adamw_step(g.handle, p(buf), p(buf), p(buf), p(buf), ctypes.byref(hp), s) == abi.FSDP_EINVAL
    hp = abi.AdamWHparams(1e-3, 1.0, 0.999, 1e-8, 0.0, 1)   # beta1 == 1
    assert L.fsdp_adamw_step(g.handle, p(buf), p(buf), p(buf), p(buf), ctypes.byref(hp), s) == abi.FSDP_EINVAL
    grads = torch.zeros(g.N * g.P_arena, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(abi.FsdpError):
        abi.fsdp_rs_reduce(g, grads, 5, buf)
    with pytest.raises(ValueError):
        abi.fsdp_rs_reduce(g, grads[:5], W.AVG, buf)      # too small: caught in the binding
    torch.cuda.synchronize()
    assert torch.count_nonzero(buf) == 0 and torch.count_nonzero(ag.view(torch.int16)) == 0


@pytest.mark.parametrize("fused", [False, True], ids=["stages", "fused"])
def test_graph_replayed_steps_equal_eager_steps(H, fused):
    """A captured CUDA graph of one step (device step counter + AdamW scalars),
    replayed 3 times, gives the same state as 3 eager steps with host step
    counts, and stays within the AdamW tolerance of the oracle."""
    import numpy as np
    import oracle
    from fully_sharded_shard_b200 import abi
    wl = W.uneven(8)
    grp = wl.groups[0]
    g = abi.fsdp_plan_group(grp.shapes, wl.N)
    p = oracle.plan(grp.shapes, wl.N)
    NS = wl.N * g.S
    full = torch.empty(g.P_arena, device="cuda")
    W.fill_master(full, wl, grp.name)
    grads = H.make_grads(g, wl, grp, 1)
    hp = dict(W.ADAMW_DEFAULTS)
    states = []
    for _ in range(2):
        master = torch.empty(NS, device="cuda")
        abi.fsdp_shard_params(g, full, master)
        states.append((master, torch.zeros(NS, device="cuda"), torch.zeros(NS, device="cuda"),
                       torch.empty(NS, device="cuda"), torch.empty(NS, dtype=torch.bfloat16, device="cuda")))
    (pa, ma, va, ra, aga), (pb, mb, vb, rb, agb) = states
    for step in (1, 2, 3):                                  # eager, host step counts
        if fused:
            abi.fsdp_rs_adamw_step(g, grads, wl.op, pa, ma, va, step=step, ag_next=aga, **hp)
        else:
            abi.fsdp_rs_reduce(g, grads, wl.op, ra)
            abi.fsdp_adamw_step(g, pa, ma, va, ra, step=step, **hp)
    ds = abi.DeviceStep()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        abi.fsdp_adamw_prepare(ds, **hp)
        if fused:
            abi.fsdp_rs_adamw_step_dev(g, grads, wl.op, pb, mb, vb, ds, ag_next=agb)
        else:
            abi.fsdp_rs_reduce(g, grads, wl.op, rb)
            abi.fsdp_adamw_step_dev(g, pb, mb, vb, rb, ds)
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    assert int(ds.step.item()) == 3
    for a, b in ((pa, pb), (ma, mb), (va, vb)):
        assert torch.equal(a.view(torch.int32), b.view(torch.int32))
    if fused:
        assert torch.equal(aga.view(torch.int16), agb.view(torch.int16))
    # the oracle, three steps on the same reduced gradient
    red_o = oracle.reduce_scatter_direct(p, H.u16(grads), wl.op)
    mo = oracle.shard(p, H.f32(full))
    m_o, v_o = np.zeros_like(mo), np.zeros_like(mo)
    for step in (1, 2, 3):
        oracle.adamw(mo, m_o, v_o, red_o, step=step, **hp)
    for gbuf, obuf in ((pb, mo), (mb, m_o), (vb, v_o)):
        ok, ratio = H.adam_close(H.f32(gbuf), obuf)
        assert ok, ratio
    del graph
    g.destroy()


def test_bench_two_stream_schedules_match_one_stream(H):
    """bench.py's two-stream schedules (all-gather half on one stream, the
    update half on another) leave exactly the state of the one-stream
    schedules: the event dependencies order every buffer reuse."""
    import bench
    wl = W.llama7b(16, layers=3)
    dev = torch.device("cuda", 0)
    a = bench.Model(wl, dev, 2, 0)
    b = bench.Model(wl, dev, 2, 0)
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    for _ in range(3):
        a.step(s1)
        b.step_two_streams(s1, s2)
    torch.cuda.synchronize()
    for (_, pa, ma, va, _), (_, pb, mb, vb, _) in zip(a.instances, b.instances):
        for x, y in ((pa, pb), (ma, mb), (va, vb)):
            assert torch.equal(x.view(torch.int32), y.view(torch.int32))
    a.enable_fused()
    b.enable_fused()
    for _ in range(3):
        a.fused_step(s1)
        b.fused_step_two_streams(s1, s2)
    torch.cuda.synchronize()
    for (_, pa, ma, va, _), (_, pb, mb, vb, _) in zip(a.instances, b.instances):
        for x, y in ((pa, pb), (ma, mb), (va, vb)):
            assert torch.equal(x.view(torch.int32), y.view(torch.int32))
    for x, y in zip(a.ag_groups, b.ag_groups):
        assert torch.equal(x.view(torch.int16), y.view(torch.int16))


EDGE = [
    _wl("max_world_1024", [(2000, 3), (5,), (1030, 1)], 1024, op=W.SUM_THEN_DIV),
    _wl("conv_like_4d", [(64, 3, 7, 7), (64,), (128, 64, 3, 3), (10, 2, 3, 1, 5)], 6),
    _wl("scalars_0d", [(), (3,), (), (17, 4)], 3),
    _wl("rows_on_rank0_only", [(1, 4096), (2, 513), (1,)], 8),
]


@pytest.mark.parametrize("wl", EDGE, ids=[w.name for w in EDGE])
def test_edge_shapes_and_world_sizes(H, wl):
    H.run_group(wl, wl.groups[0], steps=2, ops=ALL_OPS, staged=wl.N <= 64)
    H.run_group_fused(wl, wl.groups[0], steps=2)
    H.run_group_fp8(wl, wl.groups[0])
    H.run_group_fused_fp8(wl, wl.groups[0], steps=2)


def _random_group(rng, k):
    N = int(rng.integers(1, 17))
    shapes = []
    for _ in range(int(rng.integers(1, 7))):
        nd = int(rng.integers(0, 5))
        dims = [int(rng.integers(0, 40)) if rng.random() < 0.1 else int(rng.integers(1, 300))]
        dims += [int(rng.integers(1, 9)) for _ in range(max(nd - 1, 0))]
        shapes.append(tuple(dims[:nd]) if nd > 0 else ())
    return _wl(f"rand{k}", shapes, N, op=[W.SUM, W.AVG, W.SUM_THEN_DIV][k % 3])


RANDOM = [_random_group(np.random.default_rng(1000 + k), k) for k in range(40)]


@pytest.mark.parametrize("wl", RANDOM, ids=[w.name for w in RANDOM])
def test_random_groups_brute_force(H, wl):
    grp = wl.groups[0]
    H.run_group(wl, grp, steps=2, ops=ALL_OPS, staged=True)
    H.run_group_fused(wl, grp, steps=1)
    H.run_group_fp8(wl, grp)
    H.run_group_fused_fp8(wl, grp, steps=1)


def test_many_small_parameters_packed_paths(H):
    """3000 small parameters over 8 ranks: the copy-outs, the fused
    reduce-scatter and the fused update pack their short units (a warp each)
    -- every stage, the staged pack, the fused update (bf16 and FP8 next
    all-gather input) and the FP8 all-gather against the oracle."""
    from fully_sharded_shard_b200 import abi
    wl = W.small_params()
    grp = wl.groups[0]
    g = abi.fsdp_plan_group(grp.shapes, wl.N)
    assert abi.fsdp_group_check(g) == 0
    g.destroy()
    H.run_group(wl, grp, steps=2, ops=ALL_OPS, staged=True)
    H.run_group_fused(wl, grp, steps=2)
    H.run_group_fused_fp8(wl, grp, steps=2)
    H.run_group_fp8(wl, grp)


def _small(count, seed):
    return W.small_params(count=count, seed=seed).groups[0].shapes


# Groups of many small parameters, which take the flat path: N = 1 (no pads),
# an odd [N][S] (a partial last vector), long runs beside the small ones, and
# the any-N kernels (N = 11).
FLAT = [
    _wl("flat_n1", _small(4000, 15), 1, op=W.SUM),
    _wl("flat_n3", _small(1000, 11), 3, op=W.SUM),
    _wl("flat_n5_long", _small(700, 12) + [(30001, 64), (4097,), (0, 5), (1, 1)], 5),
    _wl("flat_n8", _small(600, 13), 8, op=W.SUM_THEN_DIV),
    _wl("flat_n11", _small(400, 14), 11),
]


@pytest.mark.parametrize("wl", FLAT, ids=[w.name for w in FLAT])
def test_many_small_parameters_flat_path(H, wl):
    """The flat copy-out (but at N = 1), fused reduce-scatter (every op) and
    fused update against the oracle; the FP8 paths of the same group keep the
    packs."""
    from fully_sharded_shard_b200 import abi
    grp = wl.groups[0]
    g = abi.fsdp_plan_group(grp.shapes, wl.N)
    flat, flat_copy_out, mixed_shard, mixed_arena = abi.fsdp_group_flat(g)
    assert abi.fsdp_group_check(g) == 0
    g.destroy()
    assert flat and mixed_shard > 0
    # at N = 1 every run is a whole parameter: too few elements in short runs
    # for the flat copy-out, which then takes the per-run kernel
    assert flat_copy_out == (wl.N > 1) and (mixed_arena > 0) == flat_copy_out
    if wl.name == "flat_n3":
        assert (wl.N * g.S) % 8 != 0, "the partial last vector"
    H.run_group(wl, grp, steps=2, ops=ALL_OPS, staged=False)
    H.run_group_fused(wl, grp, steps=2)
    H.run_group_fused_fp8(wl, grp, steps=1)


GRID = [_wl(f"grid_n{N}", [((d0, c) if c > 1 else (d0,)) for d0 in range(21) for c in (1, 3, 8)], N,
            op=[W.SUM, W.AVG, W.SUM_THEN_DIV][N % 3]) for N in range(1, 10)]


@pytest.mark.parametrize("wl", GRID, ids=[w.name for w in GRID])
def test_brute_force_grid_d0_cols_world(H, wl):
    """Every d0 in [0, 20] x cols in {1, 3, 8} as one 63-parameter group, for
    every N in [1, 9]: all stages, all ops, the fused, FP8 and fused FP8 paths."""
    grp = wl.groups[0]
    H.run_group(wl, grp, steps=2, ops=ALL_OPS, staged=True)
    H.run_group_fused(wl, grp, steps=1)
    H.run_group_fp8(wl, grp)
    H.run_group_fused_fp8(wl, grp, steps=1)


def test_checkpoint_resume_is_bit_exact(H, tmp_path):
    """Two steps, save, restore into fresh buffers, one more step: the same
    bits as three uninterrupted steps."""
    from fully_sharded_shard_b200 import abi, checkpoint as C
    wl = W.uneven(16)
    grp = wl.groups[0]
    g = abi.fsdp_plan_group(grp.shapes, wl.N)
    NS = wl.N * g.S
    full = torch.empty(g.P_arena, device="cuda")
    W.fill_master(full, wl, grp.name)
    hp = dict(W.ADAMW_DEFAULTS)
    grads = [H.make_grads(g, wl, grp, s) for s in (1, 2, 3)]
    red = torch.empty(NS, device="cuda")

    def fresh():
        p = torch.empty(NS, device="cuda")
        abi.fsdp_shard_params(g, full, p)
        return p, torch.zeros(NS, device="cuda"), torch.zeros(NS, device="cuda")

    def step(state, t):
        abi.fsdp_rs_reduce(g, grads[t - 1], wl.op, red)
        abi.fsdp_adamw_step(g, *state, red, step=t, **hp)

    a = fresh()
    for t in (1, 2, 3):
        step(a, t)
    b = fresh()
    for t in (1, 2):
        step(b, t)
    torch.cuda.synchronize()
    C.save_group_state(str(tmp_path), grp.shapes, wl.N, g.S, 2, *b)
    c = (torch.empty(NS, device="cuda"), torch.empty(NS, device="cuda"), torch.empty(NS, device="cuda"))
    t0 = C.load_group_state(str(tmp_path), grp.shapes, wl.N, g.S, *c)
    step(c, t0 + 1)
    torch.cuda.synchronize()
    for x, y in zip(a, c):
        assert torch.equal(x.view(torch.int32), y.view(torch.int32))
    g.destroy()


def _group_step_case(H, wl, grp, steps, graph, full_init=None, grads_init=None):
    """fsdp_group_step (eager, or its _dev form replayed from a CUDA graph)
    against the four stage calls on a copy of the same state, bit for bit
    (NaN as a class), and against the oracle applied to the step's own
    inputs: copy-in of the pre-step master, copy-out of that all-gather
    buffer, the reduce-scatter, and AdamW from the pre-step state."""
    import oracle
    from fully_sharded_shard_b200 import abi
    N, op = wl.N, wl.op
    g = abi.fsdp_plan_group(grp.shapes, N)
    p = oracle.plan(grp.shapes, N)
    NS, A = N * g.S, g.P_arena
    full = torch.empty(max(A, 1), device="cuda")
    if full_init is None:
        W.fill_master(full, wl, grp.name)
    else:
        full.zero_()
        full[:A].copy_(torch.from_numpy(np.ascontiguousarray(full_init, np.float32)))
    hp = dict(W.ADAMW_DEFAULTS)

    def state():
        master = torch.empty(max(NS, 1), device="cuda")
        abi.fsdp_shard_params(g, full, master)
        return {"p": master, "m": torch.zeros(max(NS, 1), device="cuda"),
                "v": torch.zeros(max(NS, 1), device="cuda"),
                "ag": torch.empty(max(NS, 1), dtype=torch.bfloat16, device="cuda"),
                "arena": torch.full((max(A, 1),), 0x3BEF, dtype=torch.int16,
                                    device="cuda").view(torch.bfloat16),
                "red": torch.empty(max(NS, 1), device="cuda")}
    a, b = state(), state()
    grads = [H._grads_for(g, wl, grp, t, (), grads_init) for t in range(1, steps + 1)]
    gbuf = torch.empty_like(grads[0])
    if graph:
        ds = abi.DeviceStep()
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        cg = torch.cuda.CUDAGraph()
        with torch.cuda.graph(cg, stream=s):
            if graph == "one_call":   # counter, scalars and step in one call
                abi.fsdp_group_step_graph(g, a["p"], a["m"], a["v"], gbuf, op, ds, ag=a["ag"],
                                          arena=a["arena"], reduced=a["red"], **hp)
            else:
                abi.fsdp_adamw_prepare(ds, **hp)
                abi.fsdp_group_step_dev(g, a["p"], a["m"], a["v"], gbuf, op, ds, ag=a["ag"],
                                        arena=a["arena"], reduced=a["red"])
    for t in range(1, steps + 1):
        torch.cuda.synchronize()
        pre = tuple(H.f32(a[k][:NS]) for k in ("p", "m", "v"))
        if graph:
            gbuf.copy_(grads[t - 1])
            cg.replay()
        else:
            abi.fsdp_group_step(g, a["p"], a["m"], a["v"], grads[t - 1], op, step=t, ag=a["ag"],
                                arena=a["arena"], reduced=a["red"], **hp)
        abi.fsdp_copy_in(g, b["p"], b["ag"])
        abi.fsdp_copy_out(g, b["ag"], b["arena"])
        abi.fsdp_rs_reduce(g, grads[t - 1], op, b["red"])
        abi.fsdp_adamw_step(g, b["p"], b["m"], b["v"], b["red"], step=t, **hp)
        torch.cuda.synchronize()
        for k in ("p", "m", "v", "red"):
            assert H.equal_nan_class(H.f32(a[k]), H.f32(b[k]), "f32"), f"{k} step {t}"
        for k in ("ag", "arena"):
            assert H.equal_nan_class(H.u16(a[k]), H.u16(b[k]), "bf16"), f"{k} step {t}"
        ag_h = H.u16(a["ag"][:NS])
        assert H.equal_nan_class(ag_h, oracle.copy_in(p, pre[0]), "bf16"), f"copy-in step {t}"
        arena_o = oracle.copy_out(p, ag_h, np.full(A, 0x3BEF, np.uint16))
        assert H.bits_equal(H.u16(a["arena"][:A]), arena_o), f"copy-out step {t}"
        red_o = oracle.reduce_scatter(p, H.u16(grads[t - 1]), op)
        red_h = H.f32(a["red"][:NS])
        assert H.equal_nan_class(red_h, red_o, "f32"), f"reduce-scatter step {t}"
        want = H.adamw_from_state(*pre, red_h, t, hp)
        for k, w in zip(("p", "m", "v"), want):
            ok, ratio = H.adam_close_special(H.f32(a[k][:NS]), w)
            assert ok, f"adamw {k} step {t}: {ratio}"
    if graph:
        assert int(ds.step.item()) == steps
        del cg
    g.destroy()


# + two groups of many small parameters (the flat kernels inside the one call)
GROUP_STEP = SMALL + [W.tiny_mlp(), W.uneven(64), W.moe(64), FLAT[1], FLAT[4]]


@pytest.mark.parametrize("wl", GROUP_STEP, ids=[w.name for w in GROUP_STEP])
def test_group_step_equals_the_four_stage_calls(H, wl):
    from fully_sharded_shard_b200 import abi
    for grp in wl.groups:
        _group_step_case(H, wl, grp, steps=3, graph=False)
    small = [grp for grp in wl.groups
             if wl.N * abi.fsdp_plan_group(grp.shapes, wl.N).S <= abi.FSDP_SMALL_STEP_ELEMS]
    for grp in small[:1]:
        _group_step_case(H, wl, grp, steps=3, graph=True)
        _group_step_case(H, wl, grp, steps=3, graph="one_call")
    big = [grp for grp in wl.groups if grp not in small]
    for grp in big[:1]:   # the prepare kernel and the four stage kernels in one call
        _group_step_case(H, wl, grp, steps=2, graph="one_call")


@pytest.mark.parametrize("wl", GRID[:3], ids=[w.name for w in GRID[:3]])
def test_group_step_single_launch_on_the_brute_force_grid(H, wl):
    _group_step_case(H, wl, wl.groups[0], steps=2, graph=False)


F32 = SMALL + [W.tiny_mlp(), W.uneven(16), W.moe(16)]


@pytest.mark.parametrize("wl", F32, ids=[w.name for w in F32])
def test_fp32_param_dtype_all_gather_is_the_identity(H, wl):
    """param_dtype fp32 (test mode): the copy-in equals the oracle's padded
    shards bit for bit, and the copy-out of it gives back every parameter
    exactly (all-gather(shard(x)) == x), gaps untouched."""
    import numpy as np
    import oracle
    from fully_sharded_shard_b200 import abi
    for grp in wl.groups:
        g = abi.fsdp_plan_group(grp.shapes, wl.N)
        p = oracle.plan(grp.shapes, wl.N)
        NS, A = wl.N * g.S, g.P_arena
        full = torch.empty(max(A, 1), device="cuda")
        W.fill_master(full, wl, grp.name)
        master = torch.empty(max(NS, 1), device="cuda")
        abi.fsdp_shard_params(g, full, master)
        ag32 = H.Guarded(NS, torch.float32)
        abi.fsdp_copy_in_f32(g, master[:NS], ag32.t)
        arena = H.Guarded(A, torch.float32)
        abi.fsdp_copy_out_f32(g, ag32.t, arena.t)
        torch.cuda.synchronize()
        assert ag32.guards_intact() and arena.guards_intact()
        full_h = H.f32(full)[:A]
        shard_o = oracle.shard(p, full_h) if A else np.zeros(0, np.float32)
        assert H.bits_equal(H.f32(ag32.t), shard_o), "fp32 copy-in: " + H.first_mismatch(H.f32(ag32.t), shard_o)
        got = H.f32(arena.t)
        real = np.zeros(A, bool)
        for i in range(g.n):
            real[g.arena_off[i]:g.arena_off[i] + g.numel[i]] = True
        assert np.array_equal(got[real].view(np.uint32), full_h[real].view(np.uint32)), \
            "fp32 all-gather is not the identity"
        assert np.all(got[~real] == np.float32(-12345.5)), "fp32 copy-out wrote a gap"
        g.destroy()
