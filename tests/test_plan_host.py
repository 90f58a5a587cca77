"""The C++ plan builder on the host (no GPU): every layout table against the
oracle's plan, and the library's own consistency check of its work tables
(extents, exact coverage, Shard(0) arena positions, pad intervals, copy-in
tile ranges), over the workloads, random groups and the brute-force grid
d0 in [0, 20] x cols in {1, 3, 8} x N in [1, 9]."""
import ctypes

import numpy as np
import pytest


@pytest.fixture(scope="module")
def abi():
    from fully_sharded_shard_b200 import build
    build.build()
    from fully_sharded_shard_b200 import abi as _abi
    return _abi


def _compare(abi, oracle, shapes, N):
    g = abi.fsdp_plan_group_host(shapes, N)
    p = oracle.plan(shapes, N)
    assert (g.S, g.P, g.P_arena) == (p.S, p.P, p.P_arena)
    assert list(g.shard_off) == [int(x) for x in p.shard_off]
    assert list(g.arena_off) == [int(x) for x in p.arena_off]
    assert list(g.chunk_rows) == [int(x) for x in p.chunk_rows]
    assert abi.fsdp_group_check(g) == 0, (shapes, N)
    g.destroy()


def test_workload_plans_on_host(abi, oracle):
    from fully_sharded_shard_b200 import workloads as W
    for wl in (W.tiny_mlp(), W.llama_block(), W.uneven(), W.moe(), W.llama7b(),
               W.small_params(), W.toy_llm()):
        for grp in wl.groups:
            _compare(abi, oracle, grp.shapes, wl.N)


def test_random_and_extreme_plans_on_host(abi, oracle):
    rng = np.random.default_rng(7)
    for k in range(200):
        N = int(rng.integers(1, 65))
        shapes = []
        for _ in range(int(rng.integers(0, 8))):
            nd = int(rng.integers(0, 4))
            dims = [int(rng.integers(0, 3000))] + [int(rng.integers(1, 9)) for _ in range(max(nd - 1, 0))]
            shapes.append(tuple(dims[:nd]) if nd else ())
        _compare(abi, oracle, shapes, N)
    _compare(abi, oracle, [(5, 3), (1,), (2, 2)], 1024)        # most ranks empty
    _compare(abi, oracle, [(20000, 1)], 3)                     # units split at 8192
    _compare(abi, oracle, [], 4)                               # no parameters


def test_brute_force_grid_plans_on_host(abi, oracle):
    shapes = [((d0, c) if c > 1 else (d0,)) for d0 in range(21) for c in (1, 3, 8)]
    for N in range(1, 10):
        _compare(abi, oracle, shapes, N)


def test_flat_path_for_groups_of_many_small_parameters(abi):
    """The flat tables exist for a group of thousands of small parameters
    (and pass the check), not for the transformer groups."""
    from fully_sharded_shard_b200 import workloads as W
    wl = W.small_params()
    g = abi.fsdp_plan_group_host(wl.groups[0].shapes, wl.N)
    flat, flat_copy_out, mixed_shard, mixed_arena = abi.fsdp_group_flat(g)
    assert flat and flat_copy_out and 0 < mixed_shard < wl.N * g.S // 8 // 20 and 0 < mixed_arena
    assert abi.fsdp_group_check(g) == 0
    g.destroy()
    for wl in (W.llama_block(), W.uneven(), W.moe(), W.tiny_mlp()):
        g = abi.fsdp_plan_group_host(wl.groups[0].shapes, wl.N)
        assert abi.fsdp_group_flat(g) == (False, False, 0, 0)
        g.destroy()


def test_flat_path_thresholds_on_host(abi):
    """The flat path starts at 2048 short and pad runs, and stops where an
    index space exceeds the codes' range (2^30 elements)."""
    for n, want in ((2047, False), (2048, True)):
        g = abi.fsdp_plan_group_host([(1,)] * n, 1)        # one 1-element run each
        flat, flat_copy_out, mixed_shard, mixed_arena = abi.fsdp_group_flat(g)
        assert (flat, flat_copy_out) == (want, want)
        if want:   # every vector holds several runs (shard side) or a run and gaps (arena)
            assert (mixed_shard, mixed_arena) == (n // 8, n)
        assert abi.fsdp_group_check(g) == 0
        g.destroy()
    g = abi.fsdp_plan_group_host([(3,)] * 2100 + [((1 << 30) // 8 + 8, 8)], 1)
    assert g.S > (1 << 30) and abi.fsdp_group_flat(g) == (False, False, 0, 0)
    assert abi.fsdp_group_check(g) == 0
    g.destroy()


def test_random_flat_plans_on_host(abi, oracle):
    """Random groups of thousands of small parameters (with and without a
    large one, N from 1 to 24): the flat tables pass the check and the layout
    matches the oracle's."""
    rng = np.random.default_rng(23)
    seen = set()
    for k in range(24):
        N = int(rng.integers(1, 25))
        count = int(rng.integers(2100 // N + 1, 2600))
        shapes = [(int(rng.integers(0, 200)),) if rng.random() < 0.3 else
                  (int(rng.integers(0, 120)), int(rng.integers(1, 20))) for _ in range(count)]
        if k % 3 == 0:
            shapes.insert(int(rng.integers(0, count)), (int(rng.integers(4000, 16000)), 1000))
        g = abi.fsdp_plan_group_host(shapes, N)
        flat, flat_copy_out, _, _ = abi.fsdp_group_flat(g)
        seen.add((flat, flat_copy_out))
        g.destroy()
        _compare(abi, oracle, shapes, N)
    assert (True, True) in seen and (True, False) in seen


def test_data_calls_refuse_a_host_plan(abi):
    L = abi.lib()
    g = abi.fsdp_plan_group_host([(7, 3), (5,)], 2)
    fake = ctypes.c_void_p(1 << 20)  # aligned and non-null; never dereferenced
    st = L.fsdp_copy_in(g.handle, fake, fake, None)
    assert st in (abi.FSDP_ESTATE, abi.FSDP_ECUDA)
    st = L.fsdp_rs_reduce(g.handle, fake, abi.FSDP_AVG, None, fake, None)
    assert st in (abi.FSDP_ESTATE, abi.FSDP_ECUDA)
    g.destroy()


# Mistakes planted in a copy of the host plan builder (compiled on the CPU,
# never run on a GPU): the consistency check must report each of them.
MUTANTS_PACKS = [
    ("pack one unit over the limit",
     "while (k < e && cnt < fsdpk::kPackUnits &&",
     "while (k < e && cnt <= fsdpk::kPackUnits &&"),
    ("a short unit counted as long",
     "return g->units[k].len >= fsdpk::kShortRun;",
     "return g->units[k].len >= fsdpk::kShortRun / 2;"),
]

MUTANTS_FLAT = [
    ("flat shard code one element off",
     "sruns.push_back({u.shard_pos, u.len, 2 * (u.arena_pos - u.shard_pos)});",
     "sruns.push_back({u.shard_pos, u.len, 2 * (u.arena_pos - u.shard_pos + 1)});"),
    ("flat arena code one element off",
     "aruns.push_back({u.arena_pos, u.len, 2 * (u.shard_pos - u.arena_pos)});",
     "aruns.push_back({u.arena_pos, u.len, 2 * (u.shard_pos - u.arena_pos) + 2});"),
    ("a mixed vector coded pure",
     "if (hi <= end && segs[i + 1].start >= hi) {",
     "if (hi <= end && segs[i + 1].start >= lo + 4) {"),
    ("a mixed vector's elements all given its first code",
     "while (k < end && segs[t + 1].start <= k) ++t;",
     "while (false) ++t;"),
    ("arena gaps not marked",
     "if (r[0] > at) put(at, kFlatPad);",
     "(void)0;"),
    ("flat segments not merged",
     "if (segs.empty() || segs.back().code != code)",
     "if (true)"),
    ("flat path below its threshold",
     "n_small < kFlatMinUnits ||",
     "n_small < kFlatMinUnits / 4 ||"),
    ("flat copy-out below its share of short runs",
     "if (short_elems * kFlatCopyOutShare >= g->P) {",
     "if (short_elems * kFlatCopyOutShare * 100 >= g->P) {"),
]

MUTANTS = [
    ("arena one row off",
     "g->u[i] + j * g->c[i] * g->cols[i], v * g->cols[i], 0);",
     "g->u[i] + (j + 1) * g->c[i] * g->cols[i], v * g->cols[i], 0);"),
    ("pad run one element short",
     "const int64_t len = (g->c[i] - v) * g->cols[i];",
     "const int64_t len = (g->c[i] - v) * g->cols[i] - (v < g->c[i] ? 1 : 0);"),
    ("valid rows not clamped to the chunk",
     "const int64_t v = std::clamp<int64_t>(g->d0[i] - j * g->c[i], 0, g->c[i]);\n                push_units(",
     "const int64_t v = std::max<int64_t>(g->d0[i] - j * g->c[i], 0);\n                push_units("),
    ("adjacent pads not merged",
     "if (!g->intervals.empty() && g->intervals.back().hi == lo)",
     "if (false)"),
    ("tile range one interval short",
     "g->tile_ranges[(size_t)t] = TileRange{(int32_t)a, (int32_t)b};",
     "g->tile_ranges[(size_t)t] = TileRange{(int32_t)a, (int32_t)(b > a ? b - 1 : b)};"),
]


ALL_MUTANTS = MUTANTS + MUTANTS_PACKS + MUTANTS_FLAT


@pytest.mark.parametrize("name,old,new", ALL_MUTANTS, ids=[m[0] for m in ALL_MUTANTS])
def test_group_check_reports_planted_mistakes(abi, tmp_path, name, old, new):
    import glob
    import os
    import subprocess
    from fully_sharded_shard_b200 import build as B
    src = open(os.path.join(B.CSRC, "fsdpk_api.cu")).read()
    assert src.count(old) == 1, name
    mut = tmp_path / "fsdpk_api.cu"
    mut.write_text(src.replace(old, new))
    obj = tmp_path / "fsdpk_api.o"
    subprocess.run([B.nvcc(), *B.ARCH, *B.CFLAGS, "-I", B.INCLUDE, "-I", B.CSRC, "-c", "-o",
                    str(obj), str(mut)], check=True)
    if len(glob.glob(os.path.join(B.OBJDIR, "*.o"))) < len(B.sources()):
        B.build(force=True)  # the per-file objects the mutant links against
    others = [o for o in glob.glob(os.path.join(B.OBJDIR, "*.o"))
              if os.path.basename(o) != "fsdpk_api.o"]
    lib = tmp_path / "libmut.so"
    subprocess.run([B.nvcc(), *B.ARCH, *B.LDFLAGS, "-o", str(lib), str(obj), *others], check=True)
    L = ctypes.CDLL(str(lib))
    L.fsdp_plan_group_host.argtypes = [ctypes.POINTER(abi.ParamDesc), ctypes.c_int32,
                                       ctypes.c_int32, ctypes.POINTER(ctypes.c_void_p)]
    L.fsdp_group_check.argtypes = [ctypes.c_void_p, ctypes.POINTER(ctypes.c_int64)]
    L.fsdp_destroy_group.argtypes = [ctypes.c_void_p]
    L.fsdp_destroy_group.restype = None
    # ragged rows on several ranks, pads that meet across parameters, a tile
    # boundary inside a pad run
    shapes = [(7, 3), (5,), (1, 32), (13, 9), (2, 2), (9001, 1), (3,)]
    # and enough short runs to fill several packs
    shapes += [(3 + k % 50, 1 + k % 7) for k in range(300)] + [(600, 1)] * 10
    # runs of 512-1023 elements between long ones (700 at N = 2, 3, 4, 6)
    shapes += [(1400, 1), (9001, 1), (2100, 1), (9001, 1), (2800, 1), (4200, 1), (9001, 1)]
    # and tiny ones: the flat path at N = 4 (a partial last vector) and 6, not
    # at N = 2 and 3
    shapes += [(1 + k % 13, 1 + k % 3) for k in range(150)]
    found = 0
    # the same with one large parameter: the flat reduce-scatter, the per-run
    # copy-out (short runs under a tenth of the elements)
    for sh in (shapes, shapes + [(400000, 1)]):
        for N in (2, 3, 4, 6):
            _, arr = abi._descs(sh)
            h = ctypes.c_void_p()
            assert L.fsdp_plan_group_host(arr, len(sh), N, ctypes.byref(h)) == 0
            v = ctypes.c_int64()
            assert L.fsdp_group_check(h, ctypes.byref(v)) == 0
            found += v.value
            L.fsdp_destroy_group(h)
    assert found > 0, f"planted mistake not reported: {name}"
