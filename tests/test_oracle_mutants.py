"""The oracle's pins catch plausible mistakes.

Each case below plants one mistake in a copy of oracle/fsdp_oracle.c (a
dropped term, a wrong index, a transposed operand, a wrong rounding rule),
builds it into a separate library on the CPU, points the oracle at it and
runs the pins that cover that function: at least one must fail.  The real
oracle is restored afterwards.
"""
import ctypes
import importlib
import os
import subprocess
import tempfile

import numpy as np
import pytest

import oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "fsdp_oracle.c")

t_plan = importlib.import_module("tests.test_oracle_plan")
t_bf16 = importlib.import_module("tests.test_oracle_bf16")
t_gather = importlib.import_module("tests.test_oracle_gather")
t_reduce = importlib.import_module("tests.test_oracle_reduce")
t_adamw = importlib.import_module("tests.test_oracle_adamw")
t_acc = importlib.import_module("tests.test_oracle_accumulate")
t_fp8 = importlib.import_module("tests.test_oracle_fp8")
t_acct = importlib.import_module("tests.test_accounting")

SUM, AVG, STD = 0, 1, 2
RAGGED = ("ragged", [(7, 3), (5,), (1, 32), (1,), (0, 4), (13, 9), (2, 2)], 4)


def _plan_pins(o, g):
    t_plan.test_chunk_rows_brute_force(o)
    t_plan.test_worked_shapes_from_the_pages(o, g)
    t_plan.test_tiny_mlp_sizes_and_zero1_contrast(o, g)


def _gather_pins(o, g):
    from fully_sharded_shard_b200 import workloads as W
    t_plan.test_plan_matches_torch_chunk_on_every_config_shape(o, W.uneven(64))
    t_gather.test_shard_and_copy_in_match_torch_chunk(o, *t_gather.SMALL_GROUPS[1])
    t_gather.test_all_gather_of_shard_is_identity(o, *t_gather.SMALL_GROUPS[1])
    t_gather.test_pad_rows_are_zero_even_if_master_pad_is_not(o)
    t_gather.test_shard_pads_are_positive_zero(o)


def _reduce_pins(o, g):
    for grp in (RAGGED, t_reduce.GROUPS[3], t_reduce.GROUPS[5]):   # N = 4, 9, 6
        for op in (SUM, AVG, STD):
            for form in ("packed", "direct"):
                t_reduce.test_reduce_scatter_then_all_gather_equals_all_reduce(o, *grp, op, form)
        t_reduce.test_avg_sum_relations(o, *grp)
    t_reduce.test_fold_order_is_rank_order(o)
    t_reduce.test_pack_layout_is_reduce_scatter_input(o)


def _adamw_pins(o, g):
    t_adamw.test_first_step_closed_form(o)
    t_adamw.test_zero_gradient_only_decays(o)
    t_adamw.test_sharded_adamw_matches_torch_adamw(o, [(7, 3), (5,), (1, 32), (1,), (13, 9)], 4)


def _acc_pins(o, g):
    t_acc.test_accumulate_matches_torch_fp32_adds(o)
    t_acc.test_accumulation_order_is_microbatch_order(o)
    for op in (SUM, AVG):
        t_acc.test_fp32_reduce_scatter_then_all_gather_equals_all_reduce(o, *t_acc.GROUPS[0], op)


def _fp8_pins(o, g):
    t_fp8.test_e4m3_special_values(o)
    t_fp8.test_scales_and_copy_in_against_torch(o)
    t_fp8.test_copy_out_round_trip(o)


def _bf16_pins(o, g):
    t_bf16.test_special_values(o)
    t_gather.test_shard_and_copy_in_match_torch_chunk(o, *t_gather.SMALL_GROUPS[4])


MUTANTS = [
    ("chunk rows floor", "return (d0 + N - 1) / N;", "return d0 / N + (d0 % N != 0 && d0 < N);", _plan_pins),
    ("valid rows unclamped", "    if (left > c) left = c;\n", "", _plan_pins),
    ("arena offsets unaligned", "u[i] = ((A + 7) / 8) * 8;", "u[i] = A;", _gather_pins),
    ("bf16 ties round up", "(dropped == 0x8000u && (upper & 1u))", "(dropped == 0x8000u)", _bf16_pins),
    ("bf16 truncates", "upper += 1u; /* carries", "upper += 0u; /* carries", _bf16_pins),
    ("copy-in pads keep master", ": (uint16_t)0; /* +0 in every pad row */",
     ": or_bf16_rne_bits(f32_bits(master[k]));", _gather_pins),
    ("shard pad not zero", "master[dst] = 0.0f; /* pad row */", "master[dst] = -0.0f; /* pad row */", _gather_pins),
    ("copy-out wrong slot", "int64_t local = row - r * c[i];", "int64_t local = row % c[i] + (r > 0);", _gather_pins),
    ("pack transposed ranks", "grads[(int64_t)r * A + u[i] + grow * cols[i] + col]);",
     "grads[(int64_t)j * A + u[i] + grow * cols[i] + col]);", _reduce_pins),
    ("AVG as multiply", "if (op == OR_AVG) out = out / (float)N;",
     "if (op == OR_AVG) out = out * (1.0f / (float)N);", _reduce_pins),
    ("fold skips rank 0", "float acc = packed[jk]; /* r = 0: packed[0][j][k] */",
     "float acc = 0.0f * packed[jk];", _reduce_pins),
    ("SUM_THEN_DIV without division", "for (int64_t jk = 0; jk < total; ++jk) red[jk] = red[jk] / (float)N;",
     "for (int64_t jk = 0; jk < total; ++jk) red[jk] = red[jk];", _reduce_pins),
    ("direct reduce reads shard offset", "int64_t src = u[i] + ((int64_t)j * c[i] + row) * cols[i] + col;",
     "int64_t src = off[i] + ((int64_t)j * c[i] + row) * cols[i] + col;", _reduce_pins),
    ("adamw no bias correction", "double mhat = mk / bc1;", "double mhat = mk;", _adamw_pins),
    ("adamw decay sign", "pk = pk * (1.0 - lr * wd);", "pk = pk * (1.0 + lr * wd);", _adamw_pins),
    ("adamw eps inside sqrt", "pk = pk - lr * mhat / (sqrt(vhat) + eps);",
     "pk = pk - lr * mhat / sqrt(vhat + eps);", _adamw_pins),
    ("adamw beta1 on gradient", "mk = beta1 * mk + (1.0 - beta1) * gk;", "mk = (1.0 - beta1) * mk + beta1 * gk;", _adamw_pins),
    ("adamw v without square", "vk = beta2 * vk + (1.0 - beta2) * gk * gk;", "vk = beta2 * vk + (1.0 - beta2) * fabs(gk);", _adamw_pins),
    ("accumulate ignores first", "acc[k] = first ? g : acc[k] + g;", "acc[k] = acc[k] + g;", _acc_pins),
    ("f32 reduce skips rank 0", "float acc = src[k];", "float acc = 0.0f;", _acc_pins),
    ("e4m3 subnormal grid", "double q = nearbyint(a * 512.0);", "double q = nearbyint(a * 256.0);", _fp8_pins),
    ("e4m3 exponent bias", "int field = e + 7;", "int field = e + 8;", _fp8_pins),
    ("fp8 scale constant", "return 448.0f / a;", "return 240.0f / a;", _fp8_pins),
    ("fp8 no clamp", "    if (y > 448.0f) y = 448.0f;\n", "", _fp8_pins),
]


def _build_mutant(src_text: str, tmpdir: str) -> str:
    c = os.path.join(tmpdir, "mutant.c")
    so = os.path.join(tmpdir, "libmutant.so")
    with open(c, "w") as f:
        f.write(src_text)
    subprocess.run(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
                    "-fPIC", "-shared", "-o", so, c, "-lm"], check=True, capture_output=True)
    return so


@pytest.mark.parametrize("name,old,new,pins", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_is_caught(name, old, new, pins, golden):
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation site not found: {old!r}"
    mutated = src.replace(old, new)
    assert mutated != src
    real = O.lib()
    with tempfile.TemporaryDirectory() as d:
        so = _build_mutant(mutated, d)
        O._lib = None
        O._LIB_SAVED = O._LIB
        try:
            O._LIB = so
            O.build = lambda force=False, _so=so: _so  # the mutant is prebuilt
            caught = False
            try:
                pins(O, golden)
            except (AssertionError, ValueError, IndexError):
                caught = True
            assert caught, f"planted mistake '{name}' passed every pin"
        finally:
            O._LIB = O._LIB_SAVED
            O._lib = real
            O.build = _orig_build


_orig_build = O.build
