"""The debug build (libfsdpk_debug.so, -DFSDPK_DEBUG): every table-driven
kernel checks each work unit against the extents of the buffers it was
given, skips a unit that would reach outside and counts it in the caller's
error words, without trapping or waiting.

Run in child processes with FSDPK_DEBUG=1 (the binding picks the library at
import): the brute-force grid, 40 random groups and the emulated
several-device pulls through every stage report zero violations, bit-exact
against the oracle as in the release build; with every extent narrowed by
one element (the test-only `shrink`), valid tables trip the copy-out and
reduce-scatter checks and the skipped units are left untouched.
"""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(mode: str) -> dict:
    from fully_sharded_shard_b200 import build
    build.build(debug=True)
    env = dict(os.environ, FSDPK_DEBUG="1")
    p = subprocess.run([sys.executable, os.path.join(ROOT, "tests", "_debug_run.py"), mode],
                       env=env, capture_output=True, text=True, timeout=1500)
    assert p.returncode == 0, p.stdout[-2000:] + p.stderr[-4000:]
    line = [x for x in p.stdout.splitlines() if x.startswith("RESULT ")][-1]
    return json.loads(line[len("RESULT "):])


def test_debug_build_grid_has_no_violations():
    out = _run("grid")
    assert out["cases"] == 54          # 9 grid groups, 40 random groups, 2 peer cases, 3 flat
    assert out["words"][0] == 0, f"violations: {out['words']}"


def test_debug_build_checks_fire_on_narrowed_extents():
    out = _run("shrink")
    assert out["copy_out"][0] > 0 and out["copy_out"][1] == 2, out   # kDbgCopyOut
    assert out["tail_kept"], "a skipped unit was written"
    assert out["reduce"][0] > 0 and out["reduce"][1] == 5, out       # kDbgReduce
    # the flat path of a group of many small parameters
    assert out["flat_copy_out"][0] > 0 and out["flat_copy_out"][1] == 19, out  # kDbgCopyOutFlat
    assert out["flat_tail_kept"], "a skipped element was written"
    assert out["flat_reduce"][0] > 0 and out["flat_reduce"][1] == 17, out      # kDbgReduceFlat
    assert out["flat_reduce_kept"], out
    assert out["flat_update"][0] > 0 and out["flat_update"][1] == 18, out      # kDbgRsAdamwFlat
    assert out["flat_update_kept"], out
