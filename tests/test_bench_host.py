"""Host-side logic of bench.py without a GPU: the byte model, the
max-over-ranks timing reduction across two gloo ranks, the clock-sample
parser and the reference arm (the oracle on the host cores)."""
import json
import os
import socket
import subprocess
import sys

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402
from fully_sharded_shard_b200 import workloads as W  # noqa: E402


def test_byte_model_is_42_plus_2n_per_unpadded_param(oracle):
    for N in (2, 6, 8):
        assert bench.group_bytes(N, 1000, N * 1000) == (42 + 2 * N) * N * 1000
    wl = W.llama7b()
    total = 0
    for g in wl.groups:
        p = oracle.plan(g.shapes, wl.N)
        total += g.repeat * bench.group_bytes(wl.N, p.S, p.P)
    assert total == 58 * 6_738_415_616 == 390_828_105_728


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank(rank, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE="2", LOCAL_RANK=str(rank))
    bench.init_dist("gloo")
    v = bench.max_over_ranks(10.0 + 5.0 * rank)
    bench.barrier()
    with open(os.path.join(out, f"{rank}.txt"), "w") as f:
        f.write(repr(v))
    import torch.distributed as dist
    dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks(tmp_path):
    mp.spawn(_rank, args=(_free_port(), str(tmp_path)), nprocs=2, join=True)
    for r in range(2):
        assert float(open(tmp_path / f"{r}.txt").read()) == 15.0


def test_clock_sampler_parses_nvidia_smi_rows(tmp_path):
    cs = bench.ClockSampler(0)
    with open(cs.out.name, "w") as f:
        f.write("0, 1965, 1965, 650.2, 0x0, Not Active, Not Active, Not Active, Active\n")
        f.write("0, 1950, 1965, 700.1, 0x4, Not Active, Not Active, Not Active, Active\n")
        f.write("0, 345, 1965, 90.0, 0x0, Not Active, Not Active, Not Active, Not Active\n")
    cs.proc = type("P", (), {"terminate": lambda s: None, "wait": lambda s, timeout=None: 0})()
    rep = cs.stop()
    assert rep["sm_max_mhz"] == 1965 and rep["samples"] == 3 and rep["samples_under_load"] == 2
    assert rep["sm_mhz"] == 1957.5 and rep["reasons"] == ["sw_power_cap"]


def test_reference_arm_prints_one_json_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "llama7b_div16_l1", "--steps", "1", "--warmup", "0"],
                       capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    out = json.loads(lines[0])
    assert out["impl"] == "reference" and out["unit"] == "GB/s" and out["value"] > 0
    assert out["cpu_baseline"]["kind"] == "oracle" and out["cpu_baseline"]["cores"] >= 1
    assert out["e2e"]["h2d_bytes_per_step"] == 0 and out["metric"] == bench.METRIC


def test_fused_byte_model_is_30_plus_2n_per_unpadded_param():
    for N in (2, 6, 8):
        assert sum(bench.fused_stage_bytes(N, 1000, N * 1000).values()) == (30 + 2 * N) * N * 1000


def test_fused_fp8_byte_model_is_27_plus_2n_per_unpadded_param():
    for N in (1, 2, 8):
        b = bench.fused_fp8_stage_bytes(N, 1000, N * 1000, 0)
        assert sum(b.values()) == (27 + 2 * N) * N * 1000
        assert bench.fused_fp8_stage_bytes(N, 1000, N * 1000, 5)["rs_adamw_copy_in_fp8"] \
            == b["rs_adamw_copy_in_fp8"] + 60


def test_peer_byte_model_reduces_to_the_single_device_model():
    N, S, P = 8, 1000, 7900
    one = bench.peer_stage_bytes(N, S, P, N, P)
    assert sum(one.values()) == bench.group_bytes(N, S, P)
    assert bench.peer_exchange_bytes(N, S, N, P, 1) == 0
    # spread over 4 devices: the local stages split, every device copies out all
    P_local = [2000, 2000, 2000, 1900]
    per = [bench.peer_stage_bytes(N, S, P, 2, pl) for pl in P_local]
    assert sum(b["copy_in"] for b in per) == one["copy_in"]
    assert sum(b["rs_reduce"] for b in per) == one["rs_reduce"]
    assert sum(b["adamw"] for b in per) == one["adamw"]
    assert all(b["copy_out"] == one["copy_out"] for b in per)
    assert bench.peer_exchange_bytes(N, S, 2, 2000, 4) == 2 * 6 * S + 2 * 6 * 2000


def test_staged_byte_model_is_the_fused_one_plus_8n_per_param():
    for N in (2, 6, 8):
        fused = 2 * N * N * 1000 + 4 * N * 1000
        assert bench.staged_rs_bytes(N, 1000, N * 1000) == fused + 8 * N * N * 1000


def test_local_real_elems_split_the_group_across_devices(oracle):
    from fully_sharded_shard_b200 import workloads as W
    for wl in (W.uneven(), W.moe(), W.llama7b(), W.tiny_mlp()):
        for grp in wl.groups:
            p = oracle.plan(grp.shapes, wl.N)
            rows = [int(x) for x in p.chunk_rows]
            for D in [d for d in range(1, wl.N + 1) if wl.N % d == 0]:
                L = wl.N // D
                parts = [bench.local_real_elems(grp.shapes, rows, d * L, L) for d in range(D)]
                assert sum(parts) == p.P
                for d in range(D):  # against the oracle's valid rows, rank by rank
                    want = sum(p.valid_rows(i, j) * int(p.cols[i])
                               for i in range(p.n) for j in range(d * L, (d + 1) * L))
                    assert parts[d] == want


def test_profile_stages_byte_model_matches_the_bench():
    """The single-stage profiler counts each stage's algorithmic bytes with
    the bench's byte model (the fused update: reduce-scatter + AdamW + next
    copy-in, 2N B per real element + 26 B per padded element)."""
    from fully_sharded_shard_b200 import profile_stages as PS
    for N, S, P in ((8, 1000, 8000), (6, 1001, 5990), (2, 7, 13)):
        sb = bench.stage_bytes(N, S, P)
        for k in ("copy_in", "copy_out", "rs_reduce", "adamw"):
            assert PS.stage_bytes(k, N, S, P) == sb[k], k
        assert PS.stage_bytes("rs_adamw", N, S, P) == sum(bench.fused_stage_bytes(N, S, P).values()) \
            - bench.fused_stage_bytes(N, S, P)["copy_out"]
