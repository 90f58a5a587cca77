"""Two gloo ranks on CPU: the collectives the sharding step stands in for.

"Sharded Training: FSDP2, DTensor, Tensor and Pipeline Parallelism" runs its
lab as two gloo processes and compares with a single-process reference (the
lab paragraph); this file does the same for the oracle's layouts:

* all_gather_into_tensor of each rank's bf16 shard produces exactly the
  oracle's rank-major copy-in buffer, and the oracle's copy-out of it gives
  back the bf16 parameters;
* reduce_scatter_tensor(SUM) over each rank's packed fp32 buffer produces
  exactly the oracle's reduced shard (two addends commute, so the result is
  order-independent at world size 2);
* reduce-scatter with AVG, and SUM followed by FSDP's own division by the
  world size (set_force_sum_reduction_for_comms, "Other controls" paragraph),
  give the oracle's AVG; the ratio SUM / AVG-as-run is 1.0 (a fixed gloo) or
  2.0 (the bug described in "The bug Adam hid").
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

SHAPES = [(7, 3), (5,), (1, 32), (1,), (13, 9), (2, 2)]
N = 2


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, port, result_dir):
    import oracle
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}",
                            rank=rank, world_size=N)
    try:
        p = oracle.plan(SHAPES, N)
        g = torch.Generator().manual_seed(7)
        full = torch.randn(p.P_arena, generator=g).numpy()
        master = oracle.shard(p, full)
        ag_oracle = oracle.copy_in(p, master)
        # rank-local cast of this rank's padded shard, then the collective
        mine = torch.from_numpy(master[rank * p.S:(rank + 1) * p.S].copy())
        mine_bf16 = mine.to(torch.bfloat16).view(torch.uint8)
        out = torch.empty(N * p.S * 2, dtype=torch.uint8)
        dist.all_gather_into_tensor(out, mine_bf16)
        gathered = out.numpy().view(np.uint16)
        ok_ag = bool(np.array_equal(gathered, ag_oracle))

        # per-rank full gradients (every rank draws all, uses its own)
        grads = torch.randn(N, p.P_arena, generator=g).to(torch.bfloat16)
        grads_np = grads.view(torch.int16).numpy().view(np.uint16).reshape(-1).copy()
        packed = oracle.pack(p, grads_np).reshape(N, N * p.S)
        red_sum = oracle.reduce_packed(p, packed.reshape(-1), oracle.SUM)
        red_avg = oracle.reduce_packed(p, packed.reshape(-1), oracle.AVG)
        send = torch.from_numpy(packed[rank].copy())
        recv = torch.empty(p.S)
        dist.reduce_scatter_tensor(recv, send, op=dist.ReduceOp.SUM)
        mine_sum = red_sum[rank * p.S:(rank + 1) * p.S]
        ok_sum = bool(np.array_equal(recv.numpy().view(np.uint32), mine_sum.view(np.uint32)))
        # SUM then FSDP's own division by the world size
        divided = (recv / N).numpy()
        mine_avg = red_avg[rank * p.S:(rank + 1) * p.S]
        ok_div = bool(np.array_equal(divided.view(np.uint32), mine_avg.view(np.uint32)))
        recv_avg = torch.empty(p.S)
        dist.reduce_scatter_tensor(recv_avg, send, op=dist.ReduceOp.AVG)
        nz = np.abs(mine_avg) > 0
        ratio = float(np.median(recv_avg.numpy()[nz] / mine_avg[nz]))
        with open(os.path.join(result_dir, f"r{rank}.txt"), "w") as f:
            f.write(f"{ok_ag} {ok_sum} {ok_div} {ratio}\n")
    finally:
        dist.destroy_process_group()


def test_gloo_all_gather_and_reduce_scatter_match_oracle(tmp_path, oracle, golden):
    mp.spawn(_worker, args=(_free_port(), str(tmp_path)), nprocs=N, join=True)
    accepted = golden["avg_bug"]["gloo_avg_over_sum_ratio_accepted"]
    for r in range(N):
        ok_ag, ok_sum, ok_div, ratio = open(tmp_path / f"r{r}.txt").read().split()
        assert ok_ag == "True", f"rank {r}: all-gather layout differs"
        assert ok_sum == "True", f"rank {r}: reduce-scatter SUM differs"
        assert ok_div == "True", f"rank {r}: SUM + divide differs from AVG"
        assert any(abs(float(ratio) - a) < 1e-6 for a in accepted), ratio
