"""A device that leaves the exchange between steps, on the host (gloo, CPU).

The several-device exchange orders the devices with one host barrier per
step (fully_sharded_shard_b200.peer.host_barrier).  When one process leaves
between steps -- it exits, raises, or stays alive without joining -- the
others must get an error from their next barrier within the process group's
timeout instead of waiting for good.  The failure is made on the host; no
GPU is involved.
"""
import datetime
import os
import socket
import time

import pytest
import torch.multiprocessing as mp

TIMEOUT_S = 6


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, port, ws, mode, result_dir):
    import torch.distributed as dist
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=ws, timeout=datetime.timedelta(seconds=TIMEOUT_S))
    from fully_sharded_shard_b200 import peer
    msg = "completed"
    t_fail = None
    try:
        for step in range(4):
            if rank == ws - 1 and step == 2:
                if mode == "exit":
                    os._exit(0)
                if mode == "raise":
                    raise RuntimeError("planted failure between steps")
                if mode == "hang":           # alive, never joins the next barrier
                    time.sleep(TIMEOUT_S + 8)
                    os._exit(0)
            t_fail = time.time()
            peer.host_barrier()
    except RuntimeError as e:
        msg = f"error {time.time() - t_fail:.1f} {type(e).__name__}"
        if "planted" in str(e):
            msg = "planted"
    with open(os.path.join(result_dir, f"r{rank}.txt"), "w") as f:
        f.write(msg + "\n")
    os._exit(0)   # no destroy_process_group: a peer is gone


@pytest.mark.parametrize("mode", ["exit", "raise", "hang"])
def test_survivors_get_an_error_when_a_device_leaves_between_steps(tmp_path, mode):
    ws = 3
    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, port, ws, mode, str(tmp_path)))
             for r in range(ws)]
    for p in procs:
        p.start()
    deadline = time.time() + TIMEOUT_S + 60
    for p in procs:
        p.join(max(1.0, deadline - time.time()))
    alive = [p.pid for p in procs if p.is_alive()]
    for p in procs:
        if p.is_alive():
            p.kill()
    assert not alive, f"processes still waiting after {TIMEOUT_S + 60} s: {alive}"
    for r in range(ws - 1):
        msg = open(tmp_path / f"r{r}.txt").read().split()
        assert msg[0] == "error", f"rank {r}: {msg}"
        assert float(msg[1]) <= TIMEOUT_S + 10, f"rank {r} took {msg[1]} s to notice"
