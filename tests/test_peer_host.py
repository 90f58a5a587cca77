"""Host logic of the several-device exchange, on CPU.

* rank_pointer_tables: rank r is row r % L of device r // L's slot and
  gradient arenas;
* two gloo processes swap their IPC handles and build the same tables;
* PeerGroup's protocol against a stand-in of the library (no GPU): it opens
  every other device's two shared buffers and never its own, passes the
  tables in rank order, and on close unmaps the peers' buffers before freeing
  its own, with a barrier on each side.
"""
import os
import socket
import types

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from fully_sharded_shard_b200.peer import rank_pointer_tables


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def test_rank_pointer_tables_rows_of_devices():
    slot_bases = [0x10000, 0x20000, 0x30000]
    grad_bases = [0x90000, 0xA0000, 0xB0000]
    L, S, A = 2, 5, 16
    ag, gr = rank_pointer_tables(slot_bases, grad_bases, L, S, A)
    assert len(ag) == len(gr) == 6
    for r in range(6):
        d, row = divmod(r, L)
        assert ag[r] == slot_bases[d] + row * S * 2
        assert gr[r] == grad_bases[d] + row * A * 2
    # one device holding every rank is the single-buffer [N][S] layout
    ag1, gr1 = rank_pointer_tables([0x1000], [0x8000], 4, 7, 24)
    assert ag1 == [0x1000 + 14 * r for r in range(4)]
    assert gr1 == [0x8000 + 48 * r for r in range(4)]
    with pytest.raises(ValueError):
        rank_pointer_tables([1, 2], [3], 1, 1, 8)


class _FakeLib:
    """The calls PeerGroup makes, recorded; pointers are fake integers that
    encode (device, buffer)."""

    def __init__(self, d, log):
        self.d, self.log = d, log

    def fsdp_plan_group(self, shapes, N):
        return types.SimpleNamespace(N=N, S=10, P_arena=24, n=len(shapes),
                                     destroy=lambda: self.log.append("g.destroy"))

    def fsdp_peer_plan(self, g, D, d):
        L = g.N // D
        return types.SimpleNamespace(L=L, r0=d * L, destroy=lambda: self.log.append("pp.destroy"))

    def fsdp_ipc_alloc(self, nbytes):
        kind = sum(1 for e in self.log if e[0] == "alloc")
        ptr = (self.d + 1) * 0x1000000 + kind * 0x100000
        self.log.append(("alloc", ptr, nbytes))
        return ptr, ptr.to_bytes(8, "little") * 8

    def fsdp_ipc_open(self, handle):
        ptr = int.from_bytes(handle[:8], "little")
        self.log.append(("open", ptr))
        return ptr + 0x10  # mapped at another address in this process

    def fsdp_ipc_close(self, ptr):
        self.log.append(("close", ptr))

    def fsdp_ipc_free(self, ptr):
        self.log.append(("free", ptr))

    def device_tensor(self, ptr, numel, dtype, device):
        return torch.zeros(numel, dtype=dtype)

    def fsdp_peer_set_sources(self, pp, ag, gr):
        self.log.append(("tables", list(ag), list(gr)))

    def fsdp_peer_set_fp8_sources(self, pp, ag8, amax):
        self.log.append(("fp8_tables", list(ag8), list(amax)))


def _protocol_worker(rank, port, D, N, result_dir):
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=D)
    try:
        import fully_sharded_shard_b200.peer as peer
        log = []
        fake = _FakeLib(rank, log)
        peer.abi = fake
        peer.torch.cuda.synchronize = lambda *a, **k: log.append("sync")
        pg = peer.PeerGroup([(7, 3), (5,)], N, device="cpu")
        L = N // D
        assert (pg.L, pg.r0) == (L, rank * L)
        allocs = [e for e in log if e[0] == "alloc"]
        assert [a[2] for a in allocs] == [2 * L * 10, 2 * L * 24]
        opens = [e[1] for e in log if e[0] == "open"]
        # every other device's slot, then every other device's gradient arenas
        expect_open = [(j + 1) * 0x1000000 for j in range(D) if j != rank]
        expect_open += [(j + 1) * 0x1000000 + 0x100000 for j in range(D) if j != rank]
        assert opens == expect_open, (opens, expect_open)
        tables = [e for e in log if e[0] == "tables"]
        assert len(tables) == 1
        _, ag, gr = tables[0]
        for r in range(N):
            j, row = divmod(r, L)
            base_s = (j + 1) * 0x1000000 + (0 if j == rank else 0x10)
            base_g = (j + 1) * 0x1000000 + 0x100000 + (0 if j == rank else 0x10)
            assert ag[r] == base_s + 2 * 10 * row
            assert gr[r] == base_g + 2 * 24 * row
        n_before = len(log)
        pg.close()
        tail = log[n_before:]
        kinds = [e if isinstance(e, str) else e[0] for e in tail]
        # barrier, unmap peers, barrier, free own, destroy plans
        assert kinds[0] == "sync"
        first_free = kinds.index("free")
        assert all(k != "close" for k in kinds[first_free:])
        assert "sync" in kinds[kinds.index("close") if "close" in kinds else 0:first_free]
        assert [e[1] for e in tail if e[0] == "close"] == [p + 0x10 for p in expect_open]
        assert sorted(e[1] for e in tail if e[0] == "free") == sorted(a[1] for a in allocs)
        assert kinds[-2:] == ["pp.destroy", "g.destroy"]
        with open(os.path.join(result_dir, f"r{rank}.txt"), "w") as f:
            f.write("ok\n")
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("D,N", [(2, 4), (3, 3)])
def test_peer_group_protocol_gloo(tmp_path, D, N):
    mp.spawn(_protocol_worker, args=(_free_port(), D, N, str(tmp_path)), nprocs=D, join=True)
    for r in range(D):
        assert open(tmp_path / f"r{r}.txt").read().strip() == "ok"


def _fp8_protocol_worker(rank, port, D, N, result_dir):
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=D)
    try:
        import fully_sharded_shard_b200.peer as peer
        log = []
        peer.abi = _FakeLib(rank, log)
        peer.torch.cuda.synchronize = lambda *a, **k: log.append("sync")
        pg = peer.PeerGroup([(7, 3), (5,)], N, device="cpu", fp8=True)
        L = N // D
        allocs = [e for e in log if e[0] == "alloc"]
        # bf16 slot, gradients, E4M3 slot (1 B per element), partial amax (4 B per
        # parameter); every shared buffer is at least 16 bytes
        assert [a[2] for a in allocs] == [2 * L * 10, 2 * L * 24, max(L * 10, 16), max(4 * 2, 16)]
        fp8 = [e for e in log if e[0] == "fp8_tables"]
        assert len(fp8) == 1
        _, ag8, amax = fp8[0]
        for r in range(N):
            j, row = divmod(r, L)
            base = (j + 1) * 0x1000000 + 2 * 0x100000 + (0 if j == rank else 0x10)
            assert ag8[r] == base + 10 * row  # byte rows
        assert amax == [(j + 1) * 0x1000000 + 3 * 0x100000 + (0 if j == rank else 0x10)
                        for j in range(D)]
        n_before = len(log)
        pg.close()
        tail = log[n_before:]
        assert sorted(e[1] for e in tail if e[0] == "free") == sorted(a[1] for a in allocs)
        assert len([e for e in tail if e[0] == "close"]) == 4 * (D - 1)
        with open(os.path.join(result_dir, f"r{rank}.txt"), "w") as f:
            f.write("ok\n")
    finally:
        dist.destroy_process_group()


def test_peer_group_fp8_protocol_gloo(tmp_path):
    D, N = 2, 4
    mp.spawn(_fp8_protocol_worker, args=(_free_port(), D, N, str(tmp_path)), nprocs=D, join=True)
    for r in range(D):
        assert open(tmp_path / f"r{r}.txt").read().strip() == "ok"
