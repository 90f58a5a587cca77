"""One device's share of a parameter group whose N virtual ranks are spread
over the D processes of a torch.distributed process group (one per GPU).

Device d holds the L = N / D ranks [d*L, (d+1)*L): their fp32 master / m / v
shards [L][S] (the caller's), their bf16 all-gather slot [L][S] and their bf16
unsharded gradients [L][P_arena].  The slot and the gradients live in CUDA IPC
memory that every other process maps (SharedBuffer), so the two exchange
steps of the group ("Introduction to PyTorch FSDP2 Backend Features", Working
Principle: the all-gather before use, the reduce-scatter after backward) are
pulls inside the library's copy-out and reduction kernels, with the reduction
folding ranks 0..N-1 in order exactly as on one device.

torch.distributed is plumbing here: it swaps the 64-byte IPC handles once and
provides the barrier that orders the devices between the phases of a step.
Without an initialised process group everything runs as one device (D = 1).

Two orderings across devices:
  PeerGroup           -- two host barriers per step, each after a device
                         synchronisation (the phases of every device drain);
  PipelinedPeerGroup  -- one host barrier per step and no device
                         synchronisation: every cross-device dependency is a
                         stream wait on another process's CUDA event (CUDA IPC
                         events), with the slots and gradient arenas double
                         buffered by step parity, so one group's exchange
                         overlaps another group's update on the GPU.
"""
from __future__ import annotations

from typing import List, Optional, Sequence, Tuple

import torch
import torch.distributed as dist

from . import abi


def _world(group=None) -> Tuple[int, int]:
    if dist.is_available() and dist.is_initialized():
        return dist.get_world_size(group), dist.get_rank(group)
    return 1, 0


def rank_pointer_tables(slot_bases: Sequence[int], grad_bases: Sequence[int], L: int, S: int,
                        P_arena: int) -> Tuple[List[int], List[int]]:
    """Per-rank pointers: rank r is row r % L of device r // L's slot
    ([L][S] bf16) and gradient arenas ([L][P_arena] bf16)."""
    if len(slot_bases) != len(grad_bases):
        raise ValueError("one slot base and one gradient base per device")
    N = L * len(slot_bases)
    ag = [int(slot_bases[r // L]) + 2 * S * (r % L) for r in range(N)]
    gr = [int(grad_bases[r // L]) + 2 * P_arena * (r % L) for r in range(N)]
    return ag, gr


def exchange(obj, group=None) -> list:
    """Every process's `obj`, in rank order (one all_gather_object)."""
    D, _ = _world(group)
    if D == 1:
        return [obj]
    out = [None] * D
    dist.all_gather_object(out, obj, group=group)
    return out


def barrier(device, group=None) -> None:
    """Every device's queued work is complete before any device goes on."""
    torch.cuda.synchronize(device)
    if _world(group)[0] > 1:
        dist.barrier(group=group)


def host_barrier(group=None) -> None:
    """Every process of the group has reached this point of its program (what
    it enqueued before is enqueued; nothing is waited for on a device).  A
    process that has left raises here in the others within the process
    group's timeout."""
    if _world(group)[0] > 1:
        dist.barrier(group=group)


class SharedBuffer:
    """`nbytes` of this device's memory, mapped into every process of the
    group: `bases[j]` is device j's buffer as seen from this process."""

    def __init__(self, nbytes: int, *, group=None, device=None):
        self.D, self.d = _world(group)
        self.device = device
        self.nbytes = int(nbytes)
        self.ptr, handle = abi.fsdp_ipc_alloc(max(self.nbytes, 16))
        self._opened: List[int] = []
        self.bases: List[int] = []
        for j, h in enumerate(exchange(handle, group)):
            if j == self.d:
                self.bases.append(self.ptr)
            else:
                p = abi.fsdp_ipc_open(h)
                self._opened.append(p)
                self.bases.append(p)

    def view(self, numel: int, dtype: torch.dtype) -> torch.Tensor:
        """This device's buffer as a tensor (valid until release())."""
        return abi.device_tensor(self.ptr, numel, dtype, self.device)

    def unmap_peers(self) -> None:
        for p in self._opened:
            abi.fsdp_ipc_close(p)
        self._opened = []

    def release(self) -> None:
        if self.ptr:
            abi.fsdp_ipc_free(self.ptr)
            self.ptr = 0


def release_all(buffers: Sequence[SharedBuffer], device, group=None) -> None:
    """Unmap every peer buffer, then free this device's, with a barrier
    before each half so that no process still reads a buffer being freed."""
    barrier(device, group)
    for b in buffers:
        b.unmap_peers()
    barrier(device, group)
    for b in buffers:
        b.release()


class PeerGroup:
    """This process's device's part of one parameter group over N virtual
    ranks on the D processes of `group` (default: the world).

    Order of a step across devices (the caller's, via barrier()):
      copy_in (own slot)            -> barrier -> copy_out (pulls every slot)
      gradients into self.grads     -> barrier -> rs_adamw_step / rs_reduce
    and no slot is rewritten before every device's copy-out of it is done
    (the second barrier covers that when copy-outs precede it).
    `grads` may be another PeerGroup's gradient buffer of the same group
    shapes (several instances of one layer share one gradient buffer)."""

    def __init__(self, shapes: Sequence[Sequence[int]], N: int, *, group=None, device=None,
                 grads: Optional[SharedBuffer] = None, fp8: bool = False):
        self.pg = group
        self.device = torch.device(device) if device is not None else torch.device(
            "cuda", torch.cuda.current_device())
        self.D, self.d = _world(group)
        self.g = abi.fsdp_plan_group(shapes, N)
        self.pp = abi.fsdp_peer_plan(self.g, self.D, self.d)
        L, S, A = self.pp.L, self.g.S, self.g.P_arena
        self.L, self.r0, self.S, self.P_arena, self.N = L, self.pp.r0, S, A, self.g.N
        self.slot_buf = SharedBuffer(2 * L * S, group=group, device=self.device)
        self._own_grads = grads is None
        if grads is None:
            grads = SharedBuffer(2 * L * A, group=group, device=self.device)
        elif grads.nbytes < 2 * L * A:
            raise ValueError("shared gradient buffer too small for this group")
        self.grad_buf = grads
        self.ag_slot = self.slot_buf.view(L * S, torch.bfloat16)
        self.grads = self.grad_buf.view(L * A, torch.bfloat16).view(L, A)
        ag, gr = rank_pointer_tables(self.slot_buf.bases, self.grad_buf.bases, L, S, A)
        abi.fsdp_peer_set_sources(self.pp, ag, gr)
        self.slot8_buf = self.amax_buf = None
        if fp8:
            # E4M3 slot rows (1 byte per element) and this device's partial
            # per-parameter amax, both mapped by every device
            self.slot8_buf = SharedBuffer(L * S, group=group, device=self.device)
            self.amax_buf = SharedBuffer(4 * self.g.n, group=group, device=self.device)
            self.ag8_slot = self.slot8_buf.view(L * S, torch.uint8)
            self.amax = self.amax_buf.view(self.g.n, torch.int32)
            ag8 = [int(self.slot8_buf.bases[r // L]) + S * (r % L) for r in range(self.N)]
            abi.fsdp_peer_set_fp8_sources(self.pp, ag8, self.amax_buf.bases)
        self.barrier()

    def barrier(self) -> None:
        barrier(self.device, self.pg)

    # the stages of this device's ranks
    def copy_in(self, master: torch.Tensor, stream=None) -> None:
        abi.fsdp_peer_copy_in(self.pp, master, self.ag_slot, stream)

    def copy_out(self, arena: torch.Tensor, stream=None) -> None:
        abi.fsdp_peer_copy_out(self.pp, arena, stream)

    def rs_reduce(self, op: int, reduced: torch.Tensor, stream=None) -> None:
        abi.fsdp_peer_rs_reduce(self.pp, op, reduced, stream)

    def adamw_step(self, master, m, v, grad, *, stream=None, **hp) -> None:
        abi.fsdp_peer_adamw_step(self.pp, master, m, v, grad, stream=stream, **hp)

    def rs_adamw_step(self, op: int, master, m, v, *, next_copy_in: bool = True,
                      reduced: Optional[torch.Tensor] = None, stream=None, **hp) -> None:
        abi.fsdp_peer_rs_adamw_step(self.pp, op, master, m, v,
                                    ag_next=self.ag_slot if next_copy_in else None,
                                    reduced=reduced, stream=stream, **hp)

    # the FP8 all-gather (delayed scaling): copy-in with given scales, the
    # fused update writing the E4M3 slot and the partial amax, the scales
    # from every device's partial amax (after a barrier), the byte copy-out
    def copy_in_fp8(self, master: torch.Tensor, scales: torch.Tensor, stream=None) -> None:
        abi.fsdp_peer_copy_in_fp8_scaled(self.pp, master, scales, self.ag8_slot, stream)

    def rs_adamw_step_fp8(self, op: int, master, m, v, *, scales_prev: torch.Tensor,
                          reduced: Optional[torch.Tensor] = None, stream=None, **hp) -> None:
        abi.fsdp_peer_rs_adamw_step_fp8(self.pp, op, master, m, v, scales_prev=scales_prev,
                                        ag8_next=self.ag8_slot, amax_local=self.amax,
                                        reduced=reduced, stream=stream, **hp)

    def fp8_scales(self, scales_next: torch.Tensor, stream=None) -> None:
        abi.fsdp_peer_fp8_scales(self.pp, scales_next, stream)

    def copy_out_fp8(self, arena8: torch.Tensor, stream=None) -> None:
        abi.fsdp_peer_copy_out_fp8(self.pp, arena8, stream)

    def buffers(self) -> List[SharedBuffer]:
        extra = [b for b in (self.slot8_buf, self.amax_buf) if b is not None]
        return [self.slot_buf] + ([self.grad_buf] if self._own_grads else []) + extra

    def close(self) -> None:
        """Release the shared buffers (after barriers, so that no peer still
        reads them) and the plans."""
        if self.pp is None:
            return
        self.ag_slot = self.grads = None
        self.ag8_slot = self.amax = None
        release_all(self.buffers(), self.device, self.pg)
        self.pp.destroy()
        self.g.destroy()
        self.pp = None


class PeerEvents:
    """Named interprocess CUDA events of this process, opened by every other
    process of the group: record(name) marks a point on one of this process's
    streams; wait_all(name) makes a stream wait for that point on every
    device (this one included).  A wait on an event never recorded is a
    no-op, so the first step waits for nothing."""

    def __init__(self, names: Sequence[str], *, group=None, device=None):
        self.D, self.d = _world(group)
        with torch.cuda.device(device):
            self.own = {n: torch.cuda.Event(interprocess=True) for n in names}
            handles = {n: e.ipc_handle() for n, e in self.own.items()}
        self.peers = []
        for j, h in enumerate(exchange(handles, group)):
            if j == self.d:
                self.peers.append(self.own)
            else:
                self.peers.append({n: torch.cuda.Event.from_ipc_handle(device, h[n])
                                   for n in names})

    def record(self, name: str, stream) -> None:
        self.own[name].record(stream)

    def wait_all(self, name: str, stream) -> None:
        for ev in self.peers:
            stream.wait_event(ev[name])


def _round_up(x: int, k: int) -> int:
    return (x + k - 1) // k * k


class PipelinedPeerGroup:
    """This device's part of one parameter group, ordered across devices by
    CUDA IPC events instead of device-draining barriers.

    Buffers come in two copies, selected by the parity of the step
    (par = step % 2): the all-gather slot rows [L][S] and the gradient arenas
    [L][P_arena].  Each call waits, on the stream it is given, for the events
    of every device that the data it touches depends on, and records its own:
      copy_in(par)       waits: every device done reading slot[par] (the
                         copy-outs two steps back); writes slot[par];
                         records "in{par}"
      copy_out(par)      waits: every device's "in{par}"; pulls every rank's
                         slot[par] rows; records "out{par}"
      grads_begin(par)   waits: every device done reading grads[par]
      grads_end(par)     records "gw{par}" (the caller wrote grads[par])
      rs_reduce(par)     waits: every device's "gw{par}"; pulls; records "gr{par}"
      rs_adamw_step(par) as rs_reduce, and with the next copy-in it also waits
                         for every device done reading slot[1 - par] and
                         records "in{1 - par}" after writing it
    The caller runs each step in two phases with ONE host barrier between
    them (host_barrier(), which waits for no device): phase A enqueues the
    step's copy-ins and gradient writes, phase B its copy-outs and
    reductions.  That barrier is what makes every wait see the record it
    needs: a wait of phase B sees the records of phase A of the same step,
    and a wait of phase A sees the records of phase B two steps back (the
    buffers of the other parity serve the step in between).  Ordering inside
    this process (for example an update before the next copy-in of the same
    master) is the caller's, as with any two streams.

    With fp8=True the all-gather can also move E4M3 bytes (delayed scaling):
    slot8[par] rows and partial amax arrays amax[par], double buffered too.
      copy_in_fp8(par)        as copy_in, on slot8 ("in8", "out8")
      copy_out_fp8(par)       as copy_out, on slot8
      rs_adamw_step_fp8(par)  waits: every "gw{par}", every "out8{1 - par}"
                              (slot8[1 - par] is rewritten) and every
                              "sc{par}" (amax[par] is zeroed and refilled);
                              records "gr{par}", "in8{1 - par}", "ax{par}"
      fp8_scales(par)         waits: every "ax{par}"; the next scales from
                              every device's amax[par]; records "sc{par}"
    A step's fused update fills amax[par], and the scales it yields are the
    next step's scales_prev: call fp8_scales(par) in phase B of the NEXT step
    (after its host barrier, so that every device's "ax{par}" record is
    enqueued), before that step's fused update."""

    EVENTS = tuple(f"{k}{p}" for k in ("in", "out", "gw", "gr") for p in (0, 1))
    EVENTS_FP8 = tuple(f"{k}{p}" for k in ("in8", "out8", "ax", "sc") for p in (0, 1))

    def __init__(self, shapes: Sequence[Sequence[int]], N: int, *, group=None, device=None,
                 grads: Optional["PipelinedPeerGroup"] = None, fp8: bool = False):
        self.pg = group
        self.device = torch.device(device) if device is not None else torch.device(
            "cuda", torch.cuda.current_device())
        self.D, self.d = _world(group)
        self.g = abi.fsdp_plan_group(shapes, N)
        self.pps = [abi.fsdp_peer_plan(self.g, self.D, self.d) for _ in range(2)]
        L, S, A = self.pps[0].L, self.g.S, self.g.P_arena
        self.L, self.r0, self.S, self.P_arena, self.N = L, self.pps[0].r0, S, A, self.g.N
        self._slot_half = _round_up(2 * L * S, 256)
        self._grad_half = _round_up(2 * L * A, 256)
        self.slot_buf = SharedBuffer(2 * self._slot_half, group=group, device=self.device)
        # `grads`: share another instance's gradient arenas (same shapes), for
        # gradients that are written once and only read afterwards
        self._own_grads = grads is None
        if grads is None:
            self.grad_buf = SharedBuffer(2 * self._grad_half, group=group, device=self.device)
        elif grads.P_arena != A or grads.L != L:
            raise ValueError("shared gradient arenas of another layout")
        else:
            self.grad_buf = grads.grad_buf
        self.ag_slots, self.grads = [], []
        for par in range(2):
            so, go = par * self._slot_half, par * self._grad_half
            self.ag_slots.append(abi.device_tensor(self.slot_buf.ptr + so, L * S, torch.bfloat16,
                                                   self.device))
            self.grads.append(abi.device_tensor(self.grad_buf.ptr + go, L * A, torch.bfloat16,
                                                self.device).view(L, A))
            ag, gr = rank_pointer_tables([b + so for b in self.slot_buf.bases],
                                         [b + go for b in self.grad_buf.bases], L, S, A)
            abi.fsdp_peer_set_sources(self.pps[par], ag, gr)
        self.slot8_buf = self.amax_buf = None
        self.ag8_slots, self.amax = [], []
        if fp8:
            self._slot8_half = _round_up(L * S, 256)
            self._amax_half = _round_up(4 * self.g.n, 256)
            self.slot8_buf = SharedBuffer(2 * self._slot8_half, group=group, device=self.device)
            self.amax_buf = SharedBuffer(2 * self._amax_half, group=group, device=self.device)
            for par in range(2):
                so, ao = par * self._slot8_half, par * self._amax_half
                self.ag8_slots.append(abi.device_tensor(self.slot8_buf.ptr + so, L * S,
                                                        torch.uint8, self.device))
                self.amax.append(abi.device_tensor(self.amax_buf.ptr + ao, self.g.n,
                                                   torch.int32, self.device))
                ag8 = [int(self.slot8_buf.bases[r // L]) + so + S * (r % L)
                       for r in range(self.N)]
                abi.fsdp_peer_set_fp8_sources(self.pps[par], ag8,
                                              [b + ao for b in self.amax_buf.bases])
        self.ev = PeerEvents(self.EVENTS + (self.EVENTS_FP8 if fp8 else ()), group=group,
                             device=self.device)
        barrier(self.device, group)

    # phase A
    def copy_in(self, par: int, master: torch.Tensor, stream) -> None:
        self.ev.wait_all(f"out{par}", stream)
        abi.fsdp_peer_copy_in(self.pps[par], master, self.ag_slots[par], stream)
        self.ev.record(f"in{par}", stream)

    def grads_begin(self, par: int, stream) -> torch.Tensor:
        """Wait until no device still reads grads[par]; returns the buffer to
        write on `stream` (call grads_end after the write)."""
        self.ev.wait_all(f"gr{par}", stream)
        return self.grads[par]

    def grads_end(self, par: int, stream) -> None:
        self.ev.record(f"gw{par}", stream)

    # phase B
    def copy_out(self, par: int, arena: torch.Tensor, stream) -> None:
        self.ev.wait_all(f"in{par}", stream)
        abi.fsdp_peer_copy_out(self.pps[par], arena, stream)
        self.ev.record(f"out{par}", stream)

    def rs_reduce(self, par: int, op: int, reduced: torch.Tensor, stream) -> None:
        self.ev.wait_all(f"gw{par}", stream)
        abi.fsdp_peer_rs_reduce(self.pps[par], op, reduced, stream)
        self.ev.record(f"gr{par}", stream)

    def rs_adamw_step(self, par: int, op: int, master, m, v, *, stream, next_copy_in: bool = True,
                      reduced: Optional[torch.Tensor] = None, **hp) -> None:
        nxt = 1 - par
        self.ev.wait_all(f"gw{par}", stream)
        if next_copy_in:
            self.ev.wait_all(f"out{nxt}", stream)
        abi.fsdp_peer_rs_adamw_step(self.pps[par], op, master, m, v,
                                    ag_next=self.ag_slots[nxt] if next_copy_in else None,
                                    reduced=reduced, stream=stream, **hp)
        self.ev.record(f"gr{par}", stream)
        if next_copy_in:
            self.ev.record(f"in{nxt}", stream)

    # the FP8 all-gather
    def copy_in_fp8(self, par: int, master: torch.Tensor, scales: torch.Tensor, stream) -> None:
        self.ev.wait_all(f"out8{par}", stream)
        abi.fsdp_peer_copy_in_fp8_scaled(self.pps[par], master, scales, self.ag8_slots[par],
                                         stream)
        self.ev.record(f"in8{par}", stream)

    def copy_out_fp8(self, par: int, arena8: torch.Tensor, stream) -> None:
        self.ev.wait_all(f"in8{par}", stream)
        abi.fsdp_peer_copy_out_fp8(self.pps[par], arena8, stream)
        self.ev.record(f"out8{par}", stream)

    def rs_adamw_step_fp8(self, par: int, op: int, master, m, v, *, scales_prev: torch.Tensor,
                          stream, reduced: Optional[torch.Tensor] = None, **hp) -> None:
        nxt = 1 - par
        self.ev.wait_all(f"gw{par}", stream)
        self.ev.wait_all(f"out8{nxt}", stream)
        self.ev.wait_all(f"sc{par}", stream)
        abi.fsdp_peer_rs_adamw_step_fp8(self.pps[par], op, master, m, v, scales_prev=scales_prev,
                                        ag8_next=self.ag8_slots[nxt], amax_local=self.amax[par],
                                        reduced=reduced, stream=stream, **hp)
        self.ev.record(f"gr{par}", stream)
        self.ev.record(f"in8{nxt}", stream)
        self.ev.record(f"ax{par}", stream)

    def fp8_scales(self, par: int, scales_next: torch.Tensor, stream) -> None:
        self.ev.wait_all(f"ax{par}", stream)
        abi.fsdp_peer_fp8_scales(self.pps[par], scales_next, stream)
        self.ev.record(f"sc{par}", stream)

    def buffers(self) -> List[SharedBuffer]:
        extra = [b for b in (self.slot8_buf, self.amax_buf) if b is not None]
        return [self.slot_buf] + ([self.grad_buf] if self._own_grads else []) + extra

    def close(self) -> None:
        """Release the shared buffers (after barriers that drain every device,
        so that no peer still reads them), the events and the plans.  An
        instance that shares another's gradient arenas closes first."""
        if self.pps is None:
            return
        self.ag_slots = self.grads = None
        self.ag8_slots = self.amax = None
        release_all(self.buffers(), self.device, self.pg)
        self.ev = None
        for pp in self.pps:
            pp.destroy()
        self.g.destroy()
        self.pps = None
