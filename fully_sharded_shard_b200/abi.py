"""Thin ctypes binding of libfsdpk.so (declared in include/fsdpk.h).

Argument marshalling only: every step of the path runs in the library's CUDA
kernels.  Tensors are passed by ``data_ptr()``; the stream defaults to torch's
current stream on the tensors' device.  There is no fallback: importing this
module without the built library raises, and every non-OK status raises
``FsdpError``.

Function names follow the C entry points:
``fsdp_plan_group``, ``fsdp_shard_params``, ``fsdp_copy_in``,
``fsdp_copy_out``, ``fsdp_rs_reduce``, ``fsdp_adamw_step``,
``fsdp_rs_adamw_step`` (reduce-scatter + AdamW + next copy-in, fused) and
``fsdp_rs_reduce_noalloc``.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
# FSDPK_DEBUG=1 loads the debug build (kernels check every work unit against
# the extents of their buffers; see fsdp_debug_set_error_words)
DEBUG = os.environ.get("FSDPK_DEBUG", "") == "1"
LIB_PATH = os.path.join(_PKG, "libfsdpk_debug.so" if DEBUG else "libfsdpk.so")

FSDP_MAX_NDIM = 8
FSDP_MAX_WORLD = 1024

FSDP_OK, FSDP_EINVAL, FSDP_ENOMEM, FSDP_ECUDA, FSDP_EALIGN, FSDP_ESTATE = 0, -1, -2, -3, -4, -5
FSDP_SUM, FSDP_AVG, FSDP_SUM_THEN_DIV = 0, 1, 2
FSDP_PEER_MAX_RANKS = 64

EXPORTED = (
    "fsdp_plan_group", "fsdp_group_sizes", "fsdp_group_param_offsets",
    "fsdp_destroy_group", "fsdp_shard_params", "fsdp_copy_in", "fsdp_copy_out",
    "fsdp_rs_reduce", "fsdp_adamw_step", "fsdp_status_string",
    "fsdp_last_cuda_error", "fsdp_abi_version",
)


class FsdpError(RuntimeError):
    def __init__(self, status: int, where: str):
        msg = _lib.fsdp_status_string(status).decode()
        if status == FSDP_ECUDA:
            msg += f" (cudaError {_lib.fsdp_last_cuda_error()})"
        super().__init__(f"{where}: {msg} [{status}]")
        self.status = status


class ParamDesc(ctypes.Structure):
    _fields_ = [("ndim", ctypes.c_int32), ("shape", ctypes.c_int64 * FSDP_MAX_NDIM)]


class IpcHandle(ctypes.Structure):
    _fields_ = [("bytes", ctypes.c_uint8 * 64)]


class AdamWHparams(ctypes.Structure):
    _fields_ = [("lr", ctypes.c_double), ("beta1", ctypes.c_double),
                ("beta2", ctypes.c_double), ("eps", ctypes.c_double),
                ("weight_decay", ctypes.c_double), ("step", ctypes.c_int64)]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{os.path.basename(LIB_PATH)} is not built ({LIB_PATH}); run "
            "`python -m fully_sharded_shard_b200.build" + (" --debug" if DEBUG else "") +
            "` (needs nvcc)")
    L = ctypes.CDLL(LIB_PATH)
    vp, i32, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
    L.fsdp_plan_group.argtypes = [ctypes.POINTER(ParamDesc), i32, i32, ctypes.POINTER(vp)]
    L.fsdp_group_sizes.argtypes = [vp, ctypes.POINTER(i64), ctypes.POINTER(i64), ctypes.POINTER(i64)]
    L.fsdp_group_param_offsets.argtypes = [vp, vp, vp, vp]
    L.fsdp_destroy_group.argtypes = [vp]
    L.fsdp_destroy_group.restype = None
    L.fsdp_shard_params.argtypes = [vp, vp, vp, vp]
    L.fsdp_copy_in.argtypes = [vp, vp, vp, vp]
    L.fsdp_copy_out.argtypes = [vp, vp, vp, vp]
    L.fsdp_rs_reduce.argtypes = [vp, vp, i32, vp, vp, vp]
    L.fsdp_adamw_step.argtypes = [vp, vp, vp, vp, vp, ctypes.POINTER(AdamWHparams), vp]
    L.fsdp_rs_adamw_step.argtypes = [vp, vp, i32, vp, vp, vp, ctypes.POINTER(AdamWHparams), vp,
                                     vp, vp]
    L.fsdp_rs_adamw_step.restype = ctypes.c_int
    L.fsdp_grad_accumulate.argtypes = [vp, vp, vp, i32, vp]
    L.fsdp_grad_accumulate.restype = ctypes.c_int
    L.fsdp_rs_reduce_accumulated.argtypes = [vp, vp, vp, i32, vp, vp]
    L.fsdp_rs_reduce_accumulated.restype = ctypes.c_int
    L.fsdp_copy_in_fp8.argtypes = [vp, vp, vp, vp, vp]
    L.fsdp_copy_in_fp8.restype = ctypes.c_int
    L.fsdp_copy_in_fp8_scaled.argtypes = [vp, vp, vp, vp, vp]
    L.fsdp_copy_in_fp8_scaled.restype = ctypes.c_int
    L.fsdp_rs_adamw_step_fp8.argtypes = [vp, vp, i32, vp, vp, vp, ctypes.POINTER(AdamWHparams),
                                         vp, vp, vp, vp, vp]
    L.fsdp_rs_adamw_step_fp8.restype = ctypes.c_int
    L.fsdp_copy_out_fp8.argtypes = [vp, vp, vp, vp]
    L.fsdp_copy_out_fp8.restype = ctypes.c_int
    L.fsdp_adamw_prepare.argtypes = [ctypes.POINTER(AdamWHparams), vp, vp, vp]
    L.fsdp_adamw_prepare.restype = ctypes.c_int
    L.fsdp_adamw_step_dev.argtypes = [vp, vp, vp, vp, vp, vp, vp]
    L.fsdp_adamw_step_dev.restype = ctypes.c_int
    L.fsdp_rs_adamw_step_dev.argtypes = [vp, vp, i32, vp, vp, vp, vp, vp, vp, vp]
    L.fsdp_rs_adamw_step_dev.restype = ctypes.c_int
    L.fsdp_debug_build.restype = ctypes.c_int
    L.fsdp_debug_set_error_words.argtypes = [vp, i64]
    L.fsdp_debug_set_error_words.restype = ctypes.c_int
    L.fsdp_rs_reduce_noalloc.argtypes = [ctypes.POINTER(ParamDesc), i32, i32, vp, i32, vp, vp]
    L.fsdp_rs_reduce_noalloc.restype = ctypes.c_int
    L.fsdp_copy_in_f32.argtypes = [vp, vp, vp, vp]
    L.fsdp_copy_in_f32.restype = ctypes.c_int
    L.fsdp_copy_out_f32.argtypes = [vp, vp, vp, vp]
    L.fsdp_copy_out_f32.restype = ctypes.c_int
    L.fsdp_plan_group_host.argtypes = [ctypes.POINTER(ParamDesc), i32, i32, ctypes.POINTER(vp)]
    L.fsdp_plan_group_host.restype = ctypes.c_int
    L.fsdp_group_check.argtypes = [vp, ctypes.POINTER(i64)]
    L.fsdp_group_check.restype = ctypes.c_int
    L.fsdp_group_flat.argtypes = [vp, ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(i64),
                                  ctypes.POINTER(i64)]
    L.fsdp_group_flat.restype = ctypes.c_int
    L.fsdp_group_step.argtypes = [vp, vp, vp, vp, vp, i32, ctypes.POINTER(AdamWHparams), vp, vp,
                                  vp, vp]
    L.fsdp_group_step.restype = ctypes.c_int
    L.fsdp_group_step_dev.argtypes = [vp, vp, vp, vp, vp, i32, vp, vp, vp, vp, vp]
    L.fsdp_group_step_dev.restype = ctypes.c_int
    L.fsdp_group_step_graph.argtypes = [vp, vp, vp, vp, vp, i32, ctypes.POINTER(AdamWHparams),
                                        vp, vp, vp, vp, vp, vp]
    L.fsdp_group_step_graph.restype = ctypes.c_int
    L.fsdp_peer_plan.argtypes = [vp, i32, i32, ctypes.POINTER(vp)]
    L.fsdp_peer_local_ranks.argtypes = [vp, ctypes.POINTER(i32), ctypes.POINTER(i32)]
    L.fsdp_peer_set_sources.argtypes = [vp, vp, vp]
    L.fsdp_destroy_peer_plan.argtypes = [vp]
    L.fsdp_destroy_peer_plan.restype = None
    L.fsdp_peer_copy_in.argtypes = [vp, vp, vp, vp]
    L.fsdp_peer_copy_out.argtypes = [vp, vp, vp]
    L.fsdp_peer_rs_reduce.argtypes = [vp, i32, vp, vp]
    L.fsdp_peer_adamw_step.argtypes = [vp, vp, vp, vp, vp, ctypes.POINTER(AdamWHparams), vp]
    L.fsdp_peer_rs_adamw_step.argtypes = [vp, i32, vp, vp, vp, ctypes.POINTER(AdamWHparams),
                                          vp, vp, vp]
    L.fsdp_peer_set_fp8_sources.argtypes = [vp, vp, vp]
    L.fsdp_peer_copy_in_fp8_scaled.argtypes = [vp, vp, vp, vp, vp]
    L.fsdp_peer_copy_out_fp8.argtypes = [vp, vp, vp]
    L.fsdp_peer_rs_adamw_step_fp8.argtypes = [vp, i32, vp, vp, vp, ctypes.POINTER(AdamWHparams),
                                              vp, vp, vp, vp, vp]
    L.fsdp_peer_fp8_scales.argtypes = [vp, vp, vp]
    for name in ("fsdp_peer_set_fp8_sources", "fsdp_peer_copy_in_fp8_scaled",
                 "fsdp_peer_copy_out_fp8", "fsdp_peer_rs_adamw_step_fp8", "fsdp_peer_fp8_scales"):
        getattr(L, name).restype = ctypes.c_int
    L.fsdp_ipc_alloc.argtypes = [i64, ctypes.POINTER(vp), ctypes.POINTER(IpcHandle)]
    L.fsdp_ipc_free.argtypes = [vp]
    L.fsdp_ipc_open.argtypes = [ctypes.POINTER(IpcHandle), ctypes.POINTER(vp)]
    L.fsdp_ipc_close.argtypes = [vp]
    for name in ("fsdp_peer_plan", "fsdp_peer_local_ranks", "fsdp_peer_set_sources",
                 "fsdp_peer_copy_in", "fsdp_peer_copy_out", "fsdp_peer_rs_reduce",
                 "fsdp_peer_adamw_step", "fsdp_peer_rs_adamw_step", "fsdp_ipc_alloc",
                 "fsdp_ipc_free", "fsdp_ipc_open", "fsdp_ipc_close"):
        getattr(L, name).restype = ctypes.c_int
    L.fsdp_status_string.argtypes = [ctypes.c_int]
    L.fsdp_status_string.restype = ctypes.c_char_p
    for name in ("fsdp_plan_group", "fsdp_group_sizes", "fsdp_group_param_offsets",
                 "fsdp_shard_params", "fsdp_copy_in", "fsdp_copy_out", "fsdp_rs_reduce",
                 "fsdp_adamw_step", "fsdp_last_cuda_error", "fsdp_abi_version"):
        getattr(L, name).restype = ctypes.c_int
    return L


_lib = _load()


def lib() -> ctypes.CDLL:
    return _lib


def _check(status: int, where: str) -> None:
    if status != FSDP_OK:
        raise FsdpError(status, where)


def _descs(shapes):
    shapes = [tuple(int(d) for d in s) for s in shapes]
    arr = (ParamDesc * max(1, len(shapes)))()
    for i, s in enumerate(shapes):
        if len(s) > FSDP_MAX_NDIM:
            raise ValueError(f"parameter {i}: more than {FSDP_MAX_NDIM} dims")
        arr[i].ndim = len(s)
        for k, d in enumerate(s):
            arr[i].shape[k] = d
    return shapes, arr


class Group:
    """A plan of one parameter group (one fully_shard call) over N ranks."""

    def __init__(self, shapes: Sequence[Sequence[int]], world_size: int, host_only: bool = False):
        shapes, arr = _descs(shapes)
        h = ctypes.c_void_p()
        fn = _lib.fsdp_plan_group_host if host_only else _lib.fsdp_plan_group
        _check(fn(arr, len(shapes), int(world_size), ctypes.byref(h)),
               "fsdp_plan_group_host" if host_only else "fsdp_plan_group")
        self._h = h
        self.shapes = shapes
        self.N = int(world_size)
        self.n = len(shapes)
        S, P, A = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int64()
        _check(_lib.fsdp_group_sizes(h, ctypes.byref(S), ctypes.byref(P), ctypes.byref(A)),
               "fsdp_group_sizes")
        self.S, self.P, self.P_arena = S.value, P.value, A.value
        n = max(1, self.n)
        off, arena, rows = (ctypes.c_int64 * n)(), (ctypes.c_int64 * n)(), (ctypes.c_int64 * n)()
        _check(_lib.fsdp_group_param_offsets(h, off, arena, rows), "fsdp_group_param_offsets")
        self.shard_off = list(off)[:self.n]
        self.arena_off = list(arena)[:self.n]
        self.chunk_rows = list(rows)[:self.n]
        self.numel = [int(torch.Size(s).numel()) if len(s) else 1 for s in shapes]

    @property
    def handle(self) -> ctypes.c_void_p:
        if self._h is None:
            raise ValueError("group destroyed")
        return self._h

    def destroy(self) -> None:
        if getattr(self, "_h", None) is not None:
            _lib.fsdp_destroy_group(self._h)
            self._h = None

    def __del__(self):
        try:
            self.destroy()
        except Exception:
            pass


def fsdp_plan_group(shapes: Sequence[Sequence[int]], world_size: int) -> Group:
    return Group(shapes, world_size)


def fsdp_plan_group_host(shapes: Sequence[Sequence[int]], world_size: int) -> Group:
    """The same plan on the host only (no CUDA call): for inspection and
    fsdp_group_check; data calls refuse it."""
    return Group(shapes, world_size, host_only=True)


def fsdp_group_check(g: Group) -> int:
    """Number of failed consistency checks of the plan's work tables (0 expected)."""
    v = ctypes.c_int64()
    _check(_lib.fsdp_group_check(g.handle, ctypes.byref(v)), "fsdp_group_check")
    return v.value


def fsdp_group_flat(g: Group) -> tuple:
    """(flat, flat_copy_out, mixed shard-side vectors, mixed arena-side
    vectors) of a plan: whether its fused reduce-scatter and fused update take
    the flat path, whether its copy-out does, and how many vectors of each
    side go element by element."""
    f = ctypes.c_int32()
    ms = ctypes.c_int64()
    ma = ctypes.c_int64()
    _check(_lib.fsdp_group_flat(g.handle, ctypes.byref(f), ctypes.byref(ms), ctypes.byref(ma)),
           "fsdp_group_flat")
    return bool(f.value & 1), bool(f.value & 2), ms.value, ma.value


def _stream(stream, t: torch.Tensor):
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream(t.device).cuda_stream)
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _ptr(t: Optional[torch.Tensor], dtypes, numel: int, name: str):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: expected a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name}: must be a CUDA tensor")
    if t.dtype not in dtypes:
        raise TypeError(f"{name}: dtype {t.dtype} not in {dtypes}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")
    if t.numel() < numel:
        raise ValueError(f"{name}: {t.numel()} elements < required {numel}")
    return ctypes.c_void_p(t.data_ptr())


_F32 = (torch.float32,)
_B16 = (torch.bfloat16, torch.int16, torch.uint16)
_U8 = (torch.uint8, torch.int8, torch.float8_e4m3fn)


def fsdp_shard_params(g: Group, full_arena: torch.Tensor, master: torch.Tensor, stream=None):
    _check(_lib.fsdp_shard_params(g.handle, _ptr(full_arena, _F32, g.P_arena, "full_arena"),
                                  _ptr(master, _F32, g.N * g.S, "master"),
                                  _stream(stream, master)), "fsdp_shard_params")


def fsdp_copy_in(g: Group, master: torch.Tensor, ag: torch.Tensor, stream=None):
    _check(_lib.fsdp_copy_in(g.handle, _ptr(master, _F32, g.N * g.S, "master"),
                             _ptr(ag, _B16, g.N * g.S, "ag"), _stream(stream, master)),
           "fsdp_copy_in")


def fsdp_copy_out(g: Group, ag: torch.Tensor, arena: torch.Tensor, stream=None):
    _check(_lib.fsdp_copy_out(g.handle, _ptr(ag, _B16, g.N * g.S, "ag"),
                              _ptr(arena, _B16, g.P_arena, "arena"), _stream(stream, ag)),
           "fsdp_copy_out")


def fsdp_rs_reduce(g: Group, grads: torch.Tensor, op: int, reduced: torch.Tensor,
                   packed: Optional[torch.Tensor] = None, stream=None):
    _check(_lib.fsdp_rs_reduce(g.handle, _ptr(grads, _B16, g.N * g.P_arena, "grads"), int(op),
                               _ptr(packed, _F32, g.N * g.N * g.S, "packed"),
                               _ptr(reduced, _F32, g.N * g.S, "reduced"),
                               _stream(stream, reduced)), "fsdp_rs_reduce")


def fsdp_adamw_step(g: Group, master: torch.Tensor, m: torch.Tensor, v: torch.Tensor,
                    grad: torch.Tensor, *, lr: float, beta1: float, beta2: float, eps: float,
                    weight_decay: float, step: int, stream=None):
    hp = AdamWHparams(float(lr), float(beta1), float(beta2), float(eps), float(weight_decay),
                      int(step))
    n = g.N * g.S
    _check(_lib.fsdp_adamw_step(g.handle, _ptr(master, _F32, n, "master"),
                                _ptr(m, _F32, n, "m"), _ptr(v, _F32, n, "v"),
                                _ptr(grad, _F32, n, "grad"), ctypes.byref(hp),
                                _stream(stream, master)), "fsdp_adamw_step")



def fsdp_rs_adamw_step(g: Group, grads: torch.Tensor, op: int, master: torch.Tensor,
                       m: torch.Tensor, v: torch.Tensor, *, lr: float, beta1: float,
                       beta2: float, eps: float, weight_decay: float, step: int,
                       ag_next: Optional[torch.Tensor] = None,
                       reduced: Optional[torch.Tensor] = None, stream=None):
    hp = AdamWHparams(float(lr), float(beta1), float(beta2), float(eps), float(weight_decay),
                      int(step))
    n = g.N * g.S
    _check(_lib.fsdp_rs_adamw_step(g.handle, _ptr(grads, _B16, g.N * g.P_arena, "grads"),
                                   int(op), _ptr(master, _F32, n, "master"),
                                   _ptr(m, _F32, n, "m"), _ptr(v, _F32, n, "v"),
                                   ctypes.byref(hp), _ptr(ag_next, _B16, n, "ag_next"),
                                   _ptr(reduced, _F32, n, "reduced"),
                                   _stream(stream, master)), "fsdp_rs_adamw_step")


FSDP_SMALL_STEP_ELEMS = 8192


def fsdp_group_step(g: Group, master: torch.Tensor, m: torch.Tensor, v: torch.Tensor,
                    grads: torch.Tensor, op: int, *, lr: float, beta1: float, beta2: float,
                    eps: float, weight_decay: float, step: int, ag: torch.Tensor,
                    arena: torch.Tensor, reduced: torch.Tensor, stream=None):
    """The whole step of one group (copy-in, copy-out, reduce-scatter,
    AdamW); one launch for groups of at most FSDP_SMALL_STEP_ELEMS padded
    elements."""
    hp = AdamWHparams(float(lr), float(beta1), float(beta2), float(eps), float(weight_decay),
                      int(step))
    n = g.N * g.S
    _check(_lib.fsdp_group_step(g.handle, _ptr(master, _F32, n, "master"), _ptr(m, _F32, n, "m"),
                                _ptr(v, _F32, n, "v"),
                                _ptr(grads, _B16, g.N * g.P_arena, "grads"), int(op),
                                ctypes.byref(hp), _ptr(ag, _B16, n, "ag"),
                                _ptr(arena, _B16, g.P_arena, "arena"),
                                _ptr(reduced, _F32, n, "reduced"), _stream(stream, master)),
           "fsdp_group_step")


def fsdp_group_step_dev(g: Group, master: torch.Tensor, m: torch.Tensor, v: torch.Tensor,
                        grads: torch.Tensor, op: int, ds: "DeviceStep", *, ag: torch.Tensor,
                        arena: torch.Tensor, reduced: torch.Tensor, stream=None):
    n = g.N * g.S
    _check(_lib.fsdp_group_step_dev(g.handle, _ptr(master, _F32, n, "master"),
                                    _ptr(m, _F32, n, "m"), _ptr(v, _F32, n, "v"),
                                    _ptr(grads, _B16, g.N * g.P_arena, "grads"), int(op),
                                    _ptr(ds.scalars, _F32, 8, "scalars"),
                                    _ptr(ag, _B16, n, "ag"), _ptr(arena, _B16, g.P_arena, "arena"),
                                    _ptr(reduced, _F32, n, "reduced"), _stream(stream, master)),
           "fsdp_group_step_dev")


def fsdp_group_step_graph(g: Group, master: torch.Tensor, m: torch.Tensor, v: torch.Tensor,
                          grads: torch.Tensor, op: int, ds: "DeviceStep", *, lr: float,
                          beta1: float, beta2: float, eps: float, weight_decay: float,
                          ag: torch.Tensor, arena: torch.Tensor, reduced: torch.Tensor,
                          stream=None):
    n = g.N * g.S
    hp = AdamWHparams(float(lr), float(beta1), float(beta2), float(eps), float(weight_decay), 0)
    _check(_lib.fsdp_group_step_graph(g.handle, _ptr(master, _F32, n, "master"),
                                      _ptr(m, _F32, n, "m"), _ptr(v, _F32, n, "v"),
                                      _ptr(grads, _B16, g.N * g.P_arena, "grads"), int(op),
                                      ctypes.byref(hp), _ptr(ds.step, (torch.int64,), 1, "step"),
                                      _ptr(ds.scalars, _F32, 8, "scalars"),
                                      _ptr(ag, _B16, n, "ag"),
                                      _ptr(arena, _B16, g.P_arena, "arena"),
                                      _ptr(reduced, _F32, n, "reduced"), _stream(stream, master)),
           "fsdp_group_step_graph")


def fsdp_grad_accumulate(g: Group, grads: torch.Tensor, acc: torch.Tensor, first: bool,
                         stream=None):
    n = g.N * g.P_arena
    _check(_lib.fsdp_grad_accumulate(g.handle, _ptr(grads, _B16, n, "grads"),
                                     _ptr(acc, _F32, n, "acc"), int(bool(first)),
                                     _stream(stream, acc)), "fsdp_grad_accumulate")


def fsdp_rs_reduce_accumulated(g: Group, grads: Optional[torch.Tensor], acc: torch.Tensor,
                               op: int, reduced: torch.Tensor, stream=None):
    n = g.N * g.P_arena
    _check(_lib.fsdp_rs_reduce_accumulated(g.handle, _ptr(grads, _B16, n, "grads"),
                                           _ptr(acc, _F32, n, "acc"), int(op),
                                           _ptr(reduced, _F32, g.N * g.S, "reduced"),
                                           _stream(stream, reduced)),
           "fsdp_rs_reduce_accumulated")


def fsdp_copy_in_f32(g: Group, master: torch.Tensor, ag32: torch.Tensor, stream=None):
    """Copy-in with param_dtype fp32 (test mode: no cast)."""
    n = g.N * g.S
    _check(_lib.fsdp_copy_in_f32(g.handle, _ptr(master, _F32, n, "master"),
                                 _ptr(ag32, _F32, n, "ag32"), _stream(stream, master)),
           "fsdp_copy_in_f32")


def fsdp_copy_out_f32(g: Group, ag32: torch.Tensor, arena32: torch.Tensor, stream=None):
    """Copy-out with param_dtype fp32 (test mode: no cast)."""
    _check(_lib.fsdp_copy_out_f32(g.handle, _ptr(ag32, _F32, g.N * g.S, "ag32"),
                                  _ptr(arena32, _F32, g.P_arena, "arena32"),
                                  _stream(stream, ag32)), "fsdp_copy_out_f32")


def fsdp_copy_in_fp8(g: Group, master: torch.Tensor, ag8: torch.Tensor, scales: torch.Tensor,
                     stream=None):
    _check(_lib.fsdp_copy_in_fp8(g.handle, _ptr(master, _F32, g.N * g.S, "master"),
                                 _ptr(ag8, _U8, g.N * g.S, "ag8"),
                                 _ptr(scales, _F32, g.n, "scales"), _stream(stream, master)),
           "fsdp_copy_in_fp8")


def fsdp_copy_in_fp8_scaled(g: Group, master: torch.Tensor, scales: torch.Tensor,
                            ag8: torch.Tensor, stream=None):
    _check(_lib.fsdp_copy_in_fp8_scaled(g.handle, _ptr(master, _F32, g.N * g.S, "master"),
                                        _ptr(scales, _F32, g.n, "scales"),
                                        _ptr(ag8, _U8, g.N * g.S, "ag8"),
                                        _stream(stream, master)), "fsdp_copy_in_fp8_scaled")


def fsdp_rs_adamw_step_fp8(g: Group, grads: torch.Tensor, op: int, master: torch.Tensor,
                           m: torch.Tensor, v: torch.Tensor, *, lr: float, beta1: float,
                           beta2: float, eps: float, weight_decay: float, step: int,
                           scales_prev: torch.Tensor, ag8_next: torch.Tensor,
                           scales_next: torch.Tensor, reduced: Optional[torch.Tensor] = None,
                           stream=None):
    hp = AdamWHparams(float(lr), float(beta1), float(beta2), float(eps), float(weight_decay),
                      int(step))
    n = g.N * g.S
    _check(_lib.fsdp_rs_adamw_step_fp8(g.handle, _ptr(grads, _B16, g.N * g.P_arena, "grads"),
                                       int(op), _ptr(master, _F32, n, "master"),
                                       _ptr(m, _F32, n, "m"), _ptr(v, _F32, n, "v"),
                                       ctypes.byref(hp),
                                       _ptr(scales_prev, _F32, g.n, "scales_prev"),
                                       _ptr(ag8_next, _U8, n, "ag8_next"),
                                       _ptr(scales_next, _F32, g.n, "scales_next"),
                                       _ptr(reduced, _F32, n, "reduced"),
                                       _stream(stream, master)), "fsdp_rs_adamw_step_fp8")


def fsdp_copy_out_fp8(g: Group, ag8: torch.Tensor, arena8: torch.Tensor, stream=None):
    _check(_lib.fsdp_copy_out_fp8(g.handle, _ptr(ag8, _U8, g.N * g.S, "ag8"),
                                  _ptr(arena8, _U8, g.P_arena, "arena8"), _stream(stream, ag8)),
           "fsdp_copy_out_fp8")


class DeviceStep:
    """A device step counter and that step's AdamW scalars (for CUDA graphs)."""

    def __init__(self, device=None):
        self.step = torch.zeros(1, dtype=torch.int64, device=device or "cuda")
        self.scalars = torch.zeros(8, dtype=torch.float32, device=device or "cuda")


def fsdp_adamw_prepare(ds: DeviceStep, *, lr: float, beta1: float, beta2: float, eps: float,
                       weight_decay: float, stream=None):
    hp = AdamWHparams(float(lr), float(beta1), float(beta2), float(eps), float(weight_decay), 0)
    _check(_lib.fsdp_adamw_prepare(ctypes.byref(hp), _ptr(ds.step, (torch.int64,), 1, "step"),
                                   _ptr(ds.scalars, _F32, 8, "scalars"),
                                   _stream(stream, ds.scalars)), "fsdp_adamw_prepare")


def fsdp_adamw_step_dev(g: Group, master: torch.Tensor, m: torch.Tensor, v: torch.Tensor,
                        grad: torch.Tensor, ds: DeviceStep, stream=None):
    n = g.N * g.S
    _check(_lib.fsdp_adamw_step_dev(g.handle, _ptr(master, _F32, n, "master"),
                                    _ptr(m, _F32, n, "m"), _ptr(v, _F32, n, "v"),
                                    _ptr(grad, _F32, n, "grad"),
                                    _ptr(ds.scalars, _F32, 8, "scalars"),
                                    _stream(stream, master)), "fsdp_adamw_step_dev")


def fsdp_rs_adamw_step_dev(g: Group, grads: torch.Tensor, op: int, master: torch.Tensor,
                           m: torch.Tensor, v: torch.Tensor, ds: DeviceStep, *,
                           ag_next: Optional[torch.Tensor] = None,
                           reduced: Optional[torch.Tensor] = None, stream=None):
    n = g.N * g.S
    _check(_lib.fsdp_rs_adamw_step_dev(g.handle, _ptr(grads, _B16, g.N * g.P_arena, "grads"),
                                       int(op), _ptr(master, _F32, n, "master"),
                                       _ptr(m, _F32, n, "m"), _ptr(v, _F32, n, "v"),
                                       _ptr(ds.scalars, _F32, 8, "scalars"),
                                       _ptr(ag_next, _B16, n, "ag_next"),
                                       _ptr(reduced, _F32, n, "reduced"),
                                       _stream(stream, master)), "fsdp_rs_adamw_step_dev")

def fsdp_debug_build() -> bool:
    return bool(_lib.fsdp_debug_build())


def fsdp_debug_set_error_words(words: Optional[torch.Tensor], shrink: int = 0) -> None:
    """Debug build: record violations in `words` (int32 [4] on the device of
    the launches that follow; None stops recording)."""
    ptr = None if words is None else _ptr(words, (torch.int32,), 4, "words")
    _check(_lib.fsdp_debug_set_error_words(ptr, int(shrink)), "fsdp_debug_set_error_words")


FSDP_NOALLOC_MAX_UNITS = 131072


def group_layout(shapes: Sequence[Sequence[int]], world_size: int) -> tuple:
    """(S, P, P_arena) of a group from its shapes alone, by the layout rules
    of include/fsdpk.h: c_i = ceil(d0_i / N) chunk rows (torch.chunk along
    dim 0), S = sum c_i * cols_i, and each parameter's arena start rounded up
    to 8 elements.  Size checks only; the library derives the same values."""
    N = int(world_size)
    if N < 1:
        raise ValueError("world_size must be >= 1")
    S = P = A = 0
    for s in shapes:
        s = tuple(int(d) for d in s)
        if any(d < 0 for d in s):
            raise ValueError(f"negative dimension in {s}")
        d0 = s[0] if s else 1
        cols = 1
        for d in s[1:]:
            cols *= d
        c = -(-d0 // N)
        S += c * cols
        P += d0 * cols
        A = (A + 7) // 8 * 8 + d0 * cols
    return S, P, (A + 7) // 8 * 8


def fsdp_rs_reduce_noalloc(shapes: Sequence[Sequence[int]], world_size: int,
                           grads: torch.Tensor, op: int, reduced: torch.Tensor,
                           *, P_arena: Optional[int] = None, S: Optional[int] = None,
                           stream=None):
    """The fused reduce-scatter without any allocation (no plan object): for
    callers that cannot allocate device memory.  The tensors are size-checked
    against S and P_arena worked out here from the shapes (the C call cannot
    see buffer sizes); P_arena / S, when given, must agree with them."""
    N = int(world_size)
    shapes = [tuple(int(d) for d in s) for s in shapes]
    S_, _, A_ = group_layout(shapes, N)
    if S is not None and int(S) != S_:
        raise ValueError(f"S={S} does not match the shapes' layout (S={S_})")
    if P_arena is not None and int(P_arena) != A_:
        raise ValueError(f"P_arena={P_arena} does not match the shapes' layout (P_arena={A_})")
    shapes, arr = _descs(shapes)
    _check(_lib.fsdp_rs_reduce_noalloc(arr, len(shapes), N,
                                       _ptr(grads, _B16, N * A_, "grads"), int(op),
                                       _ptr(reduced, _F32, N * S_, "reduced"),
                                       _stream(stream, reduced)), "fsdp_rs_reduce_noalloc")


# ---------------------------------------------------------------------------
# several devices: per-rank pointer tables and CUDA IPC
# ---------------------------------------------------------------------------
class PeerPlan:
    """Device `index` of `n_devices` of a group: its local virtual ranks
    [r0, r0 + L) and the per-rank pointer tables of the exchange steps."""

    def __init__(self, group: Group, n_devices: int, index: int):
        h = ctypes.c_void_p()
        _check(_lib.fsdp_peer_plan(group.handle, int(n_devices), int(index), ctypes.byref(h)),
               "fsdp_peer_plan")
        self._h = h
        self.group = group  # the group must outlive the peer plan
        self.n_devices, self.index = int(n_devices), int(index)
        L, r0 = ctypes.c_int32(), ctypes.c_int32()
        _check(_lib.fsdp_peer_local_ranks(h, ctypes.byref(L), ctypes.byref(r0)),
               "fsdp_peer_local_ranks")
        self.L, self.r0 = L.value, r0.value
        self.N, self.S, self.P, self.P_arena, self.n = (group.N, group.S, group.P,
                                                        group.P_arena, group.n)

    @property
    def handle(self) -> ctypes.c_void_p:
        if self._h is None:
            raise ValueError("peer plan destroyed")
        return self._h

    def destroy(self) -> None:
        if getattr(self, "_h", None) is not None:
            _lib.fsdp_destroy_peer_plan(self._h)
            self._h = None

    def __del__(self):
        try:
            self.destroy()
        except Exception:
            pass


def fsdp_peer_plan(group: Group, n_devices: int, index: int) -> PeerPlan:
    return PeerPlan(group, n_devices, index)


def fsdp_peer_set_sources(pp: PeerPlan, ag_rank_ptrs: Optional[Sequence[int]],
                          grad_rank_ptrs: Optional[Sequence[int]]):
    def table(ptrs):
        if ptrs is None:
            return None
        if len(ptrs) != pp.N:
            raise ValueError(f"{len(ptrs)} pointers for {pp.N} ranks")
        return (ctypes.c_void_p * pp.N)(*[int(x) for x in ptrs])
    _check(_lib.fsdp_peer_set_sources(pp.handle, table(ag_rank_ptrs), table(grad_rank_ptrs)),
           "fsdp_peer_set_sources")


def fsdp_peer_copy_in(pp: PeerPlan, master: torch.Tensor, ag_slot: torch.Tensor, stream=None):
    n = pp.L * pp.S
    _check(_lib.fsdp_peer_copy_in(pp.handle, _ptr(master, _F32, n, "master"),
                                  _ptr(ag_slot, _B16, n, "ag_slot"), _stream(stream, master)),
           "fsdp_peer_copy_in")


def fsdp_peer_copy_out(pp: PeerPlan, arena: torch.Tensor, stream=None):
    _check(_lib.fsdp_peer_copy_out(pp.handle, _ptr(arena, _B16, pp.P_arena, "arena"),
                                   _stream(stream, arena)), "fsdp_peer_copy_out")


def fsdp_peer_rs_reduce(pp: PeerPlan, op: int, reduced: torch.Tensor, stream=None):
    _check(_lib.fsdp_peer_rs_reduce(pp.handle, int(op),
                                    _ptr(reduced, _F32, pp.L * pp.S, "reduced"),
                                    _stream(stream, reduced)), "fsdp_peer_rs_reduce")


def fsdp_peer_adamw_step(pp: PeerPlan, master: torch.Tensor, m: torch.Tensor, v: torch.Tensor,
                         grad: torch.Tensor, *, lr: float, beta1: float, beta2: float,
                         eps: float, weight_decay: float, step: int, stream=None):
    hp = AdamWHparams(float(lr), float(beta1), float(beta2), float(eps), float(weight_decay),
                      int(step))
    n = pp.L * pp.S
    _check(_lib.fsdp_peer_adamw_step(pp.handle, _ptr(master, _F32, n, "master"),
                                     _ptr(m, _F32, n, "m"), _ptr(v, _F32, n, "v"),
                                     _ptr(grad, _F32, n, "grad"), ctypes.byref(hp),
                                     _stream(stream, master)), "fsdp_peer_adamw_step")


def fsdp_peer_rs_adamw_step(pp: PeerPlan, op: int, master: torch.Tensor, m: torch.Tensor,
                            v: torch.Tensor, *, lr: float, beta1: float, beta2: float,
                            eps: float, weight_decay: float, step: int,
                            ag_next: Optional[torch.Tensor] = None,
                            reduced: Optional[torch.Tensor] = None, stream=None):
    hp = AdamWHparams(float(lr), float(beta1), float(beta2), float(eps), float(weight_decay),
                      int(step))
    n = pp.L * pp.S
    _check(_lib.fsdp_peer_rs_adamw_step(pp.handle, int(op), _ptr(master, _F32, n, "master"),
                                        _ptr(m, _F32, n, "m"), _ptr(v, _F32, n, "v"),
                                        ctypes.byref(hp), _ptr(ag_next, _B16, n, "ag_next"),
                                        _ptr(reduced, _F32, n, "reduced"),
                                        _stream(stream, master)), "fsdp_peer_rs_adamw_step")


def fsdp_peer_set_fp8_sources(pp: PeerPlan, ag8_rank_ptrs: Sequence[int],
                              amax_device_ptrs: Sequence[int]):
    if len(ag8_rank_ptrs) != pp.N or len(amax_device_ptrs) != pp.n_devices:
        raise ValueError("one slot row per rank and one amax array per device")
    ag = (ctypes.c_void_p * pp.N)(*[int(x) for x in ag8_rank_ptrs])
    am = (ctypes.c_void_p * pp.n_devices)(*[int(x) for x in amax_device_ptrs])
    _check(_lib.fsdp_peer_set_fp8_sources(pp.handle, ag, am), "fsdp_peer_set_fp8_sources")


def fsdp_peer_copy_in_fp8_scaled(pp: PeerPlan, master: torch.Tensor, scales: torch.Tensor,
                                 ag8_slot: torch.Tensor, stream=None):
    n = pp.L * pp.S
    _check(_lib.fsdp_peer_copy_in_fp8_scaled(pp.handle, _ptr(master, _F32, n, "master"),
                                             _ptr(scales, _F32, pp.n, "scales"),
                                             _ptr(ag8_slot, _U8, n, "ag8_slot"),
                                             _stream(stream, master)),
           "fsdp_peer_copy_in_fp8_scaled")


def fsdp_peer_copy_out_fp8(pp: PeerPlan, arena8: torch.Tensor, stream=None):
    _check(_lib.fsdp_peer_copy_out_fp8(pp.handle, _ptr(arena8, _U8, pp.P_arena, "arena8"),
                                       _stream(stream, arena8)), "fsdp_peer_copy_out_fp8")


_U32 = (torch.int32, torch.uint32)


def fsdp_peer_rs_adamw_step_fp8(pp: PeerPlan, op: int, master: torch.Tensor, m: torch.Tensor,
                                v: torch.Tensor, *, lr: float, beta1: float, beta2: float,
                                eps: float, weight_decay: float, step: int,
                                scales_prev: torch.Tensor, ag8_next: torch.Tensor,
                                amax_local: torch.Tensor, reduced: Optional[torch.Tensor] = None,
                                stream=None):
    hp = AdamWHparams(float(lr), float(beta1), float(beta2), float(eps), float(weight_decay),
                      int(step))
    n = pp.L * pp.S
    _check(_lib.fsdp_peer_rs_adamw_step_fp8(pp.handle, int(op), _ptr(master, _F32, n, "master"),
                                            _ptr(m, _F32, n, "m"), _ptr(v, _F32, n, "v"),
                                            ctypes.byref(hp),
                                            _ptr(scales_prev, _F32, pp.n, "scales_prev"),
                                            _ptr(ag8_next, _U8, n, "ag8_next"),
                                            _ptr(amax_local, _U32, pp.n, "amax_local"),
                                            _ptr(reduced, _F32, n, "reduced"),
                                            _stream(stream, master)), "fsdp_peer_rs_adamw_step_fp8")


def fsdp_peer_fp8_scales(pp: PeerPlan, scales_next: torch.Tensor, stream=None):
    _check(_lib.fsdp_peer_fp8_scales(pp.handle, _ptr(scales_next, _F32, pp.n, "scales_next"),
                                     _stream(stream, scales_next)), "fsdp_peer_fp8_scales")


def fsdp_ipc_alloc(nbytes: int):
    """Device memory another process can map: returns (pointer, 64-byte handle)."""
    ptr, h = ctypes.c_void_p(), IpcHandle()
    _check(_lib.fsdp_ipc_alloc(int(nbytes), ctypes.byref(ptr), ctypes.byref(h)),
           "fsdp_ipc_alloc")
    return int(ptr.value), bytes(h.bytes)


def fsdp_ipc_free(ptr: int):
    _check(_lib.fsdp_ipc_free(ctypes.c_void_p(int(ptr))), "fsdp_ipc_free")


def fsdp_ipc_open(handle: bytes) -> int:
    if len(handle) != 64:
        raise ValueError("an IPC handle has 64 bytes")
    h = IpcHandle()
    ctypes.memmove(h.bytes, handle, 64)
    ptr = ctypes.c_void_p()
    _check(_lib.fsdp_ipc_open(ctypes.byref(h), ctypes.byref(ptr)), "fsdp_ipc_open")
    return int(ptr.value)


def fsdp_ipc_close(ptr: int):
    _check(_lib.fsdp_ipc_close(ctypes.c_void_p(int(ptr))), "fsdp_ipc_close")


class _DeviceSpan:
    def __init__(self, ptr: int, nbytes: int):
        self.__cuda_array_interface__ = {"shape": (int(nbytes),), "typestr": "|u1",
                                         "data": (int(ptr), False), "version": 3}


def device_tensor(ptr: int, numel: int, dtype: torch.dtype, device) -> torch.Tensor:
    """A tensor view of `numel` elements of device memory this binding does
    not own (e.g. from fsdp_ipc_alloc); the memory must outlive the tensor."""
    esize = torch.empty(0, dtype=dtype).element_size()
    if numel == 0:
        return torch.empty(0, dtype=dtype, device=device)
    raw = torch.as_tensor(_DeviceSpan(ptr, numel * esize), device=device)
    return raw.view(dtype)
