"""CPU oracle for the FSDP2 per-parameter sharding step -- test infrastructure.

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its binding) never does: nothing here is a fallback.

The arithmetic lives in ``fsdp_oracle.c`` (plain C, built with gcc at
``-O2 -ffp-contract=off``, no fast-math, optional OpenMP over outer loops).
This module only builds and loads it and marshals numpy arrays.

Every function follows a definition from the pages (see the C file's header):

* ``plan``        -- torch.chunk rows ``c_i = ceil(d0_i / N)``, padded shards
  ("Sharded Training: FSDP2, DTensor, Tensor and Pipeline Parallelism",
  fully_shard paragraph);
* ``shard``       -- Shard(0) placement with trailing zero pad rows;
* ``cast_bf16``   -- binary32 -> bfloat16 round-to-nearest-even;
* ``copy_in``     -- padded fp32 shard -> bf16 slot of the rank-major buffer;
* ``copy_out``    -- rank-major buffer -> unsharded views, padding stripped;
* ``pack``        -- per-rank bf16 gradients -> fp32 reduce-scatter input;
* ``reduce_packed`` -- rank-ordered binary32 fold, SUM / AVG / SUM_THEN_DIV;
* ``reduce_scatter_direct`` -- pack + fold from the per-rank gradients with no
  packed intermediate (same definitions, for full-size groups);
* ``accumulate``  -- gradient accumulation without sync, fp32 left fold;
* ``reduce_scatter_f32`` -- reduce-scatter of fp32 (accumulated) arenas;
* ``e4m3_bits``, ``fp8_scales``, ``copy_in_fp8``, ``copy_out_fp8`` -- the FP8
  (E4M3, per-parameter tensorwise scale) all-gather copy-in and copy-out;
* ``adamw``       -- decoupled-weight-decay AdamW in binary64.

Parity status: every function above is pinned by tests under ``tests/``
(``test_oracle_*.py``) against torch library routines, closed forms, the
pages' worked shapes and brute force.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fsdp_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

SUM, AVG, SUM_THEN_DIV = 0, 1, 2

_i64p = ctypes.POINTER(ctypes.c_int64)


def build(force: bool = False) -> str:
    """Compile ``fsdp_oracle.c`` into ``liboracle.so`` next to it."""
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
        return _LIB
    cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
           "-fopenmp", "-fPIC", "-shared", "-Wall", "-Wextra", "-o", _LIB, _SRC,
           "-lm"]
    subprocess.run(cmd, check=True)
    return _LIB


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        vp = ctypes.c_void_p
        i32, i64, f64 = ctypes.c_int32, ctypes.c_int64, ctypes.c_double
        L.or_set_threads.argtypes = [ctypes.c_int]
        L.or_get_threads.restype = ctypes.c_int
        L.or_chunk_rows.argtypes = [i64, i32]
        L.or_chunk_rows.restype = i64
        L.or_valid_rows.argtypes = [i64, i32, i32]
        L.or_valid_rows.restype = i64
        L.or_plan.argtypes = [vp, vp, i32, i32, vp, vp, vp, vp, vp]
        L.or_bf16_rne_bits.argtypes = [ctypes.c_uint32]
        L.or_bf16_rne_bits.restype = ctypes.c_uint16
        L.or_cast_bf16.argtypes = [vp, vp, i64]
        L.or_cast_bf16_bits.argtypes = [vp, vp, i64]
        for name in ("or_shard", "or_copy_in", "or_copy_out", "or_pack"):
            getattr(L, name).argtypes = [vp, vp, i32, i32, vp, vp]
        L.or_reduce_packed.argtypes = [i32, i64, vp, i32, vp]
        L.or_reduce_scatter_direct.argtypes = [vp, vp, i32, i32, vp, i32, vp]
        L.or_accumulate.argtypes = [vp, vp, i64, i32]
        L.or_e4m3_bits.argtypes = [ctypes.c_float]
        L.or_e4m3_bits.restype = ctypes.c_uint8
        L.or_fp8_scale.argtypes = [ctypes.c_float]
        L.or_fp8_scale.restype = ctypes.c_float
        L.or_fp8_quant_input.argtypes = [ctypes.c_float, ctypes.c_float]
        L.or_fp8_quant_input.restype = ctypes.c_float
        L.or_cast_e4m3.argtypes = [vp, vp, i64]
        L.or_fp8_scales.argtypes = [vp, vp, i32, i32, vp, vp]
        L.or_copy_in_fp8.argtypes = [vp, vp, i32, i32, vp, vp, vp]
        L.or_copy_out_fp8.argtypes = [vp, vp, i32, i32, vp, vp]
        L.or_reduce_scatter_f32.argtypes = [vp, vp, i32, i32, vp, i32, vp]
        L.or_adamw.argtypes = [vp, vp, vp, vp, i64, f64, f64, f64, f64, f64, i64]
        _lib = L
    return _lib


def set_threads(t: int) -> None:
    lib().or_set_threads(int(t))


def get_threads() -> int:
    return int(lib().or_get_threads())


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data


@dataclass
class Plan:
    """Per-group layout computed by the oracle from (shapes, N)."""
    N: int
    d0: np.ndarray      # int64 [n]
    cols: np.ndarray    # int64 [n]
    chunk_rows: np.ndarray
    shard_size: np.ndarray
    shard_off: np.ndarray
    arena_off: np.ndarray
    S: int
    P: int
    P_arena: int

    @property
    def n(self) -> int:
        return int(self.d0.shape[0])

    def valid_rows(self, i: int, r: int) -> int:
        return int(lib().or_valid_rows(int(self.d0[i]), self.N, r))


def shapes_to_rows_cols(shapes):
    d0 = np.array([int(s[0]) if len(s) else 1 for s in shapes], dtype=np.int64)
    cols = np.array([int(np.prod(s[1:], dtype=np.int64)) if len(s) > 1 else 1
                     for s in shapes], dtype=np.int64)
    return d0, cols


def plan(shapes, N: int) -> Plan:
    d0, cols = shapes_to_rows_cols(shapes)
    n = d0.shape[0]
    c = np.zeros(max(n, 1), np.int64)
    s = np.zeros(max(n, 1), np.int64)
    off = np.zeros(max(n, 1), np.int64)
    u = np.zeros(max(n, 1), np.int64)
    sizes = np.zeros(3, np.int64)
    lib().or_plan(_ptr(d0), _ptr(cols), n, N, _ptr(c), _ptr(s), _ptr(off),
                  _ptr(u), _ptr(sizes))
    return Plan(N, d0, cols, c[:n], s[:n], off[:n], u[:n],
                int(sizes[0]), int(sizes[1]), int(sizes[2]))


def chunk_rows(d0: int, N: int) -> int:
    return int(lib().or_chunk_rows(d0, N))


def valid_rows(d0: int, N: int, r: int) -> int:
    return int(lib().or_valid_rows(d0, N, r))


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """binary32 array -> bfloat16 bit patterns (uint16), RNE."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    y = np.empty(x.shape, np.uint16)
    lib().or_cast_bf16(_ptr(x), _ptr(y), x.size)
    return y


def bf16_bits_from_u32(bits: np.ndarray) -> np.ndarray:
    bits = np.ascontiguousarray(bits, dtype=np.uint32)
    y = np.empty(bits.shape, np.uint16)
    lib().or_cast_bf16_bits(_ptr(bits), _ptr(y), bits.size)
    return y


def bf16_to_f32(h: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(h, np.uint16).astype(np.uint32) << 16).view(np.float32)


def shard(p: Plan, full_arena: np.ndarray) -> np.ndarray:
    """fp32 full params in arena layout [P_arena] -> padded master [N][S]."""
    full_arena = np.ascontiguousarray(full_arena, np.float32)
    assert full_arena.size >= p.P_arena
    out = np.empty(p.N * p.S, np.float32)
    lib().or_shard(_ptr(p.d0), _ptr(p.cols), p.n, p.N, _ptr(full_arena), _ptr(out))
    return out


def copy_in(p: Plan, master: np.ndarray) -> np.ndarray:
    master = np.ascontiguousarray(master, np.float32)
    assert master.size == p.N * p.S
    ag = np.empty(p.N * p.S, np.uint16)
    lib().or_copy_in(_ptr(p.d0), _ptr(p.cols), p.n, p.N, _ptr(master), _ptr(ag))
    return ag


def copy_out(p: Plan, ag: np.ndarray, arena: np.ndarray | None = None) -> np.ndarray:
    """Rank-major bf16 buffer -> arena [P_arena]; gaps keep ``arena``'s bytes."""
    ag = np.ascontiguousarray(ag, np.uint16)
    assert ag.size == p.N * p.S
    if arena is None:
        arena = np.zeros(p.P_arena, np.uint16)
    lib().or_copy_out(_ptr(p.d0), _ptr(p.cols), p.n, p.N, _ptr(ag), _ptr(arena))
    return arena


def pack(p: Plan, grads: np.ndarray) -> np.ndarray:
    """[N][P_arena] bf16 per-rank gradients -> [N][N][S] fp32."""
    grads = np.ascontiguousarray(grads, np.uint16)
    assert grads.size == p.N * p.P_arena
    out = np.empty(p.N * p.N * p.S, np.float32)
    lib().or_pack(_ptr(p.d0), _ptr(p.cols), p.n, p.N, _ptr(grads), _ptr(out))
    return out


def reduce_packed(p: Plan, packed: np.ndarray, op: int) -> np.ndarray:
    packed = np.ascontiguousarray(packed, np.float32)
    assert packed.size == p.N * p.N * p.S
    out = np.empty(p.N * p.S, np.float32)
    lib().or_reduce_packed(p.N, p.S, _ptr(packed), int(op), _ptr(out))
    return out


def reduce_scatter(p: Plan, grads: np.ndarray, op: int) -> np.ndarray:
    """pack followed by the rank-ordered reduction."""
    return reduce_packed(p, pack(p, grads), op)


def reduce_scatter_direct(p: Plan, grads: np.ndarray, op: int) -> np.ndarray:
    """The same reduce-scatter straight from the per-rank gradients, without
    the [N][N][S] packed intermediate (for groups too large to pack)."""
    grads = np.ascontiguousarray(grads, np.uint16)
    assert grads.size == p.N * p.P_arena
    out = np.empty(p.N * p.S, np.float32)
    lib().or_reduce_scatter_direct(_ptr(p.d0), _ptr(p.cols), p.n, p.N, _ptr(grads),
                                   int(op), _ptr(out))
    return out


def accumulate(acc: np.ndarray, grads: np.ndarray, first: bool) -> np.ndarray:
    """In place: acc = fp32(grads) (first microbatch) or acc + fp32(grads)."""
    assert acc.dtype == np.float32 and acc.flags["C_CONTIGUOUS"]
    grads = np.ascontiguousarray(grads, np.uint16)
    assert acc.size == grads.size
    lib().or_accumulate(_ptr(acc), _ptr(grads), acc.size, int(bool(first)))
    return acc


def reduce_scatter_f32(p: Plan, src: np.ndarray, op: int) -> np.ndarray:
    """Reduce-scatter of fp32 per-rank arenas [N][P_arena]."""
    src = np.ascontiguousarray(src, np.float32)
    assert src.size == p.N * p.P_arena
    out = np.empty(p.N * p.S, np.float32)
    lib().or_reduce_scatter_f32(_ptr(p.d0), _ptr(p.cols), p.n, p.N, _ptr(src), int(op),
                                _ptr(out))
    return out


def e4m3_bits(x: np.ndarray) -> np.ndarray:
    """binary32 (|x| <= 448 or NaN) -> E4M3 bytes, round to nearest even."""
    x = np.ascontiguousarray(x, np.float32)
    y = np.empty(x.shape, np.uint8)
    lib().or_cast_e4m3(_ptr(x), _ptr(y), x.size)
    return y


def fp8_scales(p: Plan, master: np.ndarray) -> np.ndarray:
    master = np.ascontiguousarray(master, np.float32)
    assert master.size == p.N * p.S
    out = np.empty(max(p.n, 1), np.float32)
    lib().or_fp8_scales(_ptr(p.d0), _ptr(p.cols), p.n, p.N, _ptr(master), _ptr(out))
    return out[:p.n]


def copy_in_fp8(p: Plan, master: np.ndarray, scales: np.ndarray) -> np.ndarray:
    master = np.ascontiguousarray(master, np.float32)
    scales = np.ascontiguousarray(scales, np.float32)
    assert master.size == p.N * p.S and scales.size == p.n
    out = np.empty(p.N * p.S, np.uint8)
    lib().or_copy_in_fp8(_ptr(p.d0), _ptr(p.cols), p.n, p.N, _ptr(master), _ptr(scales),
                         _ptr(out))
    return out


def copy_out_fp8(p: Plan, ag8: np.ndarray, arena8: np.ndarray | None = None) -> np.ndarray:
    ag8 = np.ascontiguousarray(ag8, np.uint8)
    assert ag8.size == p.N * p.S
    if arena8 is None:
        arena8 = np.zeros(p.P_arena, np.uint8)
    lib().or_copy_out_fp8(_ptr(p.d0), _ptr(p.cols), p.n, p.N, _ptr(ag8), _ptr(arena8))
    return arena8


def adamw(master, m, v, grad, *, lr, beta1, beta2, eps, weight_decay, step):
    """In-place AdamW on float32 arrays of equal length."""
    for a in (master, m, v):
        assert a.dtype == np.float32 and a.flags["C_CONTIGUOUS"]
    grad = np.ascontiguousarray(grad, np.float32)
    assert master.size == m.size == v.size == grad.size
    lib().or_adamw(_ptr(master), _ptr(m), _ptr(v), _ptr(grad), master.size,
                   float(lr), float(beta1), float(beta2), float(eps),
                   float(weight_decay), int(step))
