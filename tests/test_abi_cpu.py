"""The C-ABI library without a GPU: it loads, exports every function that
include/fsdpk.h declares, and rejects invalid plans on the host before any
CUDA call."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = []
    for h in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if h.endswith(".h"):
            src = open(os.path.join(ROOT, "include", h)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names += re.findall(r"^[A-Za-z_][\w \t\*]*?\b(fsdp_\w+)\s*\(", src, flags=re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def abi():
    from fully_sharded_shard_b200 import build
    build.build()
    from fully_sharded_shard_b200 import abi as _abi
    return _abi


def test_every_declared_symbol_is_exported(abi):
    names = _declared()
    assert "fsdp_plan_group" in names and "fsdp_rs_reduce" in names
    L = abi.lib()
    for n in names:
        assert hasattr(L, n), f"{n} declared in include/ but not exported"
    assert set(abi.EXPORTED) <= set(names)


def test_version_and_status_strings(abi):
    L = abi.lib()
    assert L.fsdp_abi_version() == 1
    for st in (0, -1, -2, -3, -4, -5):
        assert len(L.fsdp_status_string(st)) > 0
    assert L.fsdp_status_string(99) == b"unknown status"


def test_plan_validation_on_host(abi):
    L = abi.lib()
    h = ctypes.c_void_p()
    one = (abi.ParamDesc * 1)()
    one[0].ndim = 2
    one[0].shape[0], one[0].shape[1] = 4, 4
    assert L.fsdp_plan_group(one, 1, 0, ctypes.byref(h)) == abi.FSDP_EINVAL       # N = 0
    assert L.fsdp_plan_group(one, 1, 2000, ctypes.byref(h)) == abi.FSDP_EINVAL    # N too big
    assert L.fsdp_plan_group(one, 1, 2, None) == abi.FSDP_EINVAL                 # no out
    assert L.fsdp_plan_group(None, 1, 2, ctypes.byref(h)) == abi.FSDP_EINVAL      # no params
    assert L.fsdp_plan_group(one, -1, 2, ctypes.byref(h)) == abi.FSDP_EINVAL      # n < 0
    bad = (abi.ParamDesc * 1)()
    bad[0].ndim = 9
    assert L.fsdp_plan_group(bad, 1, 2, ctypes.byref(h)) == abi.FSDP_EINVAL       # ndim > 8
    bad[0].ndim = 2
    bad[0].shape[0], bad[0].shape[1] = -3, 4
    assert L.fsdp_plan_group(bad, 1, 2, ctypes.byref(h)) == abi.FSDP_EINVAL       # negative dim
    bad[0].shape[0], bad[0].shape[1] = 1 << 40, 1 << 40
    assert L.fsdp_plan_group(bad, 1, 2, ctypes.byref(h)) == abi.FSDP_EINVAL       # int64 overflow
    assert h.value is None


def test_data_calls_reject_null_group(abi):
    L = abi.lib()
    assert L.fsdp_copy_in(None, None, None, None) == abi.FSDP_EINVAL
    assert L.fsdp_copy_out(None, None, None, None) == abi.FSDP_EINVAL
    assert L.fsdp_rs_reduce(None, None, 0, None, None, None) == abi.FSDP_EINVAL
    assert L.fsdp_adamw_step(None, None, None, None, None, None, None) == abi.FSDP_EINVAL
    assert L.fsdp_shard_params(None, None, None, None) == abi.FSDP_EINVAL
    assert L.fsdp_group_sizes(None, None, None, None) == abi.FSDP_EINVAL
    L.fsdp_destroy_group(None)


def test_peer_and_ipc_calls_reject_bad_arguments_on_host(abi):
    L = abi.lib()
    h = ctypes.c_void_p()
    assert L.fsdp_peer_plan(None, 1, 0, ctypes.byref(h)) == abi.FSDP_EINVAL
    assert L.fsdp_peer_plan(None, 1, 0, None) == abi.FSDP_EINVAL
    assert h.value is None
    assert L.fsdp_peer_local_ranks(None, None, None) == abi.FSDP_EINVAL
    assert L.fsdp_peer_set_sources(None, None, None) == abi.FSDP_EINVAL
    assert L.fsdp_peer_copy_in(None, None, None, None) == abi.FSDP_EINVAL
    assert L.fsdp_peer_copy_out(None, None, None) == abi.FSDP_EINVAL
    assert L.fsdp_peer_rs_reduce(None, 0, None, None) == abi.FSDP_EINVAL
    assert L.fsdp_peer_adamw_step(None, None, None, None, None, None, None) == abi.FSDP_EINVAL
    assert L.fsdp_peer_rs_adamw_step(None, 0, None, None, None, None, None, None,
                                     None) == abi.FSDP_EINVAL
    L.fsdp_destroy_peer_plan(None)
    ptr, hd = ctypes.c_void_p(), abi.IpcHandle()
    assert L.fsdp_ipc_alloc(0, ctypes.byref(ptr), ctypes.byref(hd)) == abi.FSDP_EINVAL
    assert L.fsdp_ipc_alloc(-5, ctypes.byref(ptr), ctypes.byref(hd)) == abi.FSDP_EINVAL
    assert L.fsdp_ipc_alloc(64, None, ctypes.byref(hd)) == abi.FSDP_EINVAL
    assert L.fsdp_ipc_open(None, ctypes.byref(ptr)) == abi.FSDP_EINVAL
    assert L.fsdp_ipc_free(None) == abi.FSDP_EINVAL
    assert L.fsdp_ipc_close(None) == abi.FSDP_EINVAL
    assert ctypes.sizeof(abi.IpcHandle) == 64


def test_noalloc_wrapper_derives_sizes_from_the_shapes(abi, oracle):
    """The binding of fsdp_rs_reduce_noalloc works S and P_arena out of the
    shapes (the C call cannot see buffer sizes) and refuses caller-supplied
    values that disagree, before touching the tensors or the library."""
    import torch
    cases = [([(7, 3), (5,), (1, 32), (1,), (0, 4), (13, 9), (2, 2)], 4),
             ([(32003, 64), (4096,), (17, 5)], 6), ([], 3), ([()], 2), ([(9, 5), (3,)], 12)]
    for shapes, N in cases:
        p = oracle.plan(shapes, N)
        assert abi.group_layout(shapes, N) == (p.S, p.P, p.P_arena)
    shapes, N = cases[0]
    p = oracle.plan(shapes, N)
    g = torch.zeros(4, dtype=torch.bfloat16)
    r = torch.zeros(4)
    for kw in ({"S": p.S - 1}, {"S": p.S + 8}, {"P_arena": p.P_arena - 8},
               {"P_arena": p.P_arena + 1}):
        with pytest.raises(ValueError, match="does not match"):
            abi.fsdp_rs_reduce_noalloc(shapes, N, g, 1, r, **kw)
    # right sizes: the next check (CUDA tensors of at least that size) is reached
    with pytest.raises(ValueError, match="CUDA tensor"):
        abi.fsdp_rs_reduce_noalloc(shapes, N, g, 1, r, S=p.S, P_arena=p.P_arena)


def test_debug_library_loads_and_exports_every_symbol(abi):
    """libfsdpk_debug.so (-DFSDPK_DEBUG) exports the same C API; only it
    accepts error words, and it validates them on the host."""
    from fully_sharded_shard_b200 import build
    path = build.build(debug=True)
    D = ctypes.CDLL(path)
    for n in _declared():
        assert hasattr(D, n), f"{n} not exported by the debug library"
    D.fsdp_debug_set_error_words.argtypes = [ctypes.c_void_p, ctypes.c_int64]
    assert D.fsdp_debug_build() == 1
    assert D.fsdp_debug_set_error_words(None, -1) == abi.FSDP_EINVAL
    assert D.fsdp_debug_set_error_words(ctypes.c_void_p(6), 0) == abi.FSDP_EALIGN
    assert D.fsdp_debug_set_error_words(None, 0) == abi.FSDP_OK
    R = abi.lib()
    R.fsdp_debug_set_error_words.argtypes = [ctypes.c_void_p, ctypes.c_int64]
    assert R.fsdp_debug_build() == 0
    assert R.fsdp_debug_set_error_words(None, 0) == abi.FSDP_ESTATE
