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
