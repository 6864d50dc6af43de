"""The C ABI library loads and exports every entry point the header declares,
and rejects bad arguments on the host before anything reaches a GPU.
CPU only (no CUDA device needed)."""
import ctypes
import os
import re

import pytest

from conftest import ROOT

HEADER = os.path.join(ROOT, "include", "rankcoll.h")


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(rc_[a-z_0-9]+)\s*\(", text)))


@pytest.fixture(scope="module")
def rc():
    import collective_rc_all_b200 as m
    return m


def test_header_declares_the_collectives():
    names = _declared()
    for n in ("rc_all_reduce", "rc_reduce_scatter", "rc_all_gather", "rc_reduce", "rc_broadcast",
              "rc_ring_all_reduce", "rc_hier_all_reduce"):
        assert n in names


def test_library_exports_every_declared_symbol(rc):
    for name in _declared():
        assert hasattr(rc.lib, name), f"{name} declared in include/ but not exported"


def test_status_strings(rc):
    for code in range(5):
        assert rc.lib.rc_status_string(code)
    assert rc.rc_version() == 100


def _null(p):
    return (ctypes.c_void_p * p)(*([0] * p))


def test_invalid_arguments_rejected_on_host(rc):
    L = rc.lib
    a = _null(16)
    before = rc.rc_launch_count()
    assert L.rc_all_reduce(a, a, 0, 10, 0, 0, 1.0, None) == 1          # p < 1
    assert L.rc_all_reduce(a, a, 17, 10, 0, 0, 1.0, None) == 1         # p > 16
    assert L.rc_all_reduce(a, a, 2, 10, 7, 0, 1.0, None) == 1          # dtype
    assert L.rc_all_reduce(a, a, 2, 10, 0, 9, 1.0, None) == 1          # op
    assert L.rc_all_reduce(a, a, 2, 10, 0, 1, 0.5, None) == 1          # scale with MAX
    assert L.rc_all_reduce(a, a, 2, 10, 2, 0, 0.5, None) == 1          # scale with int32
    assert L.rc_all_reduce(a, a, 2, 10, 0, 0, 1.0, None) == 1          # NULL buffers
    assert "NULL" in rc.rc_last_error()
    assert L.rc_reduce_scatter(a, a, 4, 10, 0, 0, 0, 1.0, None) == 1   # 4 does not divide 10
    assert L.rc_reduce_scatter(a, a, 2, 10, 2, 0, 0, 1.0, None) == 1   # int32 -> fp32
    assert L.rc_all_gather(a, a, 3, 10, 0, None) == 1                  # 3 does not divide 10
    assert L.rc_reduce(a, None, 4, 4, 10, 0, 0, 1.0, None) == 1        # root out of range
    assert L.rc_broadcast(None, a, 4, -1, 10, 0, None) == 1            # root out of range
    assert L.rc_hier_all_reduce(a, a, 8, 3, 10, 0, 0, 1.0, 0, None) == 1   # 3 does not divide 8
    assert L.rc_hier_all_reduce(a, a, 8, 4, 10, 0, 0, 1.0, 5, None) == 1   # variant
    assert L.rc_ring_all_reduce(a, a, 8, 10, 0, 0, 1.0, 5, None) == 1      # variant
    assert L.rc_all_reduce(None, None, 2, 10, 0, 0, 1.0, None) == 1    # NULL arrays
    assert rc.rc_launch_count() == before


def test_empty_calls_are_noops(rc):
    L = rc.lib
    a = _null(4)
    before = rc.rc_launch_count()
    assert L.rc_all_reduce(a, a, 4, 0, 0, 0, 1.0, None) == 0
    assert L.rc_reduce_scatter(a, a, 4, 0, 0, 1, 0, 0.25, None) == 0
    assert L.rc_all_gather(a, a, 4, 0, 1, None) == 0
    assert L.rc_reduce(a, None, 4, 0, 0, 2, 1, 1.0, None) == 0
    assert L.rc_broadcast(None, a, 4, 0, 0, 0, None) == 0
    assert L.rc_ring_all_reduce(a, a, 4, 0, 0, 0, 1.0, 0, None) == 0
    assert L.rc_hier_all_reduce(a, a, 4, 2, 0, 0, 0, 1.0, 1, None) == 0
    assert rc.rc_launch_count() == before


def test_host_memory_is_not_a_device_pointer(rc):
    """Without a GPU (or with one) a host address is rejected, never launched."""
    import numpy as np
    x = [np.zeros(64, np.float32) for _ in range(2)]
    ptr = (ctypes.c_void_p * 2)(*[v.ctypes.data for v in x])
    before = rc.rc_launch_count()
    assert rc.lib.rc_all_reduce(ptr, ptr, 2, 64, 0, 0, 1.0, None) == 1
    assert rc.rc_launch_count() == before


def test_optimizer_arguments_rejected_on_host(rc):
    L = rc.lib
    a = _null(8)
    hp = rc.rc_adamw_hparams(1e-3, 0.9, 0.999, 1e-8, 0.0, 1)
    bad_step = rc.rc_adamw_hparams(1e-3, 0.9, 0.999, 1e-8, 0.0, 0)
    before = rc.rc_launch_count()
    assert L.rc_zero1_step(a, a, a, a, a, 8, 64, 0, 1, 0.125, None, None) == 1           # NULL hparams
    assert L.rc_zero1_step(a, a, a, a, a, 8, 64, 0, 1, 0.125, ctypes.byref(bad_step), None) == 1
    assert L.rc_zero1_step(a, a, a, a, a, 8, 60, 0, 1, 0.125, ctypes.byref(hp), None) == 1  # 8 does not divide 60
    assert L.rc_zero1_step(a, a, a, a, a, 8, 64, 2, 1, 0.125, ctypes.byref(hp), None) == 1  # int32 grads
    assert L.rc_zero1_step(a, a, a, a, a, 8, 64, 0, 2, 0.125, ctypes.byref(hp), None) == 1  # int32 params
    assert L.rc_zero1_step(a, a, a, a, a, 17, 64, 0, 1, 0.125, ctypes.byref(hp), None) == 1  # p > 16
    assert L.rc_zero1_step(a, a, a, a, a, 8, 64, 0, 1, 0.125, ctypes.byref(hp), None) == 1  # NULL buffers
    assert L.rc_adamw_step(None, None, None, None, 0, 16, None, None) == 1
    assert L.rc_adamw_step(None, None, None, None, 2, 16, ctypes.byref(hp), None) == 1      # int32 grad
    assert L.rc_adamw_step(None, None, None, None, 0, 16, ctypes.byref(hp), None) == 1      # NULL buffers
    assert L.rc_zero1_step(a, a, a, a, a, 8, 0, 0, 1, 0.125, ctypes.byref(hp), None) == 0   # empty
    assert L.rc_adamw_step(None, None, None, None, 0, 0, ctypes.byref(hp), None) == 0
    assert rc.rc_launch_count() == before


def test_rank_view_and_ipc_arguments_rejected_on_host(rc):
    L = rc.lib
    a = _null(8)
    before = rc.rc_launch_count()
    assert L.rc_rank_all_reduce(a, a, 4, 4, 10, 0, 0, 1.0, None) == 1          # rank == p
    assert L.rc_rank_all_reduce(a, a, 4, -1, 10, 0, 0, 1.0, None) == 1         # rank < 0
    assert L.rc_rank_all_reduce(a, a, 4, 0, 10, 0, 1, 0.5, None) == 1          # scale with MAX
    assert L.rc_rank_all_reduce(a, a, 4, 0, 10, 0, 0, 1.0, None) == 1          # NULL buffers
    assert L.rc_rank_reduce_scatter(a, None, 4, 0, 10, 0, 0, 0, 1.0, None) == 1  # 4 does not divide 10
    assert L.rc_rank_all_gather(a, None, 4, 5, 8, 0, None) == 1                # rank out of range
    assert L.rc_rank_ring_step(a, a, None, 1, 0, 0, 10, 0, 0, 1.0, None) == 1  # the ring needs p >= 2
    assert L.rc_rank_ring_step(a, a, None, 4, 0, 6, 10, 0, 0, 1.0, None) == 1  # step 6 of 2(p-1) = 6
    assert L.rc_rank_ring_step(a, a, None, 4, 0, 0, 10, 1, 0, 1.0, None) == 1  # bf16 without workspaces
    assert "workspace" in rc.rc_last_error()
    assert L.rc_rank_all_reduce(a, a, 4, 0, 0, 0, 0, 1.0, None) == 0           # n = 0: nothing to do
    assert L.rc_ipc_import(None, None) == 1
    assert L.rc_ipc_release(None) == 1                                          # never imported
    h = rc.rc_ipc_handle()
    assert L.rc_ipc_export(None, 16, ctypes.byref(h)) == 1                      # NULL buffer
    assert rc.rc_launch_count() == before
