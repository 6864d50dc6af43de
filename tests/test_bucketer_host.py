"""Host-side bucket planning of the gradient bucketer (no GPU): buckets are
runs of consecutive whole tensors, each closed as soon as it holds at least
the cap; cap 0 gives one bucket per tensor, an unbounded cap one bucket."""
import numpy as np
import pytest


@pytest.fixture(scope="module")
def rc():
    import collective_rc_all_b200 as m
    return m


@pytest.mark.parametrize("seed", range(6))
@pytest.mark.parametrize("cap", [0, 1, 4096, 1 << 20, 25 << 20, 1 << 62])
def test_plan_properties(rc, seed, cap):
    r = np.random.default_rng(seed)
    numel = [int(x) for x in r.integers(1, 1 << 20, r.integers(1, 60))]
    esz = 2
    b, nb = rc.rc_plan_buckets(numel, esz, cap)
    assert b[0] == 0 and b[-1] == nb - 1
    assert all(y - x in (0, 1) for x, y in zip(b, b[1:]))           # consecutive runs, in order
    for k in range(nb):
        sizes = [numel[t] * esz for t in range(len(numel)) if b[t] == k]
        if k < nb - 1:
            assert sum(sizes) >= cap or cap == 0                     # a closed bucket reached the cap
        assert sum(sizes[:-1]) < max(cap, 1)                         # ...and not before its last tensor
    if cap == 0:
        assert nb == len(numel)
    if cap >= sum(numel) * esz:
        assert nb == 1


def test_plan_worked_case(rc):
    # 4-byte elements, cap 64 B: [40, 80 | 20, 400 | 4, 4]
    assert rc.rc_plan_buckets([10, 20, 5, 100, 1, 1], 4, 64) == ([0, 0, 1, 1, 2, 2], 3)


def test_plan_rejects_bad_arguments(rc):
    import ctypes
    nb = ctypes.c_int()
    assert rc.lib.rc_plan_buckets(2, None, 4, 64, None, ctypes.byref(nb)) == 1
    arr = (ctypes.c_size_t * 2)(1, 2)
    out = (ctypes.c_int * 2)()
    assert rc.lib.rc_plan_buckets(2, arr, 0, 64, out, ctypes.byref(nb)) == 1   # zero element size
    assert "rc_plan_buckets" in rc.rc_last_error()


def test_bucketer_create_rejects_host_memory(rc):
    import ctypes
    x = [np.zeros(64, np.float32) for _ in range(2)]
    ptr = (ctypes.c_void_p * 2)(*[v.ctypes.data for v in x])
    arr = (ctypes.c_size_t * 2)(32, 32)
    h = ctypes.c_void_p()
    before = rc.rc_launch_count()
    assert rc.lib.rc_bucketer_create(ctypes.byref(h), ptr, 2, 2, arr, 64, 0, 0.5, None) == 1
    assert not h.value
    assert rc.lib.rc_bucketer_create(ctypes.byref(h), ptr, 2, 2, arr, 64, 2, 0.5, None) == 1  # int32 + scale
    assert rc.rc_launch_count() == before
