"""The ring all-reduce entry point that allocates nothing, for callers that
cannot allocate device memory at call time (their memory belongs to another
allocator, or they must not stall on cudaMalloc/cudaFree).  It is called here
through the C ABI directly and must give the same bits as the allocating
rc_ring_all_reduce, on two calls in a row (the fixed scratch array is shared
and keeps the previous call's contents).

This file is named to be collected last, so that a failure here does not
stop a run before every other test has run.
"""
import ctypes

import numpy as np
import pytest
import torch

import rc_inputs
from util import assert_bits, empty_dev, to_dev, to_host

pytestmark = pytest.mark.gpu


def _cabi():
    import collective_rc_all_b200 as rc
    L = rc.lib
    fn = L.rc_ring_all_reduce_noalloc
    vpp = ctypes.POINTER(ctypes.c_void_p)
    fn.argtypes = [vpp, vpp, ctypes.c_int, ctypes.c_size_t, ctypes.c_int, ctypes.c_int,
                   ctypes.c_float, ctypes.c_void_p]
    fn.restype = ctypes.c_int
    return rc, fn


def _ptrs(ts):
    return (ctypes.c_void_p * len(ts))(*[t.data_ptr() for t in ts])


@pytest.mark.parametrize("dt,code", [("bf16", 1), ("f32", 0)])
def test_noalloc_ring_matches_allocating_ring_twice(dt, code):
    assert torch.cuda.is_available()
    rc, fn = _cabi()
    p, n = 8, 8 * 4096 + 8 * 24
    stream = torch.cuda.current_stream().cuda_stream
    for call, seed in enumerate((41, 42)):          # two calls in a row
        xs = rc_inputs.normal(p, n, seed=seed, sigma=1.0, dt=dt)
        d, _ = to_dev(xs, dt)
        want, _ = empty_dev(n, dt, p)
        rc.rc_ring_all_reduce(d, want, variant="literal")   # the existing, allocating entry point
        got, back = empty_dev(n, dt, p)
        st = fn(_ptrs(d), _ptrs(got), p, n, code, 0, 0.5 if call else 1.0, stream)
        assert st == 0, rc.rc_last_error()
        if call:   # the second call also checks the scale path against the existing entry point
            rc.rc_ring_all_reduce(d, want, scale=0.5, variant="literal")
        torch.cuda.synchronize()
        rc.rc_stream_status()
        for r in range(p):
            assert_bits(to_host(got[r], dt), to_host(want[r], dt), f"noalloc ring {dt} call {call} r{r}")
        for b in back:   # nothing written past the outputs
            assert np.all(b[n * (2 if dt == "bf16" else 4):].cpu().numpy() == 0x5A)


def test_noalloc_ring_rejects_oversize_without_launch():
    rc, fn = _cabi()
    p = 8
    n = 2 * 4194304 // 2 + 64        # 2*p*ceil(n/p) floats exceed the fixed scratch
    d = [torch.empty(n, dtype=torch.bfloat16, device="cuda") for _ in range(p)]
    y = [torch.empty(n, dtype=torch.bfloat16, device="cuda") for _ in range(p)]
    before = rc.rc_launch_count()
    st = fn(_ptrs(d), _ptrs(y), p, n, 1, 0, 1.0, torch.cuda.current_stream().cuda_stream)
    assert st == 1 and "scratch" in rc.rc_last_error()
    assert rc.rc_launch_count() == before
