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


def test_noalloc_ring_at_the_scratch_limit_allocates_nothing():
    """At exactly the fixed scratch's limit (p = 8, n = 2,097,152 bf16, the
    8 MiB-per-rank ring workload: 2*p*ceil(n/p) = 4,194,304 floats) the call
    is accepted, gives the existing entry point's bits, and neither grows the
    library workspace nor takes device memory; one vector more is rejected."""
    rc, fn = _cabi()
    stream = torch.cuda.current_stream().cuda_stream
    p, n = 8, 2097152
    xs = rc_inputs.normal(p, n, seed=43, sigma=1.0, dt="bf16")
    d, _ = to_dev(xs, "bf16")
    got, back = empty_dev(n, "bf16", p)
    small, _ = empty_dev(64, "bf16", p)
    assert fn(_ptrs(d), _ptrs(small), p, 64, 1, 0, 1.0, stream) == 0   # first call: address look-up
    torch.cuda.synchronize()
    rc.rc_finalize()                                   # no library workspace from here on
    assert rc.rc_workspace_bytes() == (0, 0)
    free_before = torch.cuda.mem_get_info()[0]
    st = fn(_ptrs(d), _ptrs(got), p, n, 1, 0, 1.0, stream)
    assert st == 0, rc.rc_last_error()
    torch.cuda.synchronize()
    rc.rc_stream_status()
    assert torch.cuda.mem_get_info()[0] == free_before
    assert rc.rc_workspace_bytes() == (0, 0)
    want, _ = empty_dev(n, "bf16", p)
    rc.rc_ring_all_reduce(d, want, variant="literal")
    torch.cuda.synchronize()
    rc.rc_stream_status()
    for r in range(p):
        assert_bits(to_host(got[r], "bf16"), to_host(want[r], "bf16"), f"noalloc ring at the limit r{r}")
    for b in back:
        assert np.all(b[n * 2:].cpu().numpy() == 0x5A)
    n1 = n + 8                                          # ceil(n1/p) = 262,145: 16 floats too many
    d1 = [torch.empty(n1, dtype=torch.bfloat16, device="cuda") for _ in range(p)]
    y1 = [torch.empty(n1, dtype=torch.bfloat16, device="cuda") for _ in range(p)]
    before = rc.rc_launch_count()
    assert fn(_ptrs(d1), _ptrs(y1), p, n1, 1, 0, 1.0, stream) == 1
    assert "scratch" in rc.rc_last_error()
    assert rc.rc_launch_count() == before
