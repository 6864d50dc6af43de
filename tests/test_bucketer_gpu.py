"""GPU tests of the gradient bucketer: every bucket's in-place all-reduce
against the oracle (an all-reduce of the bucket's slice of every rank's flat
buffer, x 1/p), for per-tensor, capped and single-bucket plans, tensors
marked ready in any order, producers on their own streams, several steps,
and the error paths (a tensor never marked ready, a tensor marked twice)."""
import numpy as np
import pytest
import torch

import oracle
import rc_inputs
from util import assert_bits, to_host

pytestmark = pytest.mark.gpu

SIZES = [1000, 33, 4096, 7, 20000, 512, 1, 65536, 300]


@pytest.fixture(scope="module")
def rc():
    import collective_rc_all_b200 as m
    assert torch.cuda.is_available()
    return m


def _want(rc, host, sizes, cap, dt):
    """Oracle result: all-reduce (x 1/p) of each bucket's slice, bucket plan
    from the host planner."""
    p = len(host)
    esz = 2 if dt == "bf16" else 4
    plan, nb = rc.rc_plan_buckets(sizes, esz, cap)
    off = np.concatenate([[0], np.cumsum(sizes)])
    out = [h.copy() for h in host]
    for k in range(nb):
        ts = [t for t in range(len(sizes)) if plan[t] == k]
        a, b = int(off[ts[0]]), int(off[ts[-1] + 1])
        red = oracle.all_reduce([h[a:b] for h in host], dt, "sum", 1.0 / p)
        for r in range(p):
            out[r][a:b] = red[r]
    return out


def _flat(host, dt):
    tdt = torch.bfloat16 if dt == "bf16" else torch.float32
    out = []
    for h in host:
        t = torch.from_numpy(h.view(np.int16) if dt == "bf16" else h).cuda()
        out.append(t.view(tdt) if dt == "bf16" else t)
    return out


@pytest.mark.parametrize("dt", ["f32", "bf16"])
@pytest.mark.parametrize("cap", [0, 16 << 10, 2 ** 63])
@pytest.mark.parametrize("order", ["forward", "reverse", "shuffled"])
def test_bucketed_all_reduce_matches_oracle(rc, dt, cap, order):
    p = 4
    n = sum(SIZES)
    host = rc_inputs.uniform(p, n, seed=5, dt=dt)
    flat = _flat(host, dt)
    comm = torch.cuda.Stream()
    b = rc.Bucketer(flat, SIZES, cap, comm_stream=comm)
    ts = list(range(len(SIZES)))
    if order == "reverse":
        ts = ts[::-1]
    elif order == "shuffled":
        ts = list(np.random.default_rng(3).permutation(ts))
    for t in ts:
        b.ready(int(t))
    b.flush()
    torch.cuda.synchronize()
    rc.rc_stream_status()
    want = _want(rc, host, SIZES, cap, dt)
    for r in range(p):
        assert_bits(to_host(flat[r], dt), want[r], f"bucketed AR cap={cap} {order} rank {r}")
    b.close()


def test_producers_on_their_own_streams_and_several_steps(rc):
    """Gradients written on a producer stream after a long dummy kernel: the
    bucket all-reduce must wait for them.  Two steps on the same bucketer."""
    p, dt, cap = 8, "f32", 64 << 10
    n = sum(SIZES)
    comm, prod = torch.cuda.Stream(), torch.cuda.Stream()
    flat = [torch.zeros(n, device="cuda") for _ in range(p)]
    b = rc.Bucketer(flat, SIZES, cap, comm_stream=comm)
    off = np.concatenate([[0], np.cumsum(SIZES)])
    busy = torch.empty(1 << 27, device="cuda")
    for step in range(2):
        host = rc_inputs.uniform(p, n, seed=20 + step, dt=dt)
        src = [torch.from_numpy(h).cuda() for h in host]
        torch.cuda.synchronize()
        with torch.cuda.stream(prod):
            for _ in range(4):
                busy.normal_()  # keeps the producer stream busy before the gradients appear
            for t in reversed(range(len(SIZES))):  # backward order
                a, e = int(off[t]), int(off[t + 1])
                for r in range(p):
                    flat[r][a:e].copy_(src[r][a:e])
                b.ready(t, prod)
        b.flush(torch.cuda.current_stream())
        torch.cuda.synchronize()
        rc.rc_stream_status()
        want = _want(rc, host, SIZES, cap, dt)
        for r in range(p):
            assert_bits(to_host(flat[r], dt), want[r], f"step {step} rank {r}")
    b.close()


def test_incomplete_and_double_ready_are_errors(rc):
    p, n = 2, sum(SIZES)
    flat = [torch.zeros(n, device="cuda") for _ in range(p)]
    b = rc.Bucketer(flat, SIZES, 0)
    b.ready(0)
    with pytest.raises(rc.RankCollError):
        b.ready(0)
    assert "twice" in rc.rc_last_error()
    with pytest.raises(rc.RankCollError):
        b.flush()  # tensors 1.. were never marked
    assert "incomplete" in rc.rc_last_error()
    # the next step starts clean
    for t in range(len(SIZES)):
        b.ready(t)
    b.flush()
    torch.cuda.synchronize()
    rc.rc_stream_status()
    b.close()


def test_single_rank_bucketer(rc):
    """p = 1: every bucket's all-reduce is the identity times scale (1)."""
    host = rc_inputs.uniform(1, sum(SIZES), seed=8, dt="f32")
    flat = _flat(host, "f32")
    b = rc.Bucketer(flat, SIZES, 16 << 10, scale=1.0)
    for t in range(len(SIZES)):
        b.ready(t)
    b.flush()
    torch.cuda.synchronize()
    rc.rc_stream_status()
    assert_bits(to_host(flat[0], "f32"), host[0], "bucketer p=1")
    b.close()
