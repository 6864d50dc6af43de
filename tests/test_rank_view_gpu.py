"""GPU parity of the rank view (one rank's share of a collective), with every
rank's share run in one process on one GPU: calling the rank view for every
rank must give the oracle's collective bit for bit -- all-reduce (each rank
its chunk, written to every rank), reduce-scatter (each rank its shard),
all-gather (each rank pulls every shard), and the literal ring run step by
step (every rank's step s before any rank's step s+1).  Ragged n (a short
and an empty last chunk), unaligned buffers (scalar paths), in-place
buffers, canaries after every output, and the argument checks."""
import numpy as np
import pytest
import torch

import oracle
import rc_inputs
from util import assert_bits, check_canary, empty_dev, to_dev, to_host

pytestmark = pytest.mark.gpu

ESZ = {"f32": 4, "bf16": 2, "i32": 4}


@pytest.fixture(scope="module")
def rc():
    import collective_rc_all_b200 as m
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return m


def _data(p, n, dt, seed):
    if dt == "i32":
        return rc_inputs.int_uniform(p, n, seed)
    return rc_inputs.uniform(p, n, seed, dt)


def _sync(rc):
    torch.cuda.synchronize()
    rc.rc_stream_status()


CASES = [(2, 4096), (4, 65536 + 12), (8, 8 * 3000 + 5), (8, 9), (16, 16 * 1024), (3, 100003), (5, 3)]


@pytest.mark.parametrize("p,n", CASES)
@pytest.mark.parametrize("dt", ["f32", "bf16", "i32"])
@pytest.mark.parametrize("op", ["sum", "max"])
@pytest.mark.parametrize("offset", [0, 4])
def test_rank_all_reduce_every_rank_equals_all_reduce(rc, p, n, dt, op, offset):
    xs = _data(p, n, dt, seed=7 * p + n % 97)
    scale = 1.0 / p if (op == "sum" and dt != "i32") else 1.0
    want = oracle.all_reduce(xs, dt, op, scale)
    d, _ = to_dev(xs, dt, offset_bytes=offset)
    y, yb = empty_dev(n, dt, p, offset_bytes=offset)
    for rank in range(p):
        rc.rc_rank_all_reduce(d, y, rank, op=op, scale=scale)
    _sync(rc)
    for r in range(p):
        assert_bits(to_host(y[r], dt), want[r], f"rank all_reduce p={p} n={n} {dt} {op} recv {r}")
    check_canary(yb, offset + n * ESZ[dt])


@pytest.mark.parametrize("p,n", [(2, 4096), (4, 65536 + 12), (8, 8 * 3000 + 5)])
def test_rank_all_reduce_single_rank_writes_only_its_chunk(rc, p, n):
    """One rank's call touches only its own chunk of every output."""
    xs = _data(p, n, "f32", seed=3)
    want = oracle.all_reduce(xs, "f32", "sum", 1.0)
    d, _ = to_dev(xs, "f32")
    C = (n + p - 1) // p
    for rank in range(p):
        y, _ = empty_dev(n, "f32", p, fill=0x5A)
        rc.rc_rank_all_reduce(d, y, rank)
        _sync(rc)
        lo, hi = min(n, rank * C), min(n, (rank + 1) * C)
        for r in range(p):
            got = to_host(y[r], "f32")
            assert_bits(got[lo:hi], want[r][lo:hi], f"chunk {rank} recv {r}")
            untouched = np.concatenate([got[:lo], got[hi:]]).view(np.uint32)
            assert np.all(untouched == 0x5A5A5A5A), f"rank {rank} wrote outside its chunk in recv {r}"


@pytest.mark.parametrize("p,m", [(2, 2048), (4, 3001), (8, 16384), (16, 100)])
@pytest.mark.parametrize("io", [("f32", "f32"), ("f32", "bf16"), ("bf16", "bf16"), ("i32", "i32")])
@pytest.mark.parametrize("offset", [0, 4])
def test_rank_reduce_scatter_every_rank_equals_reduce_scatter(rc, p, m, io, offset):
    in_dt, out_dt = io
    n = p * m
    xs = _data(p, n, in_dt, seed=11 + p)
    scale = 1.0 / p if in_dt != "i32" else 1.0
    want = oracle.reduce_scatter(xs, in_dt, out_dt, "sum", scale)
    d, _ = to_dev(xs, in_dt, offset_bytes=offset)
    out, ob = empty_dev(m, out_dt, p, offset_bytes=offset)
    for rank in range(p):
        rc.rc_rank_reduce_scatter(d, out[rank], rank, scale=scale)
    _sync(rc)
    for r in range(p):
        assert_bits(to_host(out[r], out_dt), want[r], f"rank reduce_scatter p={p} m={m} {io} shard {r}")
    check_canary(ob, offset + m * ESZ[out_dt])


def test_rank_reduce_scatter_in_place(rc):
    """Rank r writes its shard over chunk r of its own input, which no other
    rank reads (rank q reads chunk q of every input)."""
    p, m = 4, 5000
    xs = _data(p, p * m, "f32", seed=21)
    want = oracle.reduce_scatter(xs, "f32", "f32", "sum", 0.25)
    d, _ = to_dev(xs, "f32")
    for rank in range(p):
        rc.rc_rank_reduce_scatter(d, d[rank][rank * m:(rank + 1) * m], rank, scale=0.25)
    _sync(rc)
    for r in range(p):
        assert_bits(to_host(d[r][r * m:(r + 1) * m], "f32"), want[r], f"in place shard {r}")


@pytest.mark.parametrize("p,m", [(2, 4096), (4, 3001), (8, 65536), (16, 7)])
@pytest.mark.parametrize("dt", ["f32", "bf16", "i32"])
@pytest.mark.parametrize("offset", [0, 4])
def test_rank_all_gather_every_rank_equals_all_gather(rc, p, m, dt, offset):
    shards = _data(p, m, dt, seed=5 + m % 13)
    want = oracle.all_gather(shards, dt)
    s, _ = to_dev(shards, dt, offset_bytes=offset)
    out, ob = empty_dev(p * m, dt, p, offset_bytes=offset)
    for rank in range(p):
        rc.rc_rank_all_gather(s, out[rank], rank)
    _sync(rc)
    for r in range(p):
        assert_bits(to_host(out[r], dt), want[r], f"rank all_gather p={p} m={m} {dt} out {r}")
    check_canary(ob, offset + p * m * ESZ[dt])


def test_rank_all_gather_in_place_skips_own_shard(rc):
    p, m = 4, 1024
    shards = _data(p, m, "f32", seed=9)
    want = oracle.all_gather(shards, "f32")
    out, _ = empty_dev(p * m, "f32", p)
    for r in range(p):
        out[r][r * m:(r + 1) * m].copy_(torch.from_numpy(shards[r]))
    views = [out[r][r * m:(r + 1) * m] for r in range(p)]
    for rank in range(p):
        rc.rc_rank_all_gather(views, out[rank], rank)
    _sync(rc)
    for r in range(p):
        assert_bits(to_host(out[r], "f32"), want[r], f"in-place rank all_gather out {r}")


@pytest.mark.parametrize("p,n", [(2, 4096), (4, 65536 + 12), (8, 8 * 3000 + 5), (8, 9), (16, 16 * 257),
                                 (3, 10001)])
@pytest.mark.parametrize("dt", ["f32", "bf16", "i32"])
@pytest.mark.parametrize("op", ["sum", "min"])
@pytest.mark.parametrize("offset", [0, 4])
def test_rank_ring_steps_equal_the_literal_ring(rc, p, n, dt, op, offset):
    xs = _data(p, n, dt, seed=13 * p + 1)
    scale = 1.0 / p if (op == "sum" and dt != "i32") else 1.0
    want = oracle.ring_all_reduce(xs, dt, op, scale)
    d, _ = to_dev(xs, dt, offset_bytes=offset)
    y, yb = empty_dev(n, dt, p, offset_bytes=offset)
    C = (n + p - 1) // p
    ws = [torch.empty(2 * C, dtype=torch.float32, device="cuda") for _ in range(p)] if dt == "bf16" else None
    for step in range(2 * (p - 1)):
        for rank in range(p):
            rc.rc_rank_ring_step(d, y, rank, step, ws=ws, op=op, scale=scale)
    _sync(rc)
    for r in range(p):
        assert_bits(to_host(y[r], dt), want[r], f"rank ring p={p} n={n} {dt} {op} recv {r}")
    check_canary(yb, offset + n * ESZ[dt])


def test_rank_ring_in_place(rc):
    p, n = 4, 4 * 1000 + 3
    xs = _data(p, n, "f32", seed=31)
    want = oracle.ring_all_reduce(xs, "f32", "sum", 0.25)
    d, _ = to_dev(xs, "f32")
    for step in range(2 * (p - 1)):
        for rank in range(p):
            rc.rc_rank_ring_step(d, d, rank, step, scale=0.25)
    _sync(rc)
    for r in range(p):
        assert_bits(to_host(d[r], "f32"), want[r], f"in-place rank ring recv {r}")


def test_rank_view_argument_checks(rc):
    p, n = 4, 1024
    d, _ = to_dev(_data(p, n, "f32", 1), "f32")
    y, _ = empty_dev(n, "f32", p)
    with pytest.raises(rc.RankCollError):
        rc.rc_rank_all_reduce(d, y, 4)
    with pytest.raises(rc.RankCollError):
        rc.rc_rank_all_reduce(d, y, -1)
    with pytest.raises(rc.RankCollError):
        rc.rc_rank_reduce_scatter(d, y[0][:n // p], 0, n=n + 1)  # n % p != 0
    with pytest.raises(rc.RankCollError):
        rc.rc_rank_ring_step(d, y, 0, 2 * (p - 1))  # step out of range
    b, _ = to_dev(_data(p, n, "bf16", 1), "bf16")
    yb, _ = empty_dev(n, "bf16", p)
    with pytest.raises(rc.RankCollError):
        rc.rc_rank_ring_step(b, yb, 0, 0)  # bf16 without workspaces
    assert "workspace" in rc.rc_last_error()
    h = rc.rc_ipc_export(y[0])
    with pytest.raises(rc.RankCollError):
        rc.rc_ipc_import(h)  # own export
    assert "this process" in rc.rc_last_error()
    with pytest.raises(rc.RankCollError):
        rc.rc_ipc_release(y[0].data_ptr())  # never imported
