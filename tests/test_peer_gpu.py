"""Rank-per-process collectives through real CUDA IPC mappings: 2 and 4
processes share the one GPU of the test box, exchange their buffers with
rc_ipc_export / rc_ipc_import over a gloo group, and run the rank view fenced
by host barriers (PeerGroup).  No kernel waits for another process: every
ordering is a stream synchronise plus a host barrier.  Every rank checks its
own outputs against the oracle bit for bit: all-reduce, reduce-scatter
(fp32 -> bf16, x 1/p), all-gather, and the literal ring in fp32 and bf16
(workspaces shared like the buffers)."""
import datetime
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from conftest import ROOT

pytestmark = pytest.mark.gpu


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, n, q):
    try:
        os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
        sys.path.insert(0, ROOT)
        sys.path.insert(0, os.path.join(ROOT, "tests"))
        import torch.distributed as dist
        import collective_rc_all_b200 as rc
        from collective_rc_all_b200.peer import PeerGroup
        import oracle
        import rc_inputs
        from util import assert_bits, to_host

        torch.cuda.set_device(0)
        dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
        p, m = world, n // world
        g = PeerGroup()
        results = []

        xs = rc_inputs.uniform(p, n, seed=40 + p)
        x_own = torch.from_numpy(xs[rank]).cuda()
        y_own = torch.zeros(n, device="cuda")
        x, y = g.share(x_own), g.share(y_own)

        g.all_reduce(x, y, scale=1.0 / p)
        assert_bits(to_host(y_own, "f32"), oracle.all_reduce(xs, "f32", "sum", 1.0 / p)[rank], "all_reduce")
        results.append("all_reduce")

        shard = torch.zeros(m, dtype=torch.bfloat16, device="cuda")
        g.reduce_scatter(x, shard, scale=1.0 / p)
        want_rs = oracle.reduce_scatter(xs, "f32", "bf16", "sum", 1.0 / p)
        assert_bits(to_host(shard, "bf16"), want_rs[rank], "reduce_scatter")
        results.append("reduce_scatter")

        full = torch.zeros(n, dtype=torch.bfloat16, device="cuda")
        g.all_gather(g.share(shard), full)
        assert_bits(to_host(full, "bf16"), oracle.all_gather(want_rs, "bf16")[rank], "all_gather")
        results.append("all_gather")

        y_own.zero_()
        g.ring_all_reduce(x, y, scale=1.0 / p)
        assert_bits(to_host(y_own, "f32"), oracle.ring_all_reduce(xs, "f32", "sum", 1.0 / p)[rank], "ring f32")
        results.append("ring_f32")

        hs = rc_inputs.uniform(p, n, seed=50 + p, dt="bf16")
        h_own = torch.from_numpy(hs[rank].view(np.int16)).cuda().view(torch.bfloat16)
        hy_own = torch.zeros(n, dtype=torch.bfloat16, device="cuda")
        C = (n + p - 1) // p
        ws_own = torch.zeros(2 * C, device="cuda")
        hx, hy, ws = g.share(h_own), g.share(hy_own), g.share(ws_own)
        g.ring_all_reduce(hx, hy, ws=ws, op="max")
        assert_bits(to_host(hy_own, "bf16"), oracle.ring_all_reduce(hs, "bf16", "max", 1.0)[rank], "ring bf16")
        results.append("ring_bf16")

        rc.rc_stream_status()
        g.close()
        dist.destroy_process_group()
        q.put((rank, "ok", results))
    except Exception as e:  # report, then leave; the others fail at their next barrier
        q.put((rank, f"{type(e).__name__}: {e}", []))


# (2, 2 * 16384): every buffer and chunk 16-byte aligned, the vector paths;
# (4, 4 * 12289): chunks of an odd length, the scalar paths
@pytest.mark.parametrize("world,n", [(2, 2 * 16384), (4, 4 * 12289)])
def test_peer_group_over_ipc_on_one_gpu(world, n):
    assert torch.cuda.is_available()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, n, q)) for r in range(world)]
    for pr in procs:
        pr.start()
    got = {}
    try:
        for _ in range(world):
            rank, status, results = q.get(timeout=300)
            got[rank] = (status, results)
    finally:
        for pr in procs:
            pr.join(60)
            if pr.is_alive():
                pr.kill()
    for r in range(world):
        assert got[r][0] == "ok", f"rank {r}: {got[r][0]}"
        assert got[r][1] == ["all_reduce", "reduce_scatter", "all_gather", "ring_f32", "ring_bf16"]
