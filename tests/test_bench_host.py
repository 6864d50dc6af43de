"""Host-side logic of bench.py on CPU: the byte accounting, the multi-rank
reduction of timings (gloo, world size 2), and the reference arm under
torchrun (rank 0 prints one JSON line, the other ranks exit 0 silently)."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

from conftest import ROOT


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def test_step_bytes():
    import bench
    ops, m = bench.step_ops(8, 2097152)
    d = dict(ops)
    assert m == 262144
    assert d["all_reduce"] == 2 * 8 * 2097152 * 4 == 128 << 20
    assert d["reduce_scatter"] == (64 << 20) + (4 << 20)
    assert d["all_gather"] == (4 << 20) + (32 << 20)
    assert d["broadcast"] == 64 << 20
    assert d["ring_all_reduce"] == d["hier_all_reduce"] == d["all_reduce"]


def test_ring_time_model():
    import bench
    # 2 (N-1)/N * S/W with N = 8, S = 8 MiB, W = 1 GB/s
    assert abs(bench.ring_model_seconds(8 << 20, 8, 1e9) - 2 * 7 / 8 * (8 << 20) / 1e9) < 1e-12


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    t, b = bench.reduce_over_ranks(0.5 + rank, 100.0 * (rank + 1), world)
    q.put((rank, t, b))
    dist.destroy_process_group()


def test_reduce_over_ranks_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    for rank, t, b in got:
        assert t == 1.5          # max of the ranks' times
        assert b == 300.0        # sum of the ranks' bytes


def test_reference_arm_single():
    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1",
                          "--warmup", "3", "--ref-seconds", "1"], cwd=ROOT, capture_output=True,
                         text=True, timeout=300)
    assert out.returncode == 0, out.stderr
    line = json.loads(out.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] == 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0


def test_reference_arm_under_torchrun():
    port = _free_port()
    out = subprocess.run([sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
                          "--nproc-per-node", "2", "--master-addr", "127.0.0.1", "--master-port",
                          str(port), "bench.py", "--impl", "reference", "--gpus", "2", "--steps",
                          "1", "--warmup", "3", "--ref-seconds", "1"],
                         cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    assert json.loads(lines[0])["n_gpus"] == 2
