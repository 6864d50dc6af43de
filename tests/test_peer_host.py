"""Host logic of the rank-per-process layer (collective_rc_all_b200.peer) on
CPU, gloo, world size 2, with the library's IPC and rank-view calls replaced
by recorders: the handle exchange hands every rank the others' imported
addresses in rank order, every collective is fenced by host barriers (the
ring: one before each of its 2(p-1) steps and one after the last), close()
releases exactly the imports, and a rank that leaves makes the other's next
barrier fail instead of hanging."""
import datetime
import os
import socket
import sys

import torch.multiprocessing as mp

from conftest import ROOT


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _patch(peer, rank, log):
    peer.rc_ipc_export = lambda t: f"h{rank}:{t}".encode()
    peer.rc_ipc_import = lambda h: log.append(("import", h.decode())) or 1000 + int(h.decode()[1])
    peer.rc_ipc_release = lambda a: log.append(("release", a))
    peer.rc_rank_all_reduce = lambda s, r, k, **kw: log.append(("all_reduce", list(s), list(r), k))
    peer.rc_rank_reduce_scatter = lambda s, o, k, **kw: log.append(("reduce_scatter", list(s), o, k))
    peer.rc_rank_all_gather = lambda s, o, k, **kw: log.append(("all_gather", list(s), o, k))
    peer.rc_rank_ring_step = lambda s, r, k, step, **kw: log.append(("ring", k, step, kw.get("ws")))


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import collective_rc_all_b200.peer as peer
    log = []
    _patch(peer, rank, log)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    syncs = []
    g = peer.PeerGroup(sync=lambda: syncs.append(1))
    send = g.share("x")
    recv = g.share("y")
    b0 = g.barriers
    g.all_reduce(send, recv)
    b1 = g.barriers
    g.reduce_scatter(send, "out")
    g.all_gather(send, "full")
    b2 = g.barriers
    g.ring_all_reduce(send, recv, ws=["w"] * world)
    b3 = g.barriers
    g.close()
    q.put((rank, send, recv, log, (b0, b1, b2, b3, g.barriers), len(syncs)))
    dist.destroy_process_group()


def test_peer_group_host_logic_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = sorted(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(60)
        assert p.exitcode == 0
    for rank, send, recv, log, bars, nsync in got:
        other = 1 - rank
        # own buffer at its own index, the peer's import elsewhere
        assert send[rank] == "x" and send[other] == 1000 + other
        assert recv[rank] == "y" and recv[other] == 1000 + other
        imports = [e for e in log if e[0] == "import"]
        assert imports == [("import", f"h{other}:x"), ("import", f"h{other}:y")]
        calls = [e for e in log if e[0] not in ("import", "release")]
        assert calls[0] == ("all_reduce", send, recv, rank)
        assert calls[1] == ("reduce_scatter", send, "out", rank)
        assert calls[2] == ("all_gather", send, "full", rank)
        ring = calls[3:]
        assert ring == [("ring", rank, 0, ["w", "w"]), ("ring", rank, 1, ["w", "w"])]  # 2(p-1) = 2 steps
        b0, b1, b2, b3, b_end = bars
        assert b0 == 0 and b1 == 2 and b2 == 6       # two barriers around each collective
        assert b3 - b2 == 2 * (2 - 1) + 1            # one before each ring step, one after
        assert b_end - b3 == 2                       # close: before and after the releases
        assert [e for e in log if e[0] == "release"] == [("release", 1000 + other)] * 2
        assert nsync == b_end - 1                    # every barrier but the last waits for the stream first


def _leaver(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import collective_rc_all_b200.peer as peer
    _patch(peer, rank, [])
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=5))
    g = peer.PeerGroup(sync=lambda: None)
    send = g.share("x")
    if rank == 1:
        q.put((rank, "left"))
        q.close()
        q.join_thread()  # the message is out before the process goes
        os._exit(0)  # leaves between collectives, nothing in flight
    try:
        g.all_reduce(send, send)
        q.put((rank, "no error"))
    except Exception as e:  # the barrier reports the missing rank
        q.put((rank, "error: " + type(e).__name__))


def test_a_rank_that_leaves_fails_the_next_barrier():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_leaver, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(60)
    assert got[1] == "left"
    assert got[0].startswith("error"), got[0]
