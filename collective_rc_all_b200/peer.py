"""Rank-per-process collectives: one process per GPU, each rank's buffers
reached by the others through CUDA IPC mappings, every collective run by
this library's rank-view kernels (include/rankcoll.h, "Rank view").

Pages: "分布式训练/推理", section "从单卡到多卡：瓶颈从 HBM 扩展到互联" (past one
GPU the ranks' data crosses NVLink/NVSwitch) and section "通信原语：rank、world
size 和 collective operations" (a rank is usually one GPU or one process);
"LLM Parallelism 基础", section "Ring AllReduce" (the ring's steps).

Ordering is done on the host: before a collective every rank finishes the
work on its current stream (its inputs are complete) and meets the others at
a barrier of the process group; after it, the same again (every rank's
writes, into its own and the peers' buffers, are complete).  No kernel ever
waits for another rank, so nothing on the device can hang on a missing
peer; a rank that fails surfaces as an error of the process group's barrier
on the others (give the group a timeout).

The process group carries only the handle exchange (object all-gather) and
the barriers: gloo is enough, and it is what allows several ranks to share
one GPU (IPC on one device) as well as one rank per GPU.

Result bits equal the single-GPU collectives over the same buffers: the rank
view computes the same chunks with the same fold order.
"""
from __future__ import annotations

from typing import Callable, List, Optional, Sequence

from . import (rc_ipc_export, rc_ipc_import, rc_ipc_release, rc_rank_all_gather, rc_rank_all_reduce,
               rc_rank_reduce_scatter, rc_rank_ring_step)

__all__ = ["PeerGroup"]


def _cuda_sync():
    import torch
    torch.cuda.current_stream().synchronize()


class PeerGroup:
    """Collectives among the ranks of a torch.distributed process group.

    share(t) exchanges one buffer per rank (same shape and dtype everywhere)
    and returns the list of the p ranks' buffers as this process addresses
    them: the rank's own tensor at index `rank`, imported addresses
    elsewhere.  The collective methods take such lists.
    """

    def __init__(self, group=None, sync: Optional[Callable[[], None]] = None, dist=None):
        if dist is None:
            import torch.distributed as dist
        self._dist = dist
        self.group = group
        self.rank = dist.get_rank(group)
        self.p = dist.get_world_size(group)
        self._sync = sync or _cuda_sync
        self._imports: List[int] = []
        self.barriers = 0  # host barriers taken (for tests and accounting)

    # ------------------------------------------------------------ plumbing
    def barrier(self) -> None:
        """Finish this rank's stream work, then meet every rank."""
        self._sync()
        self._dist.barrier(group=self.group)
        self.barriers += 1

    def share(self, t) -> list:
        h = rc_ipc_export(t)
        hs: list = [None] * self.p
        self._dist.all_gather_object(hs, h, group=self.group)
        out = []
        for r, hr in enumerate(hs):
            if r == self.rank:
                out.append(t)
            else:
                a = rc_ipc_import(hr)
                self._imports.append(a)
                out.append(a)
        return out

    def close(self) -> None:
        """Drop every mapping this rank imported, after all ranks are done
        with all buffers; then a barrier, so no rank frees a buffer another
        rank still maps."""
        self.barrier()
        err = None
        for a in self._imports:
            try:
                rc_ipc_release(a)
            except Exception as e:  # keep releasing the rest
                err = err or e
        self._imports.clear()
        self._dist.barrier(group=self.group)
        self.barriers += 1
        if err is not None:
            raise err

    # ------------------------------------------------------------ collectives
    def all_reduce(self, send: Sequence, recv: Sequence, op="sum", scale=1.0, dtype=None, n=None) -> None:
        """Every rank's recv = the all-reduce of the ranks' send buffers
        (this rank computes its chunk and writes it to every rank)."""
        self.barrier()
        rc_rank_all_reduce(send, recv, self.rank, n=n, dtype=dtype, op=op, scale=scale)
        self.barrier()

    def reduce_scatter(self, send: Sequence, recv_own, op="sum", scale=1.0, in_dtype=None, out_dtype=None,
                       n=None) -> None:
        """recv_own = this rank's shard of the reduce-scatter."""
        self.barrier()
        rc_rank_reduce_scatter(send, recv_own, self.rank, n=n, in_dtype=in_dtype, out_dtype=out_dtype, op=op,
                               scale=scale)
        self.barrier()

    def all_gather(self, send: Sequence, recv_own, dtype=None, n=None) -> None:
        """recv_own = the concatenation of every rank's shard."""
        self.barrier()
        rc_rank_all_gather(send, recv_own, self.rank, n=n, dtype=dtype)
        self.barrier()

    def ring_all_reduce(self, send: Sequence, recv: Sequence, ws: Optional[Sequence] = None, op="sum",
                        scale=1.0, dtype=None, n=None) -> None:
        """The literal ring: 2(p-1) steps, a barrier before each step and
        after the last.  bf16 needs ws (each rank's 2*ceil(n/p) fp32
        partials, shared like the other buffers)."""
        if self.p == 1:
            self.all_reduce(send, recv, op=op, scale=scale, dtype=dtype, n=n)
            return
        for step in range(2 * (self.p - 1)):
            self.barrier()
            rc_rank_ring_step(send, recv, self.rank, step, ws=ws, n=n, dtype=dtype, op=op, scale=scale)
        self.barrier()
