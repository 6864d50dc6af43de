"""CPU oracle for the simulated-rank collectives -- TEST INFRASTRUCTURE.

Only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline / reference
leg may import this package.  The CUDA library never imports it, and it never
imports the CUDA library.  All arithmetic lives in rc_oracle.c (plain C, one
thread); this module only marshals numpy arrays to it.

Conventions (same as the C file):
  * rank buffers are numpy arrays: float32 for "f32", uint16 bit patterns for
    "bf16", int32 for "i32";
  * ``n`` is the full per-rank vector length; reduce_scatter / all_gather
    shards are ``n // p`` long.

Parity is pinned by tests/test_oracle_*.py (worked example, closed forms,
identities, literal ring vs direct fold, brute force, bf16 rounding,
traffic counts).
"""
from __future__ import annotations

import ctypes
import os
from typing import List, Optional, Sequence

import numpy as np

from . import build as _build

DT = {"f32": 0, "bf16": 1, "i32": 2}
OP = {"sum": 0, "max": 1, "min": 2}
NP_DT = {"f32": np.float32, "bf16": np.uint16, "i32": np.int32}

_lib = None


def _bind(path: str) -> ctypes.CDLL:
    """Load an oracle shared library and declare its C signatures."""
    L = ctypes.CDLL(path)
    vpp = ctypes.POINTER(ctypes.c_void_p)
    u64p = ctypes.POINTER(ctypes.c_uint64)
    sz, ci, cf = ctypes.c_size_t, ctypes.c_int, ctypes.c_float
    L.rco_all_reduce.argtypes = [vpp, vpp, ci, sz, ci, ci, cf]
    L.rco_reduce_scatter.argtypes = [vpp, vpp, ci, sz, ci, ci, ci, cf]
    L.rco_all_gather.argtypes = [vpp, vpp, ci, sz, ci]
    L.rco_reduce.argtypes = [vpp, ctypes.c_void_p, ci, ci, sz, ci, ci, cf]
    L.rco_broadcast.argtypes = [ctypes.c_void_p, vpp, ci, ci, sz, ci]
    L.rco_reduce_at.argtypes = [vpp, ci, sz, ci, ci, ci, cf, u64p, sz, ctypes.c_void_p]
    L.rco_ring_all_reduce.argtypes = [vpp, vpp, ci, sz, ci, ci, cf, u64p, u64p]
    L.rco_hier_all_reduce.argtypes = [vpp, vpp, ci, ci, sz, ci, ci, cf, u64p]
    L.rco_f32_to_bf16.argtypes = [ctypes.c_float]
    L.rco_f32_to_bf16.restype = ctypes.c_uint16
    L.rco_bf16_to_f32.argtypes = [ctypes.c_uint16]
    L.rco_bf16_to_f32.restype = ctypes.c_float
    L.rco_f32_to_bf16_n.argtypes = [ctypes.c_void_p, ctypes.c_void_p, sz]
    L.rco_f32_to_bf16_n.restype = None
    fp = ctypes.POINTER(ctypes.c_float)
    L.rco_adamw.argtypes = [fp, fp, fp, ctypes.c_void_p, ci, sz, cf, cf, cf, cf, cf, ctypes.c_int64]
    L.rco_all_to_all_v.argtypes = [vpp, vpp, ci, u64p, ci, u64p]
    for f in ("rco_all_reduce", "rco_reduce_scatter", "rco_all_gather", "rco_reduce",
              "rco_broadcast", "rco_reduce_at", "rco_ring_all_reduce",
              "rco_hier_all_reduce", "rco_adamw", "rco_all_to_all_v"):
        getattr(L, f).restype = ctypes.c_int
    return L


_override = None


def lib() -> ctypes.CDLL:
    """The library every function below calls (the built oracle, unless a
    test has swapped in a deliberately broken copy with ``use_library``)."""
    global _lib
    if _override is not None:
        return _override
    if _lib is None:
        # RC_ORACLE_LIB lets a test run the pins against another build of the
        # oracle source (a copy with a planted mistake).
        _lib = _bind(os.environ.get("RC_ORACLE_LIB") or _build.build())
    return _lib


class use_library:
    """Context manager: route this module's calls to another build of the
    oracle source (tests use it to check that planted mistakes are caught)."""

    def __init__(self, path: str):
        self.L = _bind(path)

    def __enter__(self):
        global _override
        self._prev, _override = _override, self.L
        return self.L

    def __exit__(self, *exc):
        global _override
        _override = self._prev
        return False


class OracleError(RuntimeError):
    pass


def _ptrs(arrs: Sequence[np.ndarray]):
    return (ctypes.c_void_p * len(arrs))(*[a.ctypes.data for a in arrs])


def _check(rc: int, what: str):
    if rc != 0:
        raise OracleError(f"{what}: oracle returned {rc}")


def _contig(xs: Sequence[np.ndarray], dt: str) -> List[np.ndarray]:
    out = []
    for x in xs:
        x = np.ascontiguousarray(x)
        if x.dtype != NP_DT[dt]:
            raise TypeError(f"expected {NP_DT[dt]} for {dt}, got {x.dtype}")
        out.append(x)
    return out


def all_reduce(xs, dt="f32", op="sum", scale=1.0):
    xs = _contig(xs, dt)
    p, n = len(xs), xs[0].size
    ys = [np.empty(n, NP_DT[dt]) for _ in range(p)]
    _check(lib().rco_all_reduce(_ptrs(xs), _ptrs(ys), p, n, DT[dt], OP[op], scale), "all_reduce")
    return ys


def reduce_scatter(xs, in_dt="f32", out_dt=None, op="sum", scale=1.0):
    out_dt = out_dt or in_dt
    xs = _contig(xs, in_dt)
    p, n = len(xs), xs[0].size
    ys = [np.empty(n // p, NP_DT[out_dt]) for _ in range(p)]
    _check(lib().rco_reduce_scatter(_ptrs(xs), _ptrs(ys), p, n, DT[in_dt], DT[out_dt],
                                    OP[op], scale), "reduce_scatter")
    return ys


def all_gather(shards, dt="f32"):
    shards = _contig(shards, dt)
    p = len(shards)
    n = shards[0].size * p
    ys = [np.empty(n, NP_DT[dt]) for _ in range(p)]
    _check(lib().rco_all_gather(_ptrs(shards), _ptrs(ys), p, n, DT[dt]), "all_gather")
    return ys


def reduce(xs, root=0, dt="f32", op="sum", scale=1.0):
    xs = _contig(xs, dt)
    p, n = len(xs), xs[0].size
    y = np.empty(n, NP_DT[dt])
    _check(lib().rco_reduce(_ptrs(xs), y.ctypes.data, p, root, n, DT[dt], OP[op], scale),
           "reduce")
    return y


def broadcast(x, p, root=0, dt="f32"):
    x = _contig([x], dt)[0]
    ys = [np.empty(x.size, NP_DT[dt]) for _ in range(p)]
    _check(lib().rco_broadcast(x.ctypes.data, _ptrs(ys), p, root, x.size, DT[dt]), "broadcast")
    return ys


def reduce_at(xs, idx, in_dt="f32", out_dt=None, op="sum", scale=1.0):
    """Reduced values y[idx] (out_dt) of the full vectors ``xs``."""
    out_dt = out_dt or in_dt
    xs = _contig(xs, in_dt)
    idx = np.ascontiguousarray(idx, dtype=np.uint64)
    out = np.empty(idx.size, NP_DT[out_dt])
    _check(lib().rco_reduce_at(_ptrs(xs), len(xs), xs[0].size, DT[in_dt], DT[out_dt], OP[op],
                               scale, idx.ctypes.data_as(ctypes.POINTER(ctypes.c_uint64)),
                               idx.size, out.ctypes.data), "reduce_at")
    return out


class RingStats:
    def __init__(self, p):
        self.elems_sent = np.zeros(p, np.uint64)
        self.steps = np.zeros(1, np.uint64)


def ring_all_reduce(xs, dt="f32", op="sum", scale=1.0, stats: Optional[RingStats] = None):
    xs = _contig(xs, dt)
    p, n = len(xs), xs[0].size
    ys = [np.empty(n, NP_DT[dt]) for _ in range(p)]
    st = stats or RingStats(p)
    u64p = ctypes.POINTER(ctypes.c_uint64)
    _check(lib().rco_ring_all_reduce(_ptrs(xs), _ptrs(ys), p, n, DT[dt], OP[op], scale,
                                     st.elems_sent.ctypes.data_as(u64p),
                                     st.steps.ctypes.data_as(u64p)), "ring_all_reduce")
    return ys


def hier_all_reduce(xs, group_size, dt="f32", op="sum", scale=1.0, traffic=None):
    """``traffic``: optional uint64 array of 4 counters (see rc_oracle.c)."""
    xs = _contig(xs, dt)
    p, n = len(xs), xs[0].size
    ys = [np.empty(n, NP_DT[dt]) for _ in range(p)]
    t = traffic if traffic is not None else np.zeros(4, np.uint64)
    _check(lib().rco_hier_all_reduce(_ptrs(xs), _ptrs(ys), p, group_size, n, DT[dt], OP[op],
                                     scale, t.ctypes.data_as(ctypes.POINTER(ctypes.c_uint64))),
           "hier_all_reduce")
    return ys


def f32_to_bf16(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bits, round half to even (the oracle's C routine)."""
    x = np.ascontiguousarray(x, dtype=np.float32).ravel()
    y = np.empty(x.size, np.uint16)
    lib().rco_f32_to_bf16_n(x.ctypes.data, y.ctypes.data, x.size)
    return y


def bf16_to_f32(h: np.ndarray) -> np.ndarray:
    h = np.ascontiguousarray(h, dtype=np.uint16).ravel()
    return (h.astype(np.uint32) << 16).view(np.float32)


# ---------------------------------------------------------------- optimizer
def adamw(theta, m, v, g, grad_dt="f32", lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8,
          weight_decay=0.0, step=1):
    """One AdamW step (rc_oracle.c rco_adamw); returns new (theta, m, v)."""
    th = np.array(theta, dtype=np.float32, copy=True).ravel()
    mm = np.array(m, dtype=np.float32, copy=True).ravel()
    vv = np.array(v, dtype=np.float32, copy=True).ravel()
    gg = np.ascontiguousarray(g, dtype=NP_DT[grad_dt]).ravel()
    if not (th.size == mm.size == vv.size == gg.size):
        raise ValueError("adamw: sizes differ")
    fp = ctypes.POINTER(ctypes.c_float)
    _check(lib().rco_adamw(th.ctypes.data_as(fp), mm.ctypes.data_as(fp), vv.ctypes.data_as(fp),
                           gg.ctypes.data, DT[grad_dt], th.size, lr, beta1, beta2, eps,
                           weight_decay, int(step)), "adamw")
    return th, mm, vv


def zero1_step(grads, master, exp_avg, exp_avg_sq, grad_dt="f32", param_dt="bf16",
               scale=None, **hp):
    """ZeRO-1 sharded optimizer step over p simulated ranks, by composition:
    reduce_scatter of the gradients (fp32 out, x scale, default 1/p), AdamW on
    each rank's own shard (fp32 master weights and moments of n/p elements),
    then all_gather of the updated weights cast to param_dt.  Returns
    (params per rank, master, exp_avg, exp_avg_sq) -- new arrays."""
    p = len(grads)
    if scale is None:
        scale = 1.0 / p
    g = reduce_scatter(grads, grad_dt, "f32", "sum", scale)
    out_m, out_a, out_s = [], [], []
    for r in range(p):
        th, mm, vv = adamw(master[r], exp_avg[r], exp_avg_sq[r], g[r], "f32", **hp)
        out_m.append(th)
        out_a.append(mm)
        out_s.append(vv)
    shards = [th if param_dt == "f32" else f32_to_bf16(th) for th in out_m]
    return all_gather(shards, param_dt), out_m, out_a, out_s


def sharded_owner_step(grads, master, exp_avg, exp_avg_sq, grad_dt="f32", param_dt="bf16",
                       scale=None, **hp):
    """The ShardedOptimizer form: tensor t (lists of per-rank arrays) is owned
    by rank t % p; every gradient is all-reduced (x scale, default 1/p), the
    owner runs AdamW on its fp32 master copy and moments, and the result is
    broadcast from the owner.  grads[t][r]: rank r's gradient of tensor t;
    master / exp_avg / exp_avg_sq[t]: the owner's state of tensor t.
    Returns (params[t][r], master, exp_avg, exp_avg_sq) -- new arrays."""
    T = len(grads)
    p = len(grads[0])
    if scale is None:
        scale = 1.0 / p
    params, out_m, out_a, out_s = [], [], [], []
    for t in range(T):
        owner = t % p
        g = all_reduce(grads[t], grad_dt, "sum", scale)
        g32 = g[owner] if grad_dt == "f32" else bf16_to_f32(g[owner])
        th, mm, vv = adamw(master[t], exp_avg[t], exp_avg_sq[t], g32, "f32", **hp)
        out_m.append(th)
        out_a.append(mm)
        out_s.append(vv)
        w = th if param_dt == "f32" else f32_to_bf16(th)
        params.append(broadcast(w, p, owner, param_dt))
    return params, out_m, out_a, out_s


# ---------------------------------------------------------------- all-to-all
def all_to_all_v(sends, counts, traffic=None):
    """sends[r]: rank r's outgoing blocks in destination order; counts[r][q]:
    elements r sends to q (any numpy dtype, copied bit for bit).  Returns the
    p receive buffers (incoming blocks in source order).  traffic, if a list
    of 2, gets [bytes staying on their rank, bytes crossing ranks] added."""
    p = len(sends)
    cnt = np.ascontiguousarray(counts, dtype=np.uint64).reshape(p, p)
    dt = sends[0].dtype
    xs = [np.ascontiguousarray(x) for x in sends]
    for r in range(p):
        if xs[r].dtype != dt or xs[r].size < int(cnt[r].sum()):
            raise ValueError("all_to_all_v: send buffer too short or of another dtype")
    outs = [np.empty(int(cnt[:, q].sum()), dt) for q in range(p)]
    tr = np.zeros(2, np.uint64)
    u64p = ctypes.POINTER(ctypes.c_uint64)
    _check(lib().rco_all_to_all_v(_ptrs(xs), _ptrs(outs), p, cnt.ctypes.data_as(u64p), dt.itemsize,
                                  tr.ctypes.data_as(u64p)), "all_to_all_v")
    if traffic is not None:
        traffic[0] += int(tr[0])
        traffic[1] += int(tr[1])
    return outs


def all_to_all(sends, traffic=None):
    """Equal splits: n = p*m elements per rank, block q of rank r -> slot r of rank q."""
    p = len(sends)
    n = sends[0].size
    if n % p:
        raise ValueError("all_to_all: n must be a multiple of p")
    return all_to_all_v(sends, np.full((p, p), n // p, np.uint64), traffic)
