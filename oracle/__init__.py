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
    for f in ("rco_all_reduce", "rco_reduce_scatter", "rco_all_gather", "rco_reduce",
              "rco_broadcast", "rco_reduce_at", "rco_ring_all_reduce",
              "rco_hier_all_reduce"):
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
