"""Python binding of librankcoll (include/rankcoll.h): collective reductions over
p simulated ranks held in one GPU's memory.

This module only marshals arguments: device pointers, sizes, enums and the
stream go straight to the C ABI, and all work runs in the library's CUDA
kernels.  There is no CPU fallback -- importing fails if the shared library
has not been built (``python collective_rc_all_b200/build.py``).

Each ``rc_*`` function mirrors the C entry point of the same name.  Buffers
may be given as CUDA tensors (contiguous) or as integer device addresses; for
tensors, ``n`` and ``dtype`` default to what the tensors say.  ``stream``
defaults to torch's current stream.  A non-OK status raises RankCollError
carrying the library's message.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence, Union

__all__ = [
    "RankCollError", "lib", "library_path",
    "FP32", "BF16", "INT32", "SUM", "MAX", "MIN", "RING_LITERAL", "RING_ONESHOT",
    "HIER_FUSED", "HIER_STAGED",
    "rc_all_reduce", "rc_reduce_scatter", "rc_all_gather", "rc_reduce", "rc_broadcast",
    "rc_ring_all_reduce", "rc_ring_all_reduce_noalloc", "rc_hier_all_reduce", "rc_copy", "rc_reserve_workspace", "rc_workspace_bytes", "rc_check_buffer",
    "rc_probe_bounded_wait",
    "rc_rank_all_reduce", "rc_rank_reduce_scatter", "rc_rank_all_gather", "rc_rank_ring_step",
    "rc_ipc_handle", "rc_ipc_export", "rc_ipc_import", "rc_ipc_release",
    "rc_stream_status", "rc_launch_count", "rc_finalize", "rc_version", "rc_last_error",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
library_path = os.path.join(_HERE, "librankcoll.so")

if not os.path.exists(library_path):
    raise ImportError(
        f"librankcoll.so not found at {library_path}; build it with "
        "`python collective_rc_all_b200/build.py` (there is no CPU fallback)")

lib = ctypes.CDLL(library_path)

# enums (values fixed by include/rankcoll.h)
FP32, BF16, INT32 = 0, 1, 2
SUM, MAX, MIN = 0, 1, 2
RING_LITERAL, RING_ONESHOT = 0, 1
HIER_FUSED, HIER_STAGED = 0, 1
_STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported", 3: "CUDA error", 4: "timeout"}

_vpp = ctypes.POINTER(ctypes.c_void_p)
_sz, _i, _f, _vp = ctypes.c_size_t, ctypes.c_int, ctypes.c_float, ctypes.c_void_p


def _decl(name, args, res=ctypes.c_int):
    fn = getattr(lib, name)
    fn.argtypes = args
    fn.restype = res
    return fn


_decl("rc_all_reduce", [_vpp, _vpp, _i, _sz, _i, _i, _f, _vp])
_decl("rc_reduce_scatter", [_vpp, _vpp, _i, _sz, _i, _i, _i, _f, _vp])
_decl("rc_all_gather", [_vpp, _vpp, _i, _sz, _i, _vp])
_decl("rc_reduce", [_vpp, _vp, _i, _i, _sz, _i, _i, _f, _vp])
_decl("rc_broadcast", [_vp, _vpp, _i, _i, _sz, _i, _vp])
_decl("rc_ring_all_reduce", [_vpp, _vpp, _i, _sz, _i, _i, _f, _i, _vp])
_decl("rc_hier_all_reduce", [_vpp, _vpp, _i, _i, _sz, _i, _i, _f, _i, _vp])
_decl("rc_ring_all_reduce_noalloc", [_vpp, _vpp, _i, _sz, _i, _i, _f, _vp])
_decl("rc_copy", [_vp, _vp, _sz, _vp])


class rc_adamw_hparams(ctypes.Structure):
    """Mirror of the C struct rc_adamw_hparams."""
    _fields_ = [("lr", ctypes.c_float), ("beta1", ctypes.c_float), ("beta2", ctypes.c_float),
                ("eps", ctypes.c_float), ("weight_decay", ctypes.c_float), ("step", ctypes.c_int64)]


_hpp = ctypes.POINTER(rc_adamw_hparams)
_decl("rc_adamw_step", [_vp, _vp, _vp, _vp, _i, _sz, _hpp, _vp])
_decl("rc_zero1_step", [_vpp, _vpp, _vpp, _vpp, _vpp, _i, _sz, _i, _i, _f, _hpp, _vp])
_decl("rc_all_to_all", [_vpp, _vpp, _i, _sz, _i, _vp])
_szp = ctypes.POINTER(ctypes.c_size_t)
_ip = ctypes.POINTER(ctypes.c_int)
_decl("rc_plan_buckets", [_i, _szp, _sz, _sz, _ip, _ip])
_decl("rc_bucketer_create", [ctypes.POINTER(_vp), _vpp, _i, _i, _szp, _sz, _i, _f, _vp])
_decl("rc_bucketer_num_buckets", [_vp, _ip])
_decl("rc_bucketer_bucket", [_vp, _i, _ip, _ip, _szp, _szp])
_decl("rc_bucketer_ready", [_vp, _i, _vp])
_decl("rc_bucketer_flush", [_vp, _vp])
_decl("rc_bucketer_destroy", [_vp])
_decl("rc_all_to_all_v", [_vpp, _vpp, _i, ctypes.POINTER(ctypes.c_size_t), _i, _vp])
_decl("rc_rank_all_reduce", [_vpp, _vpp, _i, _i, _sz, _i, _i, _f, _vp])
_decl("rc_rank_reduce_scatter", [_vpp, _vp, _i, _i, _sz, _i, _i, _i, _f, _vp])
_decl("rc_rank_all_gather", [_vpp, _vp, _i, _i, _sz, _i, _vp])
_decl("rc_rank_ring_step", [_vpp, _vpp, _vpp, _i, _i, _i, _sz, _i, _i, _f, _vp])


class rc_ipc_handle(ctypes.Structure):
    """Mirror of the C struct rc_ipc_handle (plain bytes: bytes(h) travels
    between processes, rc_ipc_handle.from_buffer_copy(b) restores it)."""
    _fields_ = [("ipc", ctypes.c_ubyte * 64), ("offset", ctypes.c_uint64), ("bytes", ctypes.c_uint64),
                ("device", ctypes.c_int32), ("pid", ctypes.c_int32)]


_decl("rc_ipc_export", [_vp, _sz, ctypes.POINTER(rc_ipc_handle)])
_decl("rc_ipc_import", [ctypes.POINTER(rc_ipc_handle), ctypes.POINTER(_vp)])
_decl("rc_ipc_release", [_vp])
_decl("rc_reserve_workspace", [_sz, _vp])
_decl("rc_workspace_bytes", [ctypes.POINTER(_sz), ctypes.POINTER(_sz)])
_decl("rc_check_buffer", [_vp, _sz])
_decl("rc_probe_bounded_wait", [ctypes.c_uint64, _vp])
_decl("rc_stream_status", [_vp])
_decl("rc_status_string", [_i], ctypes.c_char_p)
_decl("rc_last_error", [], ctypes.c_char_p)
_decl("rc_launch_count", [], ctypes.c_uint64)
_decl("rc_finalize", [])
_decl("rc_version", [])


class RankCollError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = lib.rc_last_error().decode(errors="replace")
        super().__init__(f"{where}: {_STATUS.get(status, status)}: {msg}")


def _check(status: int, where: str) -> None:
    if status != 0:
        raise RankCollError(status, where)


# ---------------------------------------------------------------- marshalling
_DT_NAMES = {"f32": FP32, "fp32": FP32, "float32": FP32, "bf16": BF16, "bfloat16": BF16,
             "i32": INT32, "int32": INT32}
_OP_NAMES = {"sum": SUM, "max": MAX, "min": MIN}


def _is_tensor(x) -> bool:
    return hasattr(x, "data_ptr") and hasattr(x, "dtype")


def _dt(dtype, like=None) -> int:
    if dtype is None:
        if like is None or not _is_tensor(like):
            raise ValueError("dtype is required when buffers are raw addresses")
        import torch
        m = {torch.float32: FP32, torch.bfloat16: BF16, torch.int32: INT32}
        if like.dtype not in m:
            raise TypeError(f"unsupported tensor dtype {like.dtype}")
        return m[like.dtype]
    if isinstance(dtype, str):
        return _DT_NAMES[dtype.lower()]
    if isinstance(dtype, int):
        return dtype
    import torch
    return {torch.float32: FP32, torch.bfloat16: BF16, torch.int32: INT32}[dtype]


def _op(op) -> int:
    return _OP_NAMES[op.lower()] if isinstance(op, str) else int(op)


def _addr(x) -> int:
    if _is_tensor(x):
        if not x.is_cuda:
            raise ValueError("tensor is not on a CUDA device")
        if not x.is_contiguous():
            raise ValueError("tensor must be contiguous")
        return x.data_ptr()
    return int(x)


def _ptrs(xs: Sequence) -> "ctypes.Array":
    return (ctypes.c_void_p * len(xs))(*[_addr(x) for x in xs])


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if hasattr(stream, "cuda_stream"):
        return stream.cuda_stream
    return int(stream)


def _numel(x, n):
    if n is not None:
        return int(n)
    if _is_tensor(x):
        return x.numel()
    raise ValueError("n is required when buffers are raw addresses")


Buf = Union[int, "torch.Tensor"]  # noqa: F821


# ---------------------------------------------------------------- entry points
def rc_all_reduce(send: Sequence[Buf], recv: Sequence[Buf], n=None, dtype=None, op="sum",
                  scale=1.0, stream=None):
    p = len(send)
    _check(lib.rc_all_reduce(_ptrs(send), _ptrs(recv), p, _numel(send[0], n), _dt(dtype, send[0]),
                             _op(op), scale, _stream(stream)), "rc_all_reduce")


def rc_reduce_scatter(send: Sequence[Buf], recv: Sequence[Buf], n=None, in_dtype=None,
                      out_dtype=None, op="sum", scale=1.0, stream=None):
    p = len(send)
    _check(lib.rc_reduce_scatter(_ptrs(send), _ptrs(recv), p, _numel(send[0], n),
                                 _dt(in_dtype, send[0]), _dt(out_dtype, recv[0]), _op(op), scale,
                                 _stream(stream)), "rc_reduce_scatter")


def rc_all_gather(send: Sequence[Buf], recv: Sequence[Buf], n=None, dtype=None, stream=None):
    p = len(send)
    nn = int(n) if n is not None else _numel(recv[0], None)
    _check(lib.rc_all_gather(_ptrs(send), _ptrs(recv), p, nn, _dt(dtype, send[0]), _stream(stream)),
           "rc_all_gather")


def rc_reduce(send: Sequence[Buf], recv_root: Buf, root=0, n=None, dtype=None, op="sum",
              scale=1.0, stream=None):
    p = len(send)
    _check(lib.rc_reduce(_ptrs(send), _addr(recv_root), p, root, _numel(send[0], n),
                         _dt(dtype, send[0]), _op(op), scale, _stream(stream)), "rc_reduce")


def rc_broadcast(send_root: Buf, recv: Sequence[Buf], root=0, n=None, dtype=None, stream=None):
    p = len(recv)
    _check(lib.rc_broadcast(_addr(send_root), _ptrs(recv), p, root, _numel(send_root, n),
                            _dt(dtype, send_root), _stream(stream)), "rc_broadcast")


def rc_ring_all_reduce(send: Sequence[Buf], recv: Sequence[Buf], n=None, dtype=None, op="sum",
                       scale=1.0, variant=RING_LITERAL, stream=None):
    p = len(send)
    v = {"literal": RING_LITERAL, "oneshot": RING_ONESHOT}.get(variant, variant)
    _check(lib.rc_ring_all_reduce(_ptrs(send), _ptrs(recv), p, _numel(send[0], n),
                                  _dt(dtype, send[0]), _op(op), scale, int(v), _stream(stream)),
           "rc_ring_all_reduce")


def rc_ring_all_reduce_noalloc(send: Sequence[Buf], recv: Sequence[Buf], n=None, dtype=None,
                               op="sum", scale=1.0, stream=None):
    """Literal ring all-reduce that allocates nothing (fixed scratch for bf16)."""
    p = len(send)
    _check(lib.rc_ring_all_reduce_noalloc(_ptrs(send), _ptrs(recv), p, _numel(send[0], n),
                                          _dt(dtype, send[0]), _op(op), scale, _stream(stream)),
           "rc_ring_all_reduce_noalloc")


def rc_hier_all_reduce(send: Sequence[Buf], recv: Sequence[Buf], group_size: int, n=None,
                       dtype=None, op="sum", scale=1.0, variant=HIER_FUSED, stream=None):
    p = len(send)
    v = {"fused": HIER_FUSED, "staged": HIER_STAGED}.get(variant, variant)
    _check(lib.rc_hier_all_reduce(_ptrs(send), _ptrs(recv), p, group_size, _numel(send[0], n),
                                  _dt(dtype, send[0]), _op(op), scale, int(v), _stream(stream)),
           "rc_hier_all_reduce")


# ---------------------------------------------------------------- rank view
# One rank's share of a collective (rank-per-GPU execution): the buffer lists
# hold the p ranks' buffers as this process addresses them -- its own tensor
# and the other ranks' imported addresses (integers).  dtype and n are
# required when the own buffer is a raw address.
def _own(xs: Sequence, rank: int):
    """The buffer that supplies n and dtype defaults: this rank's own (a
    tensor), or the first one when rank is out of range (the library then
    rejects the call)."""
    return xs[rank] if 0 <= rank < len(xs) else xs[0]


def rc_rank_all_reduce(send: Sequence[Buf], recv: Sequence[Buf], rank: int, n=None, dtype=None, op="sum",
                       scale=1.0, stream=None):
    p = len(send)
    own = _own(send, rank)
    _check(lib.rc_rank_all_reduce(_ptrs(send), _ptrs(recv), p, rank, _numel(own, n), _dt(dtype, own), _op(op),
                                  scale, _stream(stream)), "rc_rank_all_reduce")


def rc_rank_reduce_scatter(send: Sequence[Buf], recv_own: Buf, rank: int, n=None, in_dtype=None,
                           out_dtype=None, op="sum", scale=1.0, stream=None):
    p = len(send)
    own = _own(send, rank)
    _check(lib.rc_rank_reduce_scatter(_ptrs(send), _addr(recv_own), p, rank, _numel(own, n),
                                      _dt(in_dtype, own), _dt(out_dtype, recv_own), _op(op), scale,
                                      _stream(stream)), "rc_rank_reduce_scatter")


def rc_rank_all_gather(send: Sequence[Buf], recv_own: Buf, rank: int, n=None, dtype=None, stream=None):
    p = len(send)
    _check(lib.rc_rank_all_gather(_ptrs(send), _addr(recv_own), p, rank, _numel(recv_own, n),
                                  _dt(dtype, recv_own), _stream(stream)), "rc_rank_all_gather")


def rc_rank_ring_step(send: Sequence[Buf], recv: Sequence[Buf], rank: int, step: int, ws=None, n=None,
                      dtype=None, op="sum", scale=1.0, stream=None):
    p = len(send)
    own = _own(send, rank)
    wsp = _ptrs(ws) if ws is not None else None
    _check(lib.rc_rank_ring_step(_ptrs(send), _ptrs(recv), wsp, p, rank, step, _numel(own, n), _dt(dtype, own),
                                 _op(op), scale, _stream(stream)), "rc_rank_ring_step")


def rc_ipc_export(buf: Buf, nbytes=None) -> bytes:
    """Describe a device buffer (tensor or address + nbytes) for another process."""
    if nbytes is None:
        if not _is_tensor(buf):
            raise ValueError("nbytes is required for a raw address")
        nbytes = buf.numel() * buf.element_size()
    h = rc_ipc_handle()
    _check(lib.rc_ipc_export(_addr(buf), int(nbytes), ctypes.byref(h)), "rc_ipc_export")
    return bytes(h)


def rc_ipc_import(handle: bytes) -> int:
    """Map another process's exported buffer; returns its address here."""
    h = rc_ipc_handle.from_buffer_copy(handle)
    out = ctypes.c_void_p()
    _check(lib.rc_ipc_import(ctypes.byref(h), ctypes.byref(out)), "rc_ipc_import")
    return int(out.value)


def rc_ipc_release(addr: int) -> None:
    _check(lib.rc_ipc_release(int(addr)), "rc_ipc_release")


def _hparams(lr, beta1, beta2, eps, weight_decay, step):
    return rc_adamw_hparams(lr, beta1, beta2, eps, weight_decay, int(step))


def rc_adamw_step(param: Buf, exp_avg: Buf, exp_avg_sq: Buf, grad: Buf, n=None, grad_dtype=None,
                  lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.0, step=1, stream=None):
    hp = _hparams(lr, beta1, beta2, eps, weight_decay, step)
    _check(lib.rc_adamw_step(_addr(param), _addr(exp_avg), _addr(exp_avg_sq), _addr(grad),
                             _dt(grad_dtype, grad), _numel(param, n), ctypes.byref(hp),
                             _stream(stream)), "rc_adamw_step")


def rc_zero1_step(grads: Sequence[Buf], params: Sequence[Buf], master: Sequence[Buf],
                  exp_avg: Sequence[Buf], exp_avg_sq: Sequence[Buf], n=None, grad_dtype=None,
                  param_dtype=None, scale=None, lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8,
                  weight_decay=0.0, step=1, stream=None):
    p = len(grads)
    hp = _hparams(lr, beta1, beta2, eps, weight_decay, step)
    _check(lib.rc_zero1_step(_ptrs(grads), _ptrs(params), _ptrs(master), _ptrs(exp_avg),
                             _ptrs(exp_avg_sq), p, _numel(grads[0], n), _dt(grad_dtype, grads[0]),
                             _dt(param_dtype, params[0]), 1.0 / p if scale is None else scale,
                             ctypes.byref(hp), _stream(stream)), "rc_zero1_step")


def rc_all_to_all(send: Sequence[Buf], recv: Sequence[Buf], n=None, dtype=None, stream=None):
    p = len(send)
    _check(lib.rc_all_to_all(_ptrs(send), _ptrs(recv), p, _numel(send[0], n), _dt(dtype, send[0]),
                             _stream(stream)), "rc_all_to_all")


def rc_all_to_all_v(send: Sequence[Buf], recv: Sequence[Buf], counts, dtype=None, stream=None):
    """counts: p x p element counts (nested sequence or array), counts[r][q] = r -> q."""
    p = len(send)
    flat = [int(c) for row in counts for c in row]
    if len(flat) != p * p:
        raise ValueError("counts must be p x p")
    arr = (ctypes.c_size_t * (p * p))(*flat)
    _check(lib.rc_all_to_all_v(_ptrs(send), _ptrs(recv), p, arr, _dt(dtype, send[0]), _stream(stream)),
           "rc_all_to_all_v")


def rc_plan_buckets(numel: Sequence[int], elem_bytes: int, bucket_bytes: int):
    """Bucket index of every tensor under the bucketer's rule (host only)."""
    n = len(numel)
    arr = (ctypes.c_size_t * max(1, n))(*[int(x) for x in numel])
    out = (ctypes.c_int * max(1, n))()
    nb = ctypes.c_int()
    _check(lib.rc_plan_buckets(n, arr, elem_bytes, min(int(bucket_bytes), 2**64 - 1), out,
                               ctypes.byref(nb)), "rc_plan_buckets")
    return [out[i] for i in range(n)], nb.value


class Bucketer:
    """Gradient bucketing (rc_bucketer_*): p flat gradient buffers, tensors in
    ready order; ready(t, stream) after tensor t's gradients are written on
    every rank, flush(stream) at the end of the step."""

    def __init__(self, flat: Sequence[Buf], numel: Sequence[int], bucket_bytes: int, dtype=None,
                 scale=None, comm_stream=None):
        p = len(flat)
        self.numel = [int(x) for x in numel]
        arr = (ctypes.c_size_t * len(numel))(*self.numel)
        h = ctypes.c_void_p()
        self._comm = comm_stream  # keep the stream object alive
        _check(lib.rc_bucketer_create(ctypes.byref(h), _ptrs(flat), p, len(numel), arr,
                                      min(int(bucket_bytes), 2**64 - 1), _dt(dtype, flat[0]),
                                      1.0 / p if scale is None else scale, _stream(comm_stream)),
               "rc_bucketer_create")
        self.h = h.value

    def buckets(self):
        nb = ctypes.c_int()
        _check(lib.rc_bucketer_num_buckets(self.h, ctypes.byref(nb)), "rc_bucketer_num_buckets")
        out = []
        for k in range(nb.value):
            t0, t1, e0, ne = ctypes.c_int(), ctypes.c_int(), ctypes.c_size_t(), ctypes.c_size_t()
            _check(lib.rc_bucketer_bucket(self.h, k, ctypes.byref(t0), ctypes.byref(t1), ctypes.byref(e0),
                                          ctypes.byref(ne)), "rc_bucketer_bucket")
            out.append((t0.value, t1.value, e0.value, ne.value))
        return out

    def ready(self, tensor: int, stream=None):
        _check(lib.rc_bucketer_ready(self.h, tensor, _stream(stream)), "rc_bucketer_ready")

    def flush(self, stream=None):
        _check(lib.rc_bucketer_flush(self.h, _stream(stream)), "rc_bucketer_flush")

    def close(self):
        if self.h:
            lib.rc_bucketer_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def rc_copy(src: Buf, dst: Buf, nbytes=None, stream=None):
    if nbytes is None:
        nbytes = src.numel() * src.element_size()
    _check(lib.rc_copy(_addr(src), _addr(dst), int(nbytes), _stream(stream)), "rc_copy")


def rc_check_buffer(buf: Buf, nbytes: int) -> None:
    """Raise unless [buf, buf + nbytes) is device memory of the current device
    inside one allocation (no launch)."""
    _check(lib.rc_check_buffer(_addr(buf), int(nbytes)), "rc_check_buffer")


def rc_probe_bounded_wait(limit_ns: int, stream=None) -> None:
    """Launch the failure-path self test (a bounded wait that runs out); the
    next rc_stream_status on that stream reports the timeout."""
    _check(lib.rc_probe_bounded_wait(int(limit_ns), _stream(stream)), "rc_probe_bounded_wait")


def rc_reserve_workspace(nbytes: int, stream=None):
    _check(lib.rc_reserve_workspace(int(nbytes), _stream(stream)), "rc_reserve_workspace")


def rc_workspace_bytes():
    """(live, retired): bytes of the current device's workspace block and of
    the blocks kept alive for captured graphs."""
    live, retired = ctypes.c_size_t(0), ctypes.c_size_t(0)
    _check(lib.rc_workspace_bytes(ctypes.byref(live), ctypes.byref(retired)), "rc_workspace_bytes")
    return live.value, retired.value


def rc_stream_status(stream=None) -> int:
    """Synchronise the stream; raise on an asynchronous error or a device wait
    that gave up; return 0 otherwise."""
    st = lib.rc_stream_status(_stream(stream))
    _check(st, "rc_stream_status")
    return st


def rc_launch_count() -> int:
    return int(lib.rc_launch_count())


def rc_finalize():
    _check(lib.rc_finalize(), "rc_finalize")


def rc_version() -> int:
    return int(lib.rc_version())


def rc_last_error() -> str:
    return lib.rc_last_error().decode(errors="replace")
