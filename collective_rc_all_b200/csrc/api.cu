// api.cu -- the extern "C" entry points of librankcoll (include/rankcoll.h):
// argument validation, aliasing rules, workspace management, dispatch.
//
// Every check happens on the host before anything is enqueued, so a bad call
// returns an error code and never reaches the GPU.  Device pointers are
// checked against the allocation that contains them (driver address-range
// query): a host pointer, a pointer from another device, or a buffer too small
// for the requested elements is RC_ERR_INVALID_ARG.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <vector>

#include <unistd.h>

#include "../../include/rankcoll.h"
#include "common.cuh"
#include "internal.h"

namespace rc {

// ---------------------------------------------------------------- bookkeeping
namespace {
thread_local char t_last_error[512] = "";
std::atomic<uint64_t> g_launches{0};
constexpr int kMaxDevices = 64;
std::atomic<int> g_sm_count[kMaxDevices];

rc_status fail(rc_status st, const char *fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(t_last_error, sizeof t_last_error, fmt, ap);
  va_end(ap);
  return st;
}

rc_status cuda_fail(cudaError_t e, const char *what) {
  return fail(RC_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}
}  // namespace

rc_status report_error(rc_status st, const char *msg) {
  snprintf(t_last_error, sizeof t_last_error, "%s", msg);
  return st;
}

int device_sm_count() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
  int v = g_sm_count[dev].load(std::memory_order_relaxed);
  if (v <= 0) {
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) v = 148;
    g_sm_count[dev].store(v, std::memory_order_relaxed);
  }
  return v;
}

bool pdl_enabled() {
  static const bool on = env_int("RC_PDL", 1) != 0;
  return on;
}

void note_launches(int k) { g_launches.fetch_add((uint64_t)k, std::memory_order_relaxed); }

int env_int(const char *name, int dflt) {
  const char *v = getenv(name);
  if (!v || !*v) return dflt;
  return atoi(v);
}

// ---------------------------------------------------------------- pointer checks
namespace {

typedef CUresult (*MemGetAddressRangeFn)(CUdeviceptr *, size_t *, CUdeviceptr);
MemGetAddressRangeFn address_range_fn() {
  static MemGetAddressRangeFn fn = []() -> MemGetAddressRangeFn {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<MemGetAddressRangeFn>(p);
  }();
  return fn;
}

// [ptr, ptr+bytes) must be device (or managed) memory of the current device,
// inside one allocation.
// peer_ok: the memory may also belong to another device that the current
// device can access (a peer mapping).
rc_status check_device_range(const void *ptr, size_t bytes, const char *what, int idx, bool peer_ok = false) {
  if (ptr == nullptr) return fail(RC_ERR_INVALID_ARG, "%s[%d] is NULL", what, idx);
  cudaPointerAttributes at{};
  cudaError_t e = cudaPointerGetAttributes(&at, ptr);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(RC_ERR_INVALID_ARG, "%s[%d]=%p is not a CUDA pointer (%s)", what, idx, ptr,
                cudaGetErrorString(e));
  }
  if (at.type != cudaMemoryTypeDevice && at.type != cudaMemoryTypeManaged)
    return fail(RC_ERR_INVALID_ARG, "%s[%d]=%p is not device memory", what, idx, ptr);
  int dev = -1;
  cudaGetDevice(&dev);
  if (at.type == cudaMemoryTypeDevice && at.device != dev) {
    int can = 0;
    if (!peer_ok || cudaDeviceCanAccessPeer(&can, dev, at.device) != cudaSuccess || !can) {
      cudaGetLastError();
      return fail(RC_ERR_INVALID_ARG, "%s[%d]=%p lives on device %d, current device is %d%s", what, idx,
                  ptr, at.device, dev, peer_ok ? ", which cannot access it" : "");
    }
  }
  if (env_int("RC_SKIP_RANGE_CHECK", 0)) return RC_OK;
  MemGetAddressRangeFn fn = address_range_fn();
  if (fn) {
    CUdeviceptr base = 0;
    size_t size = 0;
    if (fn(&base, &size, (CUdeviceptr)(uintptr_t)ptr) == CUDA_SUCCESS) {
      const uintptr_t p = (uintptr_t)ptr;
      if (p < (uintptr_t)base || p - (uintptr_t)base > size || bytes > size - (p - (uintptr_t)base))
        return fail(RC_ERR_INVALID_ARG,
                    "%s[%d]=%p: %zu bytes run past the end of its allocation (%zu bytes at %p)", what,
                    idx, ptr, bytes, size, (void *)base);
    }
  }
  return RC_OK;
}

struct Buf {
  uintptr_t lo, hi;   // byte range
  intptr_t origin;    // address of global element 0 under this buffer's indexing
  int esz;
  int rank;
  bool out;
  const char *what;
  int idx;
};

Buf make_buf(const void *p, uint64_t elems, int esz, uint64_t index0, int rank, bool out,
             const char *what, int idx) {
  Buf b;
  b.lo = (uintptr_t)p;
  b.hi = b.lo + elems * (uint64_t)esz;
  b.origin = (intptr_t)(b.lo - index0 * (uint64_t)esz);
  b.esz = esz;
  b.rank = rank;
  b.out = out;
  b.what = what;
  b.idx = idx;
  return b;
}

// Outputs must not overlap each other; an output may overlap an input only if
// both belong to the same rank and address the same elements identically.
rc_status check_aliasing(const std::vector<Buf> &bs) {
  for (size_t i = 0; i < bs.size(); ++i) {
    for (size_t j = i + 1; j < bs.size(); ++j) {
      const Buf &a = bs[i], &b = bs[j];
      if (!a.out && !b.out) continue;
      if (a.lo >= b.hi || b.lo >= a.hi || a.lo == a.hi || b.lo == b.hi) continue;
      if (a.out && b.out)
        return fail(RC_ERR_INVALID_ARG, "output buffers %s[%d] and %s[%d] overlap", a.what, a.idx,
                    b.what, b.idx);
      if (a.rank != b.rank || a.esz != b.esz || a.origin != b.origin)
        return fail(RC_ERR_INVALID_ARG,
                    "%s[%d] and %s[%d] overlap in a way other than same-rank in-place", a.what,
                    a.idx, b.what, b.idx);
    }
  }
  return RC_OK;
}

rc_status check_ranges(const std::vector<Buf> &bs, bool peer_ok = false) {
  for (const Buf &b : bs) {
    if (b.esz > 1 && b.lo % (uintptr_t)b.esz != 0)
      return fail(RC_ERR_INVALID_ARG, "%s[%d]=%p is not aligned to its %d-byte elements", b.what, b.idx,
                  (void *)b.lo, b.esz);
    rc_status st = check_device_range((const void *)b.lo, b.hi - b.lo, b.what, b.idx, peer_ok);
    if (st != RC_OK) return st;
  }
  return RC_OK;
}

int dt_size(rc_dtype d) { return d == RC_BF16 ? 2 : 4; }
bool dt_ok(int d) { return d == RC_FP32 || d == RC_BF16 || d == RC_INT32; }
bool op_ok(int o) { return o == RC_SUM || o == RC_MAX || o == RC_MIN; }

constexpr uint64_t kMaxElems = (1ull << 40);  // 1 Ti elements per rank

rc_status check_p_n(int p, size_t n) {
  if (p < 1 || p > kMaxP) return fail(RC_ERR_INVALID_ARG, "p=%d outside [1, %d]", p, kMaxP);
  if (n > kMaxElems) return fail(RC_ERR_INVALID_ARG, "n=%zu too large", n);
  return RC_OK;
}

rc_status check_reduce_types(rc_dtype in, rc_dtype out, rc_op op, float scale) {
  if (!dt_ok(in) || !dt_ok(out)) return fail(RC_ERR_INVALID_ARG, "unknown dtype");
  if (!op_ok(op)) return fail(RC_ERR_INVALID_ARG, "unknown op");
  if ((in == RC_INT32) != (out == RC_INT32))
    return fail(RC_ERR_INVALID_ARG, "int32 reduces only to int32");
  if ((in == RC_INT32 || op != RC_SUM) && scale != 1.0f)
    return fail(RC_ERR_INVALID_ARG, "scale must be 1 unless op is SUM on a floating type");
  return RC_OK;
}

rc_status launched(cudaError_t e, const char *what) {
  if (e != cudaSuccess) return cuda_fail(e, what);
  return RC_OK;
}

// ---------------------------------------------------------------- workspace
// One workspace per device.  A call on a stream other than the last user's
// first waits for the last user's work (event), so concurrent streams never
// share it; growth frees the old block in stream order.  A block that a stream
// capture has taken is never freed before rc_finalize: the captured graph
// keeps its address and may be replayed after the workspace has grown, so on
// growth such a block is retired (kept allocated) instead of freed.
struct Workspace {
  void *ptr = nullptr;
  size_t cap = 0;
  cudaStream_t last = nullptr;
  cudaEvent_t done = nullptr;
  bool used = false;
  bool captured = false;        // a stream capture holds ptr
  std::vector<void *> retired;  // captured blocks replaced by a larger one
  size_t retired_bytes = 0;
};
std::mutex g_ws_mu;
Workspace g_ws[kMaxDevices];

rc_status ws_acquire(size_t bytes, cudaStream_t s, void **out, int *dev_out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(RC_ERR_UNSUPPORTED, "device index %d", dev);
  Workspace &w = g_ws[dev];
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  cudaStreamIsCapturing(s, &cap);
  if (cap != cudaStreamCaptureStatusNone) {
    if (w.cap < bytes)
      return fail(RC_ERR_INVALID_ARG,
                  "workspace of %zu bytes needed during stream capture: call "
                  "rc_reserve_workspace first",
                  bytes);
    *out = w.ptr;
    *dev_out = -1;  // no event bookkeeping inside a capture
    w.captured = true;
    return RC_OK;
  }
  if (!w.done) {
    if ((e = cudaEventCreateWithFlags(&w.done, cudaEventDisableTiming)) != cudaSuccess)
      return cuda_fail(e, "cudaEventCreate");
  }
  if (w.used && w.last != s) {
    if ((e = cudaStreamWaitEvent(s, w.done, 0)) != cudaSuccess)
      return cuda_fail(e, "cudaStreamWaitEvent");
  }
  if (w.cap < bytes) {
    if (w.ptr) {
      if (w.captured) {  // a graph may still use it: keep it until rc_finalize
        w.retired.push_back(w.ptr);
        w.retired_bytes += w.cap;
      } else if ((e = cudaFreeAsync(w.ptr, s)) != cudaSuccess) {
        return cuda_fail(e, "cudaFreeAsync");
      }
      w.ptr = nullptr;
      w.cap = 0;
      w.captured = false;
    }
    const size_t want = (bytes + 255) & ~(size_t)255;
    if ((e = cudaMallocAsync(&w.ptr, want, s)) != cudaSuccess) {
      w.ptr = nullptr;
      return cuda_fail(e, "cudaMallocAsync(workspace)");
    }
    w.cap = want;
  }
  *out = w.ptr;
  *dev_out = dev;
  return RC_OK;
}

void ws_release(int dev, cudaStream_t s) {
  if (dev < 0) return;
  Workspace &w = g_ws[dev];
  cudaEventRecord(w.done, s);
  w.last = s;
  w.used = true;
}

}  // namespace
}  // namespace rc

using namespace rc;

extern "C" {

rc_status rc_all_reduce(const void *const *send, void *const *recv, int p, size_t n, rc_dtype dt,
                        rc_op op, float scale, rc_stream_t stream) {
  rc_status st;
  if ((st = check_p_n(p, n)) != RC_OK) return st;
  if ((st = check_reduce_types(dt, dt, op, scale)) != RC_OK) return st;
  if (n == 0) return RC_OK;
  if (!send || !recv) return fail(RC_ERR_INVALID_ARG, "pointer array is NULL");
  const int s = dt_size(dt);
  std::vector<Buf> bs;
  for (int r = 0; r < p; ++r) bs.push_back(make_buf(send[r], n, s, 0, r, false, "send", r));
  for (int r = 0; r < p; ++r) bs.push_back(make_buf(recv[r], n, s, 0, r, true, "recv", r));
  if ((st = check_ranges(bs)) != RC_OK) return st;
  if ((st = check_aliasing(bs)) != RC_OK) return st;
  ReduceJob j{};
  j.p = p;
  j.n = n;
  for (int r = 0; r < p; ++r) {
    j.src[r] = send[r];
    j.dst[r] = recv[r];
  }
  j.in_dt = j.out_dt = dt;
  j.op = op;
  j.scale = scale;
  j.mode = kModeAll;
  j.ndst = p;
  return launched(launch_reduce(j, (cudaStream_t)stream), "all_reduce launch");
}

rc_status rc_reduce_scatter(const void *const *send, void *const *recv, int p, size_t n,
                            rc_dtype in_dt, rc_dtype out_dt, rc_op op, float scale,
                            rc_stream_t stream) {
  rc_status st;
  if ((st = check_p_n(p, n)) != RC_OK) return st;
  if ((st = check_reduce_types(in_dt, out_dt, op, scale)) != RC_OK) return st;
  if (n % (size_t)p != 0) return fail(RC_ERR_INVALID_ARG, "n=%zu is not a multiple of p=%d", n, p);
  if (n == 0) return RC_OK;
  if (!send || !recv) return fail(RC_ERR_INVALID_ARG, "pointer array is NULL");
  const uint64_t m = n / p;
  std::vector<Buf> bs;
  for (int r = 0; r < p; ++r) bs.push_back(make_buf(send[r], n, dt_size(in_dt), 0, r, false, "send", r));
  for (int r = 0; r < p; ++r)
    bs.push_back(make_buf(recv[r], m, dt_size(out_dt), (uint64_t)r * m, r, true, "recv", r));
  if ((st = check_ranges(bs)) != RC_OK) return st;
  if ((st = check_aliasing(bs)) != RC_OK) return st;
  ReduceJob j{};
  j.p = p;
  j.n = n;
  for (int r = 0; r < p; ++r) {
    j.src[r] = send[r];
    j.dst[r] = recv[r];
  }
  j.in_dt = in_dt;
  j.out_dt = out_dt;
  j.op = op;
  j.scale = scale;
  j.mode = kModeScatter;
  return launched(launch_reduce(j, (cudaStream_t)stream), "reduce_scatter launch");
}

rc_status rc_all_gather(const void *const *send, void *const *recv, int p, size_t n, rc_dtype dt,
                        rc_stream_t stream) {
  rc_status st;
  if ((st = check_p_n(p, n)) != RC_OK) return st;
  if (!dt_ok(dt)) return fail(RC_ERR_INVALID_ARG, "unknown dtype");
  if (n % (size_t)p != 0) return fail(RC_ERR_INVALID_ARG, "n=%zu is not a multiple of p=%d", n, p);
  if (n == 0) return RC_OK;
  if (!send || !recv) return fail(RC_ERR_INVALID_ARG, "pointer array is NULL");
  const int s = dt_size(dt);
  const uint64_t m = n / p;
  std::vector<Buf> bs;
  for (int r = 0; r < p; ++r) bs.push_back(make_buf(send[r], m, s, (uint64_t)r * m, r, false, "send", r));
  for (int r = 0; r < p; ++r) bs.push_back(make_buf(recv[r], n, s, 0, r, true, "recv", r));
  if ((st = check_ranges(bs)) != RC_OK) return st;
  if ((st = check_aliasing(bs)) != RC_OK) return st;
  FanoutJob f{};
  f.nsrc = p;
  f.p = p;
  f.src_bytes = m * s;
  f.elem_bytes = s;
  for (int r = 0; r < p; ++r) {
    f.src[r] = send[r];
    f.dst[r] = recv[r];
  }
  for (int q = 0; q < p; ++q)
    for (int r = 0; r < p; ++r)
      if ((const char *)recv[q] + (uint64_t)r * m * s == (const char *)send[r]) f.skip[q] |= 1u << r;
  return launched(launch_fanout(f, (cudaStream_t)stream), "all_gather launch");
}

rc_status rc_reduce(const void *const *send, void *recv_root, int p, int root, size_t n, rc_dtype dt,
                    rc_op op, float scale, rc_stream_t stream) {
  rc_status st;
  if ((st = check_p_n(p, n)) != RC_OK) return st;
  if ((st = check_reduce_types(dt, dt, op, scale)) != RC_OK) return st;
  if (root < 0 || root >= p) return fail(RC_ERR_INVALID_ARG, "root=%d outside [0, %d)", root, p);
  if (n == 0) return RC_OK;
  if (!send) return fail(RC_ERR_INVALID_ARG, "pointer array is NULL");
  const int s = dt_size(dt);
  std::vector<Buf> bs;
  for (int r = 0; r < p; ++r) bs.push_back(make_buf(send[r], n, s, 0, r, false, "send", r));
  bs.push_back(make_buf(recv_root, n, s, 0, root, true, "recv_root", 0));
  if ((st = check_ranges(bs)) != RC_OK) return st;
  if ((st = check_aliasing(bs)) != RC_OK) return st;
  ReduceJob j{};
  j.p = p;
  j.n = n;
  for (int r = 0; r < p; ++r) j.src[r] = send[r];
  j.dst[0] = recv_root;
  j.in_dt = j.out_dt = dt;
  j.op = op;
  j.scale = scale;
  j.mode = kModeOne;
  return launched(launch_reduce(j, (cudaStream_t)stream), "reduce launch");
}

rc_status rc_broadcast(const void *send_root, void *const *recv, int p, int root, size_t n,
                       rc_dtype dt, rc_stream_t stream) {
  rc_status st;
  if ((st = check_p_n(p, n)) != RC_OK) return st;
  if (!dt_ok(dt)) return fail(RC_ERR_INVALID_ARG, "unknown dtype");
  if (root < 0 || root >= p) return fail(RC_ERR_INVALID_ARG, "root=%d outside [0, %d)", root, p);
  if (n == 0) return RC_OK;
  if (!recv) return fail(RC_ERR_INVALID_ARG, "pointer array is NULL");
  const int s = dt_size(dt);
  std::vector<Buf> bs;
  bs.push_back(make_buf(send_root, n, s, 0, root, false, "send_root", 0));
  for (int r = 0; r < p; ++r) bs.push_back(make_buf(recv[r], n, s, 0, r, true, "recv", r));
  if ((st = check_ranges(bs)) != RC_OK) return st;
  if ((st = check_aliasing(bs)) != RC_OK) return st;
  FanoutJob f{};
  f.nsrc = 1;
  f.p = p;
  f.src_bytes = (uint64_t)n * s;
  f.elem_bytes = s;
  f.src[0] = send_root;
  for (int q = 0; q < p; ++q) {
    f.dst[q] = recv[q];
    if (recv[q] == send_root) f.skip[q] = 1u;
  }
  return launched(launch_fanout(f, (cudaStream_t)stream), "broadcast launch");
}

rc_status rc_ring_all_reduce(const void *const *send, void *const *recv, int p, size_t n, rc_dtype dt,
                             rc_op op, float scale, rc_ring_variant variant, rc_stream_t stream) {
  if (variant == RC_RING_ONESHOT) return rc_all_reduce(send, recv, p, n, dt, op, scale, stream);
  if (variant != RC_RING_LITERAL) return fail(RC_ERR_INVALID_ARG, "unknown ring variant");
  rc_status st;
  if ((st = check_p_n(p, n)) != RC_OK) return st;
  if ((st = check_reduce_types(dt, dt, op, scale)) != RC_OK) return st;
  if (n == 0) return RC_OK;
  if (!send || !recv) return fail(RC_ERR_INVALID_ARG, "pointer array is NULL");
  if (p == 1) return rc_all_reduce(send, recv, p, n, dt, op, scale, stream);  // no steps
  const int s = dt_size(dt);
  std::vector<Buf> bs;
  for (int r = 0; r < p; ++r) bs.push_back(make_buf(send[r], n, s, 0, r, false, "send", r));
  for (int r = 0; r < p; ++r) bs.push_back(make_buf(recv[r], n, s, 0, r, true, "recv", r));
  if ((st = check_ranges(bs)) != RC_OK) return st;
  if ((st = check_aliasing(bs)) != RC_OK) return st;
  RingJob j{};
  j.p = p;
  j.n = n;
  j.dt = dt;
  j.op = op;
  j.scale = scale;
  for (int r = 0; r < p; ++r) {
    j.x[r] = send[r];
    j.y[r] = recv[r];
  }
  if (!ring_needs_workspace(j)) return launched(launch_ring_literal(j, (cudaStream_t)stream), "ring launch");
  int dev = -1;
  const uint64_t C = (n + p - 1) / p;
  std::lock_guard<std::mutex> lock(g_ws_mu);
  if ((st = ws_acquire(2ull * p * C * 4, (cudaStream_t)stream, &j.ws, &dev)) != RC_OK) return st;
  st = launched(launch_ring_literal(j, (cudaStream_t)stream), "ring launch");
  ws_release(dev, (cudaStream_t)stream);
  return st;
}

rc_status rc_ring_all_reduce_noalloc(const void *const *send, void *const *recv, int p, size_t n,
                                     rc_dtype dt, rc_op op, float scale, rc_stream_t stream) {
  rc_status st;
  if ((st = check_p_n(p, n)) != RC_OK) return st;
  if ((st = check_reduce_types(dt, dt, op, scale)) != RC_OK) return st;
  if (n == 0) return RC_OK;
  if (!send || !recv) return fail(RC_ERR_INVALID_ARG, "pointer array is NULL");
  if (p == 1) return rc_all_reduce(send, recv, p, n, dt, op, scale, stream);  // no steps, no scratch
  const uint64_t C = (n + p - 1) / p;
  const uint64_t need = dt == RC_BF16 ? 2ull * p * C : 0;  // fp32 partials, bf16 only
  if (need > noalloc_scratch_floats())
    return fail(RC_ERR_INVALID_ARG,
                "rc_ring_all_reduce_noalloc: bf16 with p=%d, n=%zu needs %llu floats of scratch; the "
                "fixed scratch holds %zu (2*p*ceil(n/p) must not exceed it)",
                p, n, (unsigned long long)need, noalloc_scratch_floats());
  const int s = dt_size(dt);
  std::vector<Buf> bs;
  for (int r = 0; r < p; ++r) bs.push_back(make_buf(send[r], n, s, 0, r, false, "send", r));
  for (int r = 0; r < p; ++r) bs.push_back(make_buf(recv[r], n, s, 0, r, true, "recv", r));
  if ((st = check_ranges(bs)) != RC_OK) return st;
  if ((st = check_aliasing(bs)) != RC_OK) return st;
  RingJob j{};
  j.p = p;
  j.n = n;
  j.dt = dt;
  j.op = op;
  j.scale = scale;
  j.partials_in_ws = true;  // the chain kernel, bf16 partials in the fixed scratch
  for (int r = 0; r < p; ++r) {
    j.x[r] = send[r];
    j.y[r] = recv[r];
  }
  if (dt == RC_BF16) {
    cudaError_t e = noalloc_scratch_ptr(&j.ws);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(fixed scratch)");
  }
  return launched(launch_ring_literal(j, (cudaStream_t)stream), "ring launch");
}

rc_status rc_hier_all_reduce(const void *const *send, void *const *recv, int p, int group_size,
                             size_t n, rc_dtype dt, rc_op op, float scale, rc_hier_variant variant,
                             rc_stream_t stream) {
  rc_status st;
  if ((st = check_p_n(p, n)) != RC_OK) return st;
  if ((st = check_reduce_types(dt, dt, op, scale)) != RC_OK) return st;
  if (group_size < 1 || p % group_size != 0)
    return fail(RC_ERR_INVALID_ARG, "group_size=%d does not divide p=%d", group_size, p);
  if (variant != RC_HIER_FUSED && variant != RC_HIER_STAGED)
    return fail(RC_ERR_INVALID_ARG, "unknown hierarchical variant");
  if (n == 0) return RC_OK;
  if (!send || !recv) return fail(RC_ERR_INVALID_ARG, "pointer array is NULL");
  const int s = dt_size(dt);
  std::vector<Buf> bs;
  for (int r = 0; r < p; ++r) bs.push_back(make_buf(send[r], n, s, 0, r, false, "send", r));
  for (int r = 0; r < p; ++r) bs.push_back(make_buf(recv[r], n, s, 0, r, true, "recv", r));
  if ((st = check_ranges(bs)) != RC_OK) return st;
  if ((st = check_aliasing(bs)) != RC_OK) return st;
  HierJob j{};
  j.p = p;
  j.G = group_size;
  j.n = n;
  j.dt = dt;
  j.op = op;
  j.scale = scale;
  for (int r = 0; r < p; ++r) {
    j.x[r] = send[r];
    j.y[r] = recv[r];
  }
  if (variant == RC_HIER_FUSED) return launched(launch_hier_fused(j, (cudaStream_t)stream), "hier launch");
  int dev = -1;
  std::lock_guard<std::mutex> lock(g_ws_mu);
  const uint64_t ng = (uint64_t)(p / group_size);
  if ((st = ws_acquire((ng + 1) * n * 4, (cudaStream_t)stream, &j.ws, &dev)) != RC_OK) return st;
  st = launched(launch_hier_staged(j, (cudaStream_t)stream), "hier staged launch");
  ws_release(dev, (cudaStream_t)stream);
  return st;
}

namespace {
rc_status check_hparams(const rc_adamw_hparams *hp, AdamwHyper *out) {
  if (!hp) return fail(RC_ERR_INVALID_ARG, "hparams is NULL");
  if (hp->step < 1) return fail(RC_ERR_INVALID_ARG, "step=%lld must be >= 1", (long long)hp->step);
  out->lr = hp->lr;
  out->beta1 = hp->beta1;
  out->beta2 = hp->beta2;
  out->eps = hp->eps;
  out->weight_decay = hp->weight_decay;
  out->step = hp->step;
  return RC_OK;
}
bool float_dt_ok(int d) { return d == RC_FP32 || d == RC_BF16; }
}  // namespace

rc_status rc_adamw_step(float *param, float *exp_avg, float *exp_avg_sq, const void *grad,
                        rc_dtype grad_dt, size_t n, const rc_adamw_hparams *hp, rc_stream_t stream) {
  rc_status st;
  AdamwHyper h{};
  if ((st = check_hparams(hp, &h)) != RC_OK) return st;
  if (!float_dt_ok(grad_dt)) return fail(RC_ERR_INVALID_ARG, "grad dtype must be fp32 or bf16");
  if (n > kMaxElems) return fail(RC_ERR_INVALID_ARG, "n=%zu too large", n);
  if (n == 0) return RC_OK;
  std::vector<Buf> bs;
  bs.push_back(make_buf(grad, n, dt_size(grad_dt), 0, 0, false, "grad", 0));
  bs.push_back(make_buf(param, n, 4, 0, 1, true, "param", 0));
  bs.push_back(make_buf(exp_avg, n, 4, 0, 2, true, "exp_avg", 0));
  bs.push_back(make_buf(exp_avg_sq, n, 4, 0, 3, true, "exp_avg_sq", 0));
  if ((st = check_ranges(bs)) != RC_OK) return st;
  if ((st = check_aliasing(bs)) != RC_OK) return st;
  return launched(launch_adamw(param, exp_avg, exp_avg_sq, grad, grad_dt, n, h, (cudaStream_t)stream),
                  "adamw launch");
}

rc_status rc_zero1_step(const void *const *grads, void *const *params, float *const *master,
                        float *const *exp_avg, float *const *exp_avg_sq, int p, size_t n,
                        rc_dtype grad_dt, rc_dtype param_dt, float scale,
                        const rc_adamw_hparams *hp, rc_stream_t stream) {
  rc_status st;
  AdamwHyper h{};
  if ((st = check_p_n(p, n)) != RC_OK) return st;
  if ((st = check_hparams(hp, &h)) != RC_OK) return st;
  if (!float_dt_ok(grad_dt) || !float_dt_ok(param_dt))
    return fail(RC_ERR_INVALID_ARG, "grad and param dtypes must be fp32 or bf16");
  if (n % (size_t)p != 0) return fail(RC_ERR_INVALID_ARG, "n=%zu is not a multiple of p=%d", n, p);
  if (n == 0) return RC_OK;
  if (!grads || !params || !master || !exp_avg || !exp_avg_sq)
    return fail(RC_ERR_INVALID_ARG, "pointer array is NULL");
  const uint64_t m = n / p;
  std::vector<Buf> bs;
  // ranks 0..p-1 for the gradients and parameters; the three state arrays of
  // rank r get their own "rank" ids so that no in-place overlap with a
  // gradient or parameter buffer is accepted
  for (int r = 0; r < p; ++r) bs.push_back(make_buf(grads[r], n, dt_size(grad_dt), 0, r, false, "grads", r));
  for (int r = 0; r < p; ++r) bs.push_back(make_buf(params[r], n, dt_size(param_dt), 0, r, true, "params", r));
  for (int r = 0; r < p; ++r) {
    bs.push_back(make_buf(master[r], m, 4, 0, kMaxP + 3 * r, true, "master", r));
    bs.push_back(make_buf(exp_avg[r], m, 4, 0, kMaxP + 3 * r + 1, true, "exp_avg", r));
    bs.push_back(make_buf(exp_avg_sq[r], m, 4, 0, kMaxP + 3 * r + 2, true, "exp_avg_sq", r));
  }
  if ((st = check_ranges(bs)) != RC_OK) return st;
  if ((st = check_aliasing(bs)) != RC_OK) return st;
  Zero1Job j{};
  j.p = p;
  j.n = n;
  for (int r = 0; r < p; ++r) {
    j.grad[r] = grads[r];
    j.param[r] = params[r];
    j.master[r] = master[r];
    j.exp_avg[r] = exp_avg[r];
    j.exp_avg_sq[r] = exp_avg_sq[r];
  }
  j.grad_dt = grad_dt;
  j.param_dt = param_dt;
  j.scale = scale;
  j.hp = h;
  return launched(launch_zero1(j, (cudaStream_t)stream), "zero1 launch");
}

rc_status rc_all_to_all_v(const void *const *send, void *const *recv, int p, const size_t *counts,
                          rc_dtype dt, rc_stream_t stream) {
  rc_status st;
  if ((st = check_p_n(p, 0)) != RC_OK) return st;
  if (!dt_ok(dt)) return fail(RC_ERR_INVALID_ARG, "unknown dtype");
  if (!counts) return fail(RC_ERR_INVALID_ARG, "counts is NULL");
  uint64_t total = 0;
  std::vector<uint64_t> sent(p, 0), got(p, 0);
  for (int r = 0; r < p; ++r)
    for (int q = 0; q < p; ++q) {
      const uint64_t c = counts[(size_t)r * p + q];
      if (c > kMaxElems) return fail(RC_ERR_INVALID_ARG, "counts[%d][%d]=%llu too large", r, q,
                                     (unsigned long long)c);
      sent[r] += c;
      got[q] += c;
      total += c;
    }
  for (int r = 0; r < p; ++r)
    if (sent[r] > kMaxElems || got[r] > kMaxElems)
      return fail(RC_ERR_INVALID_ARG, "rank %d sends or receives too many elements", r);
  if (total == 0) return RC_OK;
  if (!send || !recv) return fail(RC_ERR_INVALID_ARG, "pointer array is NULL");
  const int s = dt_size(dt);
  std::vector<Buf> bs;
  // sends and receives get distinct "ranks": no overlap between them is
  // accepted (a rank's incoming blocks would overwrite outgoing ones)
  for (int r = 0; r < p; ++r)
    if (sent[r]) bs.push_back(make_buf(send[r], sent[r], s, 0, r, false, "send", r));
  for (int q = 0; q < p; ++q)
    if (got[q]) bs.push_back(make_buf(recv[q], got[q], s, 0, kMaxP + q, true, "recv", q));
  if ((st = check_ranges(bs)) != RC_OK) return st;
  if ((st = check_aliasing(bs)) != RC_OK) return st;
  A2aJob j{};
  j.p = p;
  j.esz = s;
  for (int r = 0; r < p; ++r) {
    j.send[r] = send[r];
    j.recv[r] = recv[r];
  }
  for (int i = 0; i < p * p; ++i) j.counts[i] = counts[i];
  return launched(launch_all_to_all(j, (cudaStream_t)stream), "all_to_all launch");
}

rc_status rc_all_to_all(const void *const *send, void *const *recv, int p, size_t n, rc_dtype dt,
                        rc_stream_t stream) {
  rc_status st;
  if ((st = check_p_n(p, n)) != RC_OK) return st;
  if (n % (size_t)p != 0) return fail(RC_ERR_INVALID_ARG, "n=%zu is not a multiple of p=%d", n, p);
  std::vector<size_t> counts((size_t)p * p, n / p);
  return rc_all_to_all_v(send, recv, p, counts.data(), dt, stream);
}

// ---------------------------------------------------------------- rank view
rc_status rc_rank_all_reduce(const void *const *send, void *const *recv, int p, int rank, size_t n,
                             rc_dtype dt, rc_op op, float scale, rc_stream_t stream) {
  rc_status st;
  if ((st = check_p_n(p, n)) != RC_OK) return st;
  if ((st = check_reduce_types(dt, dt, op, scale)) != RC_OK) return st;
  if (rank < 0 || rank >= p) return fail(RC_ERR_INVALID_ARG, "rank=%d outside [0, %d)", rank, p);
  if (n == 0) return RC_OK;
  if (!send || !recv) return fail(RC_ERR_INVALID_ARG, "pointer array is NULL");
  const int s = dt_size(dt);
  std::vector<Buf> bs;
  for (int r = 0; r < p; ++r) bs.push_back(make_buf(send[r], n, s, 0, r, false, "send", r));
  for (int r = 0; r < p; ++r) bs.push_back(make_buf(recv[r], n, s, 0, r, true, "recv", r));
  if ((st = check_ranges(bs, true)) != RC_OK) return st;
  if ((st = check_aliasing(bs)) != RC_OK) return st;
  ReduceJob j{};
  j.p = p;
  j.n = n;
  for (int r = 0; r < p; ++r) {
    j.src[r] = send[r];
    j.dst[r] = recv[r];
  }
  j.in_dt = j.out_dt = dt;
  j.op = op;
  j.scale = scale;
  j.mode = kModeAll;
  j.ndst = p;
  j.c0 = rank;
  j.c1 = rank + 1;
  return launched(launch_reduce(j, (cudaStream_t)stream), "rank all_reduce launch");
}

rc_status rc_rank_reduce_scatter(const void *const *send, void *recv_own, int p, int rank, size_t n,
                                 rc_dtype in_dt, rc_dtype out_dt, rc_op op, float scale,
                                 rc_stream_t stream) {
  rc_status st;
  if ((st = check_p_n(p, n)) != RC_OK) return st;
  if ((st = check_reduce_types(in_dt, out_dt, op, scale)) != RC_OK) return st;
  if (rank < 0 || rank >= p) return fail(RC_ERR_INVALID_ARG, "rank=%d outside [0, %d)", rank, p);
  if (n % (size_t)p != 0) return fail(RC_ERR_INVALID_ARG, "n=%zu is not a multiple of p=%d", n, p);
  if (n == 0) return RC_OK;
  if (!send) return fail(RC_ERR_INVALID_ARG, "pointer array is NULL");
  const uint64_t m = n / p;
  std::vector<Buf> bs;
  for (int r = 0; r < p; ++r) bs.push_back(make_buf(send[r], n, dt_size(in_dt), 0, r, false, "send", r));
  bs.push_back(make_buf(recv_own, m, dt_size(out_dt), (uint64_t)rank * m, rank, true, "recv_own", 0));
  if ((st = check_ranges(bs, true)) != RC_OK) return st;
  if ((st = check_aliasing(bs)) != RC_OK) return st;
  ReduceJob j{};
  j.p = p;
  j.n = n;
  // only chunk `rank` is computed, so only dst[rank] is ever written
  for (int r = 0; r < p; ++r) {
    j.src[r] = send[r];
    j.dst[r] = recv_own;
  }
  j.in_dt = in_dt;
  j.out_dt = out_dt;
  j.op = op;
  j.scale = scale;
  j.mode = kModeScatter;
  j.c0 = rank;
  j.c1 = rank + 1;
  return launched(launch_reduce(j, (cudaStream_t)stream), "rank reduce_scatter launch");
}

rc_status rc_rank_all_gather(const void *const *send, void *recv_own, int p, int rank, size_t n,
                             rc_dtype dt, rc_stream_t stream) {
  rc_status st;
  if ((st = check_p_n(p, n)) != RC_OK) return st;
  if (!dt_ok(dt)) return fail(RC_ERR_INVALID_ARG, "unknown dtype");
  if (rank < 0 || rank >= p) return fail(RC_ERR_INVALID_ARG, "rank=%d outside [0, %d)", rank, p);
  if (n % (size_t)p != 0) return fail(RC_ERR_INVALID_ARG, "n=%zu is not a multiple of p=%d", n, p);
  if (n == 0) return RC_OK;
  if (!send) return fail(RC_ERR_INVALID_ARG, "pointer array is NULL");
  const int s = dt_size(dt);
  const uint64_t m = n / p;
  std::vector<Buf> bs;
  for (int r = 0; r < p; ++r) bs.push_back(make_buf(send[r], m, s, (uint64_t)r * m, r, false, "send", r));
  bs.push_back(make_buf(recv_own, n, s, 0, rank, true, "recv_own", 0));
  if ((st = check_ranges(bs, true)) != RC_OK) return st;
  if ((st = check_aliasing(bs)) != RC_OK) return st;
  FanoutJob f{};
  f.nsrc = p;
  f.p = 1;  // one destination: this rank's output
  f.src_bytes = m * s;
  f.elem_bytes = s;
  for (int r = 0; r < p; ++r) f.src[r] = send[r];
  f.dst[0] = recv_own;
  if ((const char *)recv_own + (uint64_t)rank * m * s == (const char *)send[rank]) f.skip[0] = 1u << rank;
  return launched(launch_fanout(f, (cudaStream_t)stream), "rank all_gather launch");
}

rc_status rc_rank_ring_step(const void *const *send, void *const *recv, void *const *ws, int p, int rank,
                            int step, size_t n, rc_dtype dt, rc_op op, float scale, rc_stream_t stream) {
  rc_status st;
  if ((st = check_p_n(p, n)) != RC_OK) return st;
  if ((st = check_reduce_types(dt, dt, op, scale)) != RC_OK) return st;
  if (p < 2) return fail(RC_ERR_INVALID_ARG, "the ring needs p >= 2 (p=%d)", p);
  if (rank < 0 || rank >= p) return fail(RC_ERR_INVALID_ARG, "rank=%d outside [0, %d)", rank, p);
  if (step < 0 || step >= 2 * (p - 1))
    return fail(RC_ERR_INVALID_ARG, "step=%d outside [0, %d)", step, 2 * (p - 1));
  if (n == 0) return RC_OK;
  if (!send || !recv) return fail(RC_ERR_INVALID_ARG, "pointer array is NULL");
  if (dt == RC_BF16 && !ws) return fail(RC_ERR_INVALID_ARG, "bf16 needs the ranks' workspaces (ws is NULL)");
  const int s = dt_size(dt);
  const uint64_t C = (n + p - 1) / p;
  std::vector<Buf> bs;
  for (int r = 0; r < p; ++r) bs.push_back(make_buf(send[r], n, s, 0, r, false, "send", r));
  for (int r = 0; r < p; ++r) bs.push_back(make_buf(recv[r], n, s, 0, r, true, "recv", r));
  if (dt == RC_BF16)
    for (int r = 0; r < p; ++r) bs.push_back(make_buf(ws[r], 2 * C, 4, 0, r, true, "ws", r));
  if ((st = check_ranges(bs, true)) != RC_OK) return st;
  if ((st = check_aliasing(bs)) != RC_OK) return st;
  RankStepJob j{};
  j.p = p;
  j.rank = rank;
  j.step = step;
  j.n = n;
  j.dt = dt;
  j.op = op;
  j.scale = scale;
  for (int r = 0; r < p; ++r) {
    j.x[r] = send[r];
    j.y[r] = recv[r];
    j.ws[r] = dt == RC_BF16 ? ws[r] : nullptr;
  }
  return launched(launch_rank_ring_step(j, (cudaStream_t)stream), "rank ring step launch");
}

// ---------------------------------------------------------------- IPC
namespace {
struct IpcMap {
  unsigned char key[sizeof(cudaIpcMemHandle_t)];
  char *base;
  size_t size;
  int refs;
};
std::mutex g_ipc_mu;
std::vector<IpcMap> g_ipc;
static_assert(sizeof(cudaIpcMemHandle_t) == sizeof(((rc_ipc_handle *)nullptr)->ipc),
              "rc_ipc_handle.ipc must hold a cudaIpcMemHandle_t");
}  // namespace

rc_status rc_ipc_export(const void *ptr, size_t bytes, rc_ipc_handle *out) {
  if (!out) return fail(RC_ERR_INVALID_ARG, "rc_ipc_export: out is NULL");
  rc_status st = check_device_range(ptr, bytes, "ptr", 0);
  if (st != RC_OK) return st;
  MemGetAddressRangeFn fn = address_range_fn();
  if (!fn) return fail(RC_ERR_UNSUPPORTED, "rc_ipc_export: allocation ranges cannot be queried");
  CUdeviceptr base = 0;
  size_t size = 0;
  if (fn(&base, &size, (CUdeviceptr)(uintptr_t)ptr) != CUDA_SUCCESS)
    return fail(RC_ERR_INVALID_ARG, "rc_ipc_export: %p is not inside a device allocation", ptr);
  cudaIpcMemHandle_t h;
  cudaError_t e = cudaIpcGetMemHandle(&h, (void *)(uintptr_t)base);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return cuda_fail(e, "cudaIpcGetMemHandle");
  }
  int dev = -1;
  cudaGetDevice(&dev);
  memset(out, 0, sizeof *out);
  memcpy(out->ipc, &h, sizeof h);
  out->offset = (uint64_t)((uintptr_t)ptr - (uintptr_t)base);
  out->bytes = bytes;
  out->device = dev;
  out->pid = (int32_t)getpid();
  return RC_OK;
}

rc_status rc_ipc_import(const rc_ipc_handle *h, void **ptr) {
  if (!h || !ptr) return fail(RC_ERR_INVALID_ARG, "rc_ipc_import: NULL argument");
  *ptr = nullptr;
  if (h->pid == (int32_t)getpid())
    return fail(RC_ERR_INVALID_ARG, "rc_ipc_import: the handle was exported by this process; use the buffer itself");
  std::lock_guard<std::mutex> lock(g_ipc_mu);
  for (IpcMap &m : g_ipc) {
    if (memcmp(m.key, h->ipc, sizeof m.key) == 0) {
      if (h->offset > m.size || h->bytes > m.size - h->offset)
        return fail(RC_ERR_INVALID_ARG, "rc_ipc_import: offset %llu + %llu bytes past the mapped allocation (%zu)",
                    (unsigned long long)h->offset, (unsigned long long)h->bytes, m.size);
      ++m.refs;
      *ptr = m.base + h->offset;
      return RC_OK;
    }
  }
  cudaIpcMemHandle_t hh;
  memcpy(&hh, h->ipc, sizeof hh);
  void *base = nullptr;
  cudaError_t e = cudaIpcOpenMemHandle(&base, hh, cudaIpcMemLazyEnablePeerAccess);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return cuda_fail(e, "cudaIpcOpenMemHandle");
  }
  size_t size = (size_t)-1;
  MemGetAddressRangeFn fn = address_range_fn();
  CUdeviceptr b = 0;
  if (fn && fn(&b, &size, (CUdeviceptr)(uintptr_t)base) != CUDA_SUCCESS) size = (size_t)-1;
  if (h->offset > size || h->bytes > size - h->offset) {
    cudaIpcCloseMemHandle(base);
    return fail(RC_ERR_INVALID_ARG, "rc_ipc_import: offset %llu + %llu bytes past the mapped allocation (%zu)",
                (unsigned long long)h->offset, (unsigned long long)h->bytes, size);
  }
  IpcMap m;
  memcpy(m.key, h->ipc, sizeof m.key);
  m.base = static_cast<char *>(base);
  m.size = size;
  m.refs = 1;
  g_ipc.push_back(m);
  *ptr = m.base + h->offset;
  return RC_OK;
}

rc_status rc_ipc_release(void *ptr) {
  std::lock_guard<std::mutex> lock(g_ipc_mu);
  const char *q = static_cast<const char *>(ptr);
  // the mapping that contains ptr; an address one past the end belongs to a
  // mapping only if no mapping starts there (an empty buffer at the end)
  size_t hit = g_ipc.size();
  for (size_t i = 0; i < g_ipc.size() && hit == g_ipc.size(); ++i)
    if (q >= g_ipc[i].base && (size_t)(q - g_ipc[i].base) < g_ipc[i].size) hit = i;
  for (size_t i = 0; i < g_ipc.size() && hit == g_ipc.size(); ++i)
    if (q >= g_ipc[i].base && (size_t)(q - g_ipc[i].base) == g_ipc[i].size) hit = i;
  if (hit == g_ipc.size()) return fail(RC_ERR_INVALID_ARG, "rc_ipc_release: %p is not an imported buffer", ptr);
  IpcMap &m = g_ipc[hit];
  if (--m.refs > 0) return RC_OK;
  cudaError_t e = cudaIpcCloseMemHandle(m.base);
  g_ipc.erase(g_ipc.begin() + (long)hit);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return cuda_fail(e, "cudaIpcCloseMemHandle");
  }
  return RC_OK;
}

rc_status rc_copy(const void *src, void *dst, size_t bytes, rc_stream_t stream) {
  if (bytes == 0) return RC_OK;
  rc_status st;
  if ((st = check_device_range(src, bytes, "src", 0)) != RC_OK) return st;
  if ((st = check_device_range(dst, bytes, "dst", 0)) != RC_OK) return st;
  const uintptr_t a = (uintptr_t)src, b = (uintptr_t)dst;
  if (a < b + bytes && b < a + bytes) return fail(RC_ERR_INVALID_ARG, "src and dst overlap");
  return launched(launch_copy(src, dst, bytes, (cudaStream_t)stream), "copy launch");
}

rc_status rc_probe_bounded_wait(uint64_t limit_ns, rc_stream_t stream) {
  if (limit_ns == 0 || limit_ns > 1000000000ull)
    return fail(RC_ERR_INVALID_ARG, "limit_ns=%llu outside (0, 1e9]", (unsigned long long)limit_ns);
  return launched(launch_wait_probe(limit_ns, (cudaStream_t)stream), "wait probe launch");
}

rc_status rc_check_buffer(const void *ptr, size_t bytes) {
  return check_device_range(ptr, bytes, "buffer", 0);
}

rc_status rc_reserve_workspace(size_t bytes, rc_stream_t stream) {
  std::lock_guard<std::mutex> lock(g_ws_mu);
  void *p = nullptr;
  int dev = -1;
  rc_status st = ws_acquire(bytes, (cudaStream_t)stream, &p, &dev);
  if (st == RC_OK) ws_release(dev, (cudaStream_t)stream);
  return st;
}

rc_status rc_stream_status(rc_stream_t stream) {
  cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "stream");
  unsigned int timeouts = 0, fold_timeouts = 0;
  e = read_and_clear_wait_timeouts(&timeouts);
  if (e == cudaSuccess) e = read_and_clear_fold_timeouts(&fold_timeouts);
  if (e != cudaSuccess) return cuda_fail(e, "status word");
  timeouts += fold_timeouts;
  if (timeouts) return fail(RC_ERR_TIMEOUT, "%u bounded device wait(s) gave up", timeouts);
  return RC_OK;
}

const char *rc_status_string(rc_status s) {
  switch (s) {
    case RC_OK: return "ok";
    case RC_ERR_INVALID_ARG: return "invalid argument";
    case RC_ERR_UNSUPPORTED: return "unsupported";
    case RC_ERR_CUDA: return "CUDA error";
    case RC_ERR_TIMEOUT: return "device wait timed out";
  }
  return "unknown status";
}

const char *rc_last_error(void) { return t_last_error; }

uint64_t rc_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

rc_status rc_finalize(void) {
  std::lock_guard<std::mutex> lock(g_ws_mu);
  int cur = 0;
  cudaGetDevice(&cur);
  rc_status st = RC_OK;
  for (int d = 0; d < kMaxDevices; ++d) {
    Workspace &w = g_ws[d];
    if (!w.ptr && !w.done) continue;
    cudaSetDevice(d);
    cudaDeviceSynchronize();
    if (w.ptr && cudaFree(w.ptr) != cudaSuccess) st = fail(RC_ERR_CUDA, "cudaFree(workspace)");
    for (void *old : w.retired)
      if (cudaFree(old) != cudaSuccess) st = fail(RC_ERR_CUDA, "cudaFree(retired workspace)");
    if (w.done) cudaEventDestroy(w.done);
    w = Workspace{};
  }
  cudaSetDevice(cur);
  noalloc_scratch_forget();
  return st;
}

rc_status rc_workspace_bytes(size_t *live, size_t *retired) {
  if (!live || !retired) return fail(RC_ERR_INVALID_ARG, "output pointer is NULL");
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(RC_ERR_UNSUPPORTED, "device index %d", dev);
  std::lock_guard<std::mutex> lock(g_ws_mu);
  *live = g_ws[dev].cap;
  *retired = g_ws[dev].retired_bytes;
  return RC_OK;
}

int rc_version(void) { return 100; }

}  // extern "C"
