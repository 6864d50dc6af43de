// bucketer.cu -- DDP-style gradient bucketing on top of the in-place
// all-reduce: host-side runtime, no kernels of its own.
//
// Page: "分布式训练/推理", section "数据并行：切 batch，复制模型" (naive DDP
// all-reduces every parameter's gradient after the whole backward: many
// calls, each with its fixed cost, all of them exposed; flattening every
// gradient into one all-reduce saves calls but waits for the last gradient;
// registering a hook per parameter and all-reducing each gradient as soon as
// it is ready hides communication under the remaining backward, at the price
// of many small messages; which is faster has to be measured, and the test
// of an overlap is how much communication remains exposed after backward).
//
// Model: every simulated rank keeps its gradients in one flat buffer; tensor
// t occupies the element range [off_t, off_t + numel_t) of every rank's
// buffer, tensors laid out in the order their gradients become ready (the
// reverse of the forward order, as in DDP).  Buckets are runs of consecutive
// whole tensors: a bucket takes tensors in order and closes as soon as it
// holds at least bucket_bytes (so it exceeds the cap by less than its last
// tensor, and a tensor of at least the cap closes its bucket).  bucket_bytes = 0 gives
// one bucket per tensor (per-parameter all-reduce), SIZE_MAX one bucket for
// everything (the flattened all-reduce).  A bucket is one contiguous slice of
// every rank's buffer and is reduced by one in-place rc_all_reduce (with
// `scale`, e.g. 1/p for the average) on the bucketer's communication stream,
// as soon as all of its tensors are marked ready; the fold order is that of
// an all-reduce of the bucket's slice.
//
// Stream protocol: rc_bucketer_ready(t, producer) records an event on the
// producer stream (after the work that wrote tensor t's gradients on every
// rank) and makes the communication stream wait for it; when it completes a
// bucket, the bucket's all-reduce is enqueued on the communication stream.
// rc_bucketer_flush(consumer) makes the consumer stream wait for every
// bucket's all-reduce and starts the next step; it fails if a bucket was left
// incomplete (a tensor never marked ready), after enqueueing nothing more.
// One host thread at a time per bucketer.
#include <cuda_runtime.h>

#include <cstdint>
#include <vector>

#include "internal.h"
#include "rankcoll.h"

struct rc_bucketer {
  int p = 0;
  int dt = 0;
  float scale = 1.0f;
  cudaStream_t comm = nullptr;
  void *flat[rc::kMaxP] = {};
  std::vector<uint64_t> off, numel;  // per tensor (elements)
  std::vector<int> bucket_of;        // per tensor
  std::vector<int> t0, t1;           // per bucket: tensors [t0, t1)
  std::vector<int> pending;          // per bucket: tensors not yet ready this step
  std::vector<char> seen;            // per tensor: marked ready this step
  std::vector<cudaEvent_t> ready_ev; // per tensor
  cudaEvent_t done = nullptr;
  int device = -1;
  int launched = 0;                  // buckets enqueued this step
};

namespace rc {
int plan_buckets(int ntensors, const size_t *numel, size_t esz, size_t bucket_bytes, int *bucket_of) {
  int b = -1;
  uint64_t fill = 0;
  for (int t = 0; t < ntensors; ++t) {
    const uint64_t bytes = (uint64_t)numel[t] * esz;
    // start a new bucket when there is none, or the open one already reached the cap
    if (b < 0 || fill >= bucket_bytes || bucket_bytes == 0) {
      ++b;
      fill = 0;
    }
    bucket_of[t] = b;
    fill += bytes;
  }
  return b + 1;
}
}  // namespace rc

extern "C" {

rc_status rc_plan_buckets(int ntensors, const size_t *numel, size_t elem_bytes, size_t bucket_bytes,
                          int *bucket_of, int *nbuckets) {
  if (ntensors < 0 || (ntensors > 0 && (!numel || !bucket_of)) || !nbuckets || elem_bytes == 0)
    return rc::report_error(RC_ERR_INVALID_ARG, "rc_plan_buckets: bad arguments");
  *nbuckets = rc::plan_buckets(ntensors, numel, elem_bytes, bucket_bytes, bucket_of);
  return RC_OK;
}

rc_status rc_bucketer_create(rc_bucketer **out, void *const *flat, int p, int ntensors, const size_t *numel,
                             size_t bucket_bytes, rc_dtype dt, float scale, rc_stream_t comm) {
  if (!out) return rc::report_error(RC_ERR_INVALID_ARG, "rc_bucketer_create: out is NULL");
  *out = nullptr;
  if (p < 1 || p > rc::kMaxP || ntensors < 1 || !numel || !flat)
    return rc::report_error(RC_ERR_INVALID_ARG, "rc_bucketer_create: bad p, tensor list or buffer array");
  if (dt != RC_FP32 && dt != RC_BF16 && dt != RC_INT32)
    return rc::report_error(RC_ERR_INVALID_ARG, "rc_bucketer_create: unknown dtype");
  if (dt == RC_INT32 && scale != 1.0f)
    return rc::report_error(RC_ERR_INVALID_ARG, "rc_bucketer_create: int32 requires scale 1");
  const size_t esz = dt == RC_BF16 ? 2 : 4;
  uint64_t total = 0;
  for (int t = 0; t < ntensors; ++t) total += numel[t];
  for (int r = 0; r < p; ++r) {
    if (!flat[r]) return rc::report_error(RC_ERR_INVALID_ARG, "rc_bucketer_create: a gradient buffer is NULL");
    rc_status st = rc_check_buffer(flat[r], total * esz);
    if (st != RC_OK) return st;
  }
  rc_bucketer *b = new rc_bucketer();
  b->p = p;
  b->dt = dt;
  b->scale = scale;
  b->comm = (cudaStream_t)comm;
  for (int r = 0; r < p; ++r) b->flat[r] = flat[r];
  b->off.resize(ntensors);
  b->numel.resize(ntensors);
  b->bucket_of.resize(ntensors);
  uint64_t o = 0;
  for (int t = 0; t < ntensors; ++t) {
    b->off[t] = o;
    b->numel[t] = numel[t];
    o += numel[t];
  }
  const int nb = rc::plan_buckets(ntensors, numel, esz, bucket_bytes, b->bucket_of.data());
  b->t0.assign(nb, ntensors);
  b->t1.assign(nb, 0);
  for (int t = 0; t < ntensors; ++t) {
    const int k = b->bucket_of[t];
    if (t < b->t0[k]) b->t0[k] = t;
    if (t + 1 > b->t1[k]) b->t1[k] = t + 1;
  }
  b->pending.resize(nb);
  for (int k = 0; k < nb; ++k) b->pending[k] = b->t1[k] - b->t0[k];
  b->seen.assign(ntensors, 0);
  b->ready_ev.assign(ntensors, nullptr);
  cudaError_t e = cudaGetDevice(&b->device);
  for (int t = 0; t < ntensors && e == cudaSuccess; ++t)
    e = cudaEventCreateWithFlags(&b->ready_ev[t], cudaEventDisableTiming);
  if (e == cudaSuccess) e = cudaEventCreateWithFlags(&b->done, cudaEventDisableTiming);
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    rc_bucketer_destroy(b);
    return rc::report_error(RC_ERR_CUDA, "rc_bucketer_create: event creation failed");
  }
  *out = b;
  return RC_OK;
}

rc_status rc_bucketer_num_buckets(const rc_bucketer *b, int *nbuckets) {
  if (!b || !nbuckets) return rc::report_error(RC_ERR_INVALID_ARG, "rc_bucketer_num_buckets: NULL argument");
  *nbuckets = (int)b->t0.size();
  return RC_OK;
}

rc_status rc_bucketer_bucket(const rc_bucketer *b, int k, int *first_tensor, int *end_tensor,
                             size_t *first_elem, size_t *nelem) {
  if (!b || k < 0 || k >= (int)b->t0.size())
    return rc::report_error(RC_ERR_INVALID_ARG, "rc_bucketer_bucket: no such bucket");
  const int t0 = b->t0[k], t1 = b->t1[k];
  if (first_tensor) *first_tensor = t0;
  if (end_tensor) *end_tensor = t1;
  if (first_elem) *first_elem = b->off[t0];
  if (nelem) *nelem = b->off[t1 - 1] + b->numel[t1 - 1] - b->off[t0];
  return RC_OK;
}

rc_status rc_bucketer_ready(rc_bucketer *b, int tensor, rc_stream_t producer) {
  if (!b || tensor < 0 || tensor >= (int)b->off.size())
    return rc::report_error(RC_ERR_INVALID_ARG, "rc_bucketer_ready: no such tensor");
  if (b->seen[tensor])
    return rc::report_error(RC_ERR_INVALID_ARG, "rc_bucketer_ready: tensor marked ready twice in one step");
  cudaError_t e = cudaEventRecord(b->ready_ev[tensor], (cudaStream_t)producer);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(b->comm, b->ready_ev[tensor], 0);
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    return rc::report_error(RC_ERR_CUDA, "rc_bucketer_ready: event record / stream wait failed");
  }
  b->seen[tensor] = 1;
  const int k = b->bucket_of[tensor];
  if (--b->pending[k] > 0) return RC_OK;
  // bucket k is complete: reduce its slice of every rank's buffer, in place
  const size_t esz = b->dt == RC_BF16 ? 2 : 4;
  const uint64_t e0 = b->off[b->t0[k]];
  const uint64_t n = b->off[b->t1[k] - 1] + b->numel[b->t1[k] - 1] - e0;
  void *sl[rc::kMaxP];
  for (int r = 0; r < b->p; ++r) sl[r] = static_cast<char *>(b->flat[r]) + e0 * esz;
  ++b->launched;
  return rc_all_reduce(sl, sl, b->p, n, (rc_dtype)b->dt, RC_SUM, b->scale, b->comm);
}

rc_status rc_bucketer_flush(rc_bucketer *b, rc_stream_t consumer) {
  if (!b) return rc::report_error(RC_ERR_INVALID_ARG, "rc_bucketer_flush: NULL bucketer");
  bool complete = true;
  for (size_t k = 0; k < b->pending.size(); ++k) complete = complete && b->pending[k] == 0;
  cudaError_t e = cudaEventRecord(b->done, b->comm);
  if (e == cudaSuccess) e = cudaStreamWaitEvent((cudaStream_t)consumer, b->done, 0);
  // next step
  for (size_t k = 0; k < b->pending.size(); ++k) b->pending[k] = b->t1[k] - b->t0[k];
  for (size_t t = 0; t < b->seen.size(); ++t) b->seen[t] = 0;
  b->launched = 0;
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    return rc::report_error(RC_ERR_CUDA, "rc_bucketer_flush: event record / stream wait failed");
  }
  return complete ? RC_OK
                  : rc::report_error(RC_ERR_INVALID_ARG,
                                     "rc_bucketer_flush: a bucket was incomplete (a tensor never marked ready)");
}

rc_status rc_bucketer_destroy(rc_bucketer *b) {
  if (!b) return RC_OK;
  for (cudaEvent_t ev : b->ready_ev)
    if (ev) cudaEventDestroy(ev);
  if (b->done) cudaEventDestroy(b->done);
  delete b;
  return RC_OK;
}

}  // extern "C"
