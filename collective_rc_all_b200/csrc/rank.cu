// rank.cu -- one step of the literal ring as executed by one receiving rank,
// for rank-per-GPU execution (each process drives its own GPU and reaches the
// other ranks' buffers through peer mappings).
//
// Page: "LLM Parallelism 基础", section "Ring AllReduce": in each of the N-1
// reduce-scatter steps every card sends one chunk to the next card, which
// adds it into its own copy of that chunk; in each of the N-1 all-gather
// steps every card forwards a finished chunk to the next card, which
// overwrites its copy.  Bandwidth model: "分布式训练/推理", section "Ring
// all-reduce 的带宽账".
//
// Here the receiver pulls: at reduce-scatter step k, rank d reads the message
// of its predecessor r = d-1 for chunk c = (d-k-2) mod p (step 0: x_r[chunk
// c]; later: r's fp32 / int32 partial of chunk c) and its own x_d[chunk c],
// and stores partial_d[chunk c] = msg (+) x_d[chunk c]; at the last step
// (c == d) it stores y_d[chunk d] = cast(scale * acc) instead.  At
// all-gather step k, rank d copies y_{d-1}[chunk (d-k-1) mod p] into its own
// y_d.  Running steps 0 .. 2(p-1)-1, each for every rank, with every rank's
// step complete before any rank starts the next, reproduces the single-GPU
// literal ring (ring.cu) bit for bit: the same messages, the same fold.
// Partials live where ring.cu keeps them: in the receiver's own y (fp32,
// int32), or for bf16 in the receiver's workspace, two C-float slots by step
// parity (the sender's slot of step k-1 and the receiver's slot of step k are
// different memory, and a slot is rewritten two steps later, after its
// reader's step).
#include <algorithm>
#include <type_traits>

#include "common.cuh"
#include "internal.h"
#include "launch.cuh"

namespace rc {
namespace {

constexpr int kStepNT = 256;

struct StepParams {
  const char *msg;  // the sender's message: input type (first step) or 32-bit partial
  const char *own;  // x_d[chunk c] (input type)
  char *dst;        // d's 32-bit partial, or y_d[chunk d] (input type) on the last step
  uint64_t len;     // elements in chunk c
  uint64_t units;   // vectors (vector path) or elements (scalar path)
  float scale;
  int first, last;
};

// Partials are 32-bit: fp32 for fp32 and bf16 inputs, int32 for int32.
template <class T>
using PartialOf = typename std::conditional<std::is_same<T, I32>::value, I32, F32>::type;

// Vector path: one 16-byte vector of input per thread, grid-stride.
template <class T, int OP>
__global__ void __launch_bounds__(kStepNT) rc_rank_ring_step_kernel(const __grid_constant__ StepParams a) {
  using Acc = typename T::Acc;
  using P = PartialOf<T>;
  constexpr int VEC = kVec<T>;
  constexpr int PW = VEC / 4;  // 16-byte words of a vector's partial
  pdl_wait();
  for (uint64_t u = blockIdx.x * (uint64_t)kStepNT + threadIdx.x; u < a.units;
       u += (uint64_t)gridDim.x * kStepNT) {
    Acc acc[VEC];
    if (a.first) {
      unpack<T>(ld_stream_v4(a.msg + u * 16), acc);
    } else {
#pragma unroll
      for (int h = 0; h < PW; ++h) {
        typename P::Acc w[4];
        unpack<P>(ld_stream_v4(a.msg + u * (16 * PW) + 16 * h), w);
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[4 * h + j] = w[j];
      }
    }
    Acc x[VEC];
    unpack<T>(ld_stream_v4(a.own + u * 16), x);
#pragma unroll
    for (int e = 0; e < VEC; ++e) acc[e] = combine<OP>(acc[e], x[e]);
    if (a.last) {
#pragma unroll
      for (int e = 0; e < VEC; ++e) acc[e] = finish<OP>(acc[e], a.scale);
      store_vec<T, VEC>(a.dst + u * 16, acc);
    } else {
#pragma unroll
      for (int h = 0; h < PW; ++h) {
        typename P::Acc w[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) w[j] = acc[4 * h + j];
        store_vec<P, 4>(a.dst + u * (16 * PW) + 16 * h, w);
      }
    }
  }
}

// Scalar path (buffers or chunks not 16-byte aligned): element by element.
template <class T, int OP>
__global__ void __launch_bounds__(kStepNT) rc_rank_ring_step_scalar_kernel(const __grid_constant__ StepParams a) {
  using Acc = typename T::Acc;
  using P = PartialOf<T>;
  pdl_wait();
  for (uint64_t e = blockIdx.x * (uint64_t)kStepNT + threadIdx.x; e < a.len; e += (uint64_t)gridDim.x * kStepNT) {
    Acc acc = a.first ? load_elem<T>(a.msg, e) : (Acc)load_elem<P>(a.msg, e);
    acc = combine<OP>(acc, load_elem<T>(a.own, e));
    if (a.last) store_elem<T>(a.dst, e, finish<OP>(acc, a.scale));
    else store_elem<P>(a.dst, e, acc);
  }
}

template <class T, int OP>
cudaError_t run_step(const StepParams &in, cudaStream_t s) {
  StepParams a = in;
  constexpr int VEC = kVec<T>;
  const bool aligned = a.len % VEC == 0 && reinterpret_cast<uintptr_t>(a.msg) % 16 == 0 &&
                       reinterpret_cast<uintptr_t>(a.own) % 16 == 0 &&
                       reinterpret_cast<uintptr_t>(a.dst) % 16 == 0;
  const uint64_t cap = (uint64_t)device_sm_count() * (2048 / kStepNT);
  if (aligned) {
    a.units = a.len / VEC;
    const uint64_t grid = std::max<uint64_t>(1, std::min<uint64_t>(cap, (a.units + kStepNT - 1) / kStepNT));
    return launch_kernel(rc_rank_ring_step_kernel<T, OP>, dim3((unsigned)grid), dim3(kStepNT), 0, s, a);
  }
  a.units = a.len;
  const uint64_t grid = std::max<uint64_t>(1, std::min<uint64_t>(cap, (a.len + kStepNT - 1) / kStepNT));
  return launch_kernel(rc_rank_ring_step_scalar_kernel<T, OP>, dim3((unsigned)grid), dim3(kStepNT), 0, s, a);
}

template <class T>
cudaError_t step_by_op(const StepParams &a, int op, cudaStream_t s) {
  switch (op) {
    case kSum: return run_step<T, kSum>(a, s);
    case kMax: return run_step<T, kMax>(a, s);
    case kMin: return run_step<T, kMin>(a, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_rank_ring_step(const RankStepJob &job, cudaStream_t s) {
  const int p = job.p, d = job.rank, k = job.step;
  if (p < 2 || d < 0 || d >= p || k < 0 || k >= 2 * (p - 1)) return cudaErrorInvalidValue;
  const int esz = job.dt == kBF16 ? 2 : 4;
  const uint64_t n = job.n, C = (n + p - 1) / p;
  const int r = d == 0 ? p - 1 : d - 1;  // the sender
  auto chunk_len = [&](int c) -> uint64_t {
    const uint64_t b = (uint64_t)c * C;
    return b >= n ? 0 : (n - b < C ? n - b : C);
  };
  if (k >= p - 1) {  // all-gather step k - (p - 1): y_d[chunk c] = y_r[chunk c]
    const int ka = k - (p - 1);
    const int c = ((d - ka - 1) % p + p) % p;
    const uint64_t len = chunk_len(c);
    if (len == 0) return cudaSuccess;
    const uint64_t off = (uint64_t)c * C * esz;
    return launch_copy(static_cast<const char *>(job.y[r]) + off, static_cast<char *>(job.y[d]) + off,
                       len * esz, s);
  }
  const int c = ((d - k - 2) % p + p) % p;
  const uint64_t len = chunk_len(c);
  if (len == 0) return cudaSuccess;
  const bool bf16 = job.dt == kBF16;
  StepParams a{};
  a.len = len;
  a.scale = job.scale;
  a.first = k == 0;
  a.last = k == p - 2;
  const uint64_t in_off = (uint64_t)c * C * esz;  // chunk c in an input / output buffer
  // the sender's message and the receiver's partial slot
  if (a.first) a.msg = static_cast<const char *>(job.x[r]) + in_off;
  else if (bf16) a.msg = static_cast<const char *>(job.ws[r]) + (uint64_t)((k - 1) & 1) * C * 4;
  else a.msg = static_cast<const char *>(job.y[r]) + in_off;
  a.own = static_cast<const char *>(job.x[d]) + in_off;
  if (a.last) a.dst = static_cast<char *>(job.y[d]) + in_off;
  else if (bf16) a.dst = static_cast<char *>(job.ws[d]) + (uint64_t)(k & 1) * C * 4;
  else a.dst = static_cast<char *>(job.y[d]) + in_off;
  switch (job.dt) {
    case kF32: return step_by_op<F32>(a, job.op, s);
    case kBF16: return step_by_op<BF16>(a, job.op, s);
    case kI32: return step_by_op<I32>(a, job.op, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace rc
