// internal.h -- job descriptions passed from the C ABI layer (api.cu) to the
// kernel launchers.  Not part of the public interface.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "rankcoll.h"

namespace rc {

constexpr int kMaxP = 16;

// Where a flat reduction writes its result.
enum ReduceMode : int {
  kModeAll = 0,      // every rank's recv buffer (all-reduce)
  kModeOne = 1,      // one buffer (reduce to root)
  kModeScatter = 2,  // chunk c to rank c's buffer at offset i - c*C (reduce-scatter)
};

struct ReduceJob {
  const void *src[kMaxP];
  void *dst[kMaxP];  // kModeAll: p buffers; kModeOne: dst[0]; kModeScatter: p shard buffers
  int p;
  uint64_t n;  // per-rank full-vector length
  int in_dt, out_dt, op;
  float scale;
  int mode;
  int ndst;  // kModeAll: number of outputs (0 means p)
  // Chunks [c0, c1) only (chunk length ceil(n/p)); c1 = 0 means all p.  A
  // rank's share of a collective is its own chunk.
  int c0, c1;
};

// A p-source fold over aligned 16-byte vectors (fold.cu).  G = p is the flat
// ring order (CG = ceil(n/p), CL = n); G < p is the hierarchical order.
struct FoldJob {
  const void *src[kMaxP];
  void *dst[kMaxP];
  int p, G;
  uint64_t n, CG, CL;
  int in_dt, out_dt, op;
  float scale;
  int mode;
  int ndst;  // outputs in kModeAll
};

struct FanoutJob {
  const void *src[kMaxP];  // nsrc sources of src_bytes each
  void *dst[kMaxP];        // p destinations; source r lands at dst[q] + r * src_bytes
  int nsrc;                // p (all-gather) or 1 (broadcast)
  int p;
  uint64_t src_bytes;
  uint32_t elem_bytes;     // 2 or 4 (for the unaligned fallback)
  uint32_t skip[kMaxP];    // bit r of skip[q]: leave (source r -> rank q) alone (in place)
};

struct RingJob {
  const void *x[kMaxP];  // send
  void *y[kMaxP];        // recv
  void *ws;              // fp32 partials when dt is bf16: 2 * p * C floats
  int p;
  uint64_t n;
  int dt, op;
  float scale;
  bool partials_in_ws;   // run a kernel that keeps bf16 partials in ws (chain / element form)
};

struct HierJob {
  const void *x[kMaxP];
  void *y[kMaxP];
  void *ws;  // staged variant: (ng + 1) * n accumulator values
  int p, G;
  uint64_t n;
  int dt, op;
  float scale;
};

// One step of the literal ring as executed by receiving rank `rank` (rank.cu):
// the p ranks' buffers as this process addresses them (own or peer-mapped).
struct RankStepJob {
  const void *x[kMaxP];  // send
  void *y[kMaxP];        // recv
  void *ws[kMaxP];       // bf16: each rank's 2 * ceil(n/p) fp32 partials
  int p, rank, step;
  uint64_t n;
  int dt, op;
  float scale;
};

// AdamW hyperparameters of one step (optim.cu).
struct AdamwHyper {
  float lr, beta1, beta2, eps, weight_decay;
  int64_t step;  // t >= 1
};

// ZeRO-1 step over p ranks (optim.cu): gradients in, full parameters out on
// every rank, fp32 master weights and moments sharded (rank r: n/p elements).
struct Zero1Job {
  const void *grad[kMaxP];
  void *param[kMaxP];
  float *master[kMaxP];
  float *exp_avg[kMaxP];
  float *exp_avg_sq[kMaxP];
  int p;
  uint64_t n;
  int grad_dt, param_dt;
  float scale;
  AdamwHyper hp;
};

// All-to-all with split counts (alltoall.cu): counts[r*p + q] elements of
// esz bytes go from rank r to rank q.
struct A2aJob {
  const void *send[kMaxP];
  void *recv[kMaxP];
  uint64_t counts[kMaxP * kMaxP];
  int p;
  int esz;
};

cudaError_t launch_reduce(const ReduceJob &job, cudaStream_t s);
bool fold_tma_eligible(const FoldJob &job);
cudaError_t launch_fold_tma(const FoldJob &job, cudaStream_t s);
cudaError_t read_and_clear_fold_timeouts(unsigned int *count);
cudaError_t launch_fanout(const FanoutJob &job, cudaStream_t s);
cudaError_t launch_ring_literal(const RingJob &job, cudaStream_t s);
// Whether launch_ring_literal will read job.ws (bf16 partials in device memory).
bool ring_needs_workspace(const RingJob &job);
size_t noalloc_scratch_floats();
cudaError_t noalloc_scratch_ptr(void **out);
void noalloc_scratch_forget();  // drop the cached addresses (rc_finalize)
cudaError_t launch_hier_fused(const HierJob &job, cudaStream_t s);
cudaError_t launch_hier_staged(const HierJob &job, cudaStream_t s);
cudaError_t launch_copy(const void *src, void *dst, size_t bytes, cudaStream_t s);
cudaError_t launch_rank_ring_step(const RankStepJob &job, cudaStream_t s);
cudaError_t launch_zero1(const Zero1Job &job, cudaStream_t s);
cudaError_t launch_all_to_all(const A2aJob &job, cudaStream_t s);
cudaError_t launch_adamw(float *param, float *exp_avg, float *exp_avg_sq, const void *grad, int grad_dt,
                         uint64_t n, const AdamwHyper &hp, cudaStream_t s);

cudaError_t launch_wait_probe(uint64_t limit_ns, cudaStream_t s);

// Device-side bounded waits report here (fanout.cu).
cudaError_t read_and_clear_wait_timeouts(unsigned int *count);

// Record msg as this thread's rc_last_error() and return st (api.cu).
rc_status report_error(rc_status st, const char *msg);

// Helpers shared by the launchers (api.cu).
int device_sm_count();        // SMs of the current device (cached)
void note_launches(int k);    // count kernels launched
int env_int(const char *name, int dflt);

}  // namespace rc
