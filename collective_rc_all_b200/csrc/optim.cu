// optim.cu -- the ZeRO-1 sharded optimizer step fused with its collectives,
// and a plain AdamW step.
//
// Page: "分布式训练/推理", section "显存账：不同数据并行的局限性" (ZeRO-1 shards the
// optimizer state -- the Adam moments and the fp32 master weights -- while
// every rank keeps the full parameters) and section "DDP 模型训练示例"
// (ShardedOptimizer: average the gradients, run AdamW on the parameters this
// rank owns, then give every rank the owner's parameters).  The pages name
// torch.optim.AdamW without printing it; the update is AdamW's published
// definition (decoupled weight decay, bias-corrected moments), t >= 1:
//   theta <- theta * (1 - lr*wd)
//   m     <- beta1*m + (1 - beta1)*g
//   v     <- beta2*v + (1 - beta2)*(g*g)
//   mhat  <- m / (1 - beta1^t)          vhat <- v / (1 - beta2^t)
//   theta <- theta - lr * (mhat / (sqrt(vhat) + eps))
// evaluated in binary32, one rounding per operation, in exactly this order
// (explicit round-to-nearest intrinsics, so no contraction can reorder it);
// the scalars 1 - lr*wd, 1 - beta1, 1 - beta2, 1 - beta1^t and 1 - beta2^t
// are binary64 expressions rounded to binary32 once on the host.
//
// rc_zero1_step, for p simulated ranks with n = p*m elements per rank:
//   g[i]          = scale * fold over the ranks' gradients at i, in the ring
//                   order of chunk c = i / m (the reduce-scatter: rank c owns
//                   shard c), accumulated in fp32
//   shard c       : AdamW on master[c][i - c*m], exp_avg[c][..], exp_avg_sq[c][..]
//   params[q][i]  = cast(master[c][i - c*m]) for every rank q (the all-gather)
// in ONE pass: each element's gradients are read once from every rank, its
// optimizer state is read and written once, and its new parameter is
// written once to every rank.  The reduce-scatter output and the all-gather
// input never exist in memory.
#include <algorithm>
#include <cmath>

#include "common.cuh"
#include "internal.h"
#include "launch.cuh"

namespace rc {
namespace {

constexpr int kNT = 256;

struct AdamwConsts {
  float lr, beta1, beta2, eps, decay, omb1, omb2, bc1, bc2;
};

__device__ __forceinline__ void adamw_elem(float &th, float &m, float &v, float g,
                                           const AdamwConsts &k) {
  float t = __fmul_rn(th, k.decay);
  const float mi = __fadd_rn(__fmul_rn(k.beta1, m), __fmul_rn(k.omb1, g));
  const float vi = __fadd_rn(__fmul_rn(k.beta2, v), __fmul_rn(k.omb2, __fmul_rn(g, g)));
  const float mhat = __fdiv_rn(mi, k.bc1);
  const float vhat = __fdiv_rn(vi, k.bc2);
  const float den = __fadd_rn(__fsqrt_rn(vhat), k.eps);
  t = __fsub_rn(t, __fmul_rn(k.lr, __fdiv_rn(mhat, den)));
  th = t;
  m = mi;
  v = vi;
}

// Coherent 16-byte load / store of optimizer state (read once, written once
// by the same thread).
__device__ __forceinline__ float4 ld_state(const float *p) {
  float4 v;
  asm volatile("ld.global.cg.v4.f32 {%0,%1,%2,%3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "l"(p)
               : "memory");
  return v;
}
__device__ __forceinline__ void st_state(float *p, float4 v) {
  asm volatile("st.global.cs.v4.f32 [%0], {%1,%2,%3,%4};" ::"l"(p), "f"(v.x), "f"(v.y), "f"(v.z),
               "f"(v.w)
               : "memory");
}

template <int VEC>
__device__ __forceinline__ void load_state(const float *p, float (&a)[VEC]) {
#pragma unroll
  for (int h = 0; h < VEC / 4; ++h) {
    const float4 v = ld_state(p + 4 * h);
    a[4 * h] = v.x;
    a[4 * h + 1] = v.y;
    a[4 * h + 2] = v.z;
    a[4 * h + 3] = v.w;
  }
}
template <int VEC>
__device__ __forceinline__ void store_state(float *p, const float (&a)[VEC]) {
#pragma unroll
  for (int h = 0; h < VEC / 4; ++h)
    st_state(p + 4 * h, make_float4(a[4 * h], a[4 * h + 1], a[4 * h + 2], a[4 * h + 3]));
}

struct Zero1Params {
  const char *grad[kMaxRanks];
  char *param[kMaxRanks];
  float *master[kMaxRanks];
  float *m1[kMaxRanks];
  float *m2[kMaxRanks];
  uint64_t n, m;  // elements per rank, shard length (n / p)
  float scale;
  int p;
  AdamwConsts k;
};

__device__ __forceinline__ int rot(uint64_t c, int k, int p) {
  int r = (int)c + 1 + k;  // c < p, k < p  ->  r < 2p
  return r >= p ? r - p : r;
}

// Vector path: block b handles vectors [v0, v0 + kNT*ILP) of shard (chunk) c;
// the blocks sweep the ranks' buffers as a front.
template <int PMAX, class TG, class TP, int ILP>
__global__ void __launch_bounds__(kNT) rc_zero1_front_kernel(const __grid_constant__ Zero1Params a,
                                                             uint64_t tiles_per_shard) {
  constexpr int VEC = kVec<TG>;
  pdl_wait();
  const int p = a.p;
  const uint64_t mvec = a.m / VEC;
  const uint64_t c = blockIdx.x / tiles_per_shard;
  const uint64_t j0 = (blockIdx.x - c * tiles_per_shard) * (uint64_t)(kNT * ILP);  // vector in shard
  if (j0 >= mvec) return;
  const char *s[PMAX];
#pragma unroll
  for (int k = 0; k < PMAX; ++k) s[k] = (k < p) ? a.grad[rot(c, k, p)] : nullptr;
  const uint64_t base = c * mvec;  // first vector of shard c in the full vector
  uint4 raw[ILP][PMAX];
  bool live[ILP];
#pragma unroll
  for (int j = 0; j < ILP; ++j) {
    const uint64_t jv = j0 + (uint64_t)j * kNT + threadIdx.x;
    live[j] = jv < mvec;
    if (live[j]) {
#pragma unroll
      for (int k = 0; k < PMAX; ++k)
        if (k < p) raw[j][k] = ld_stream_v4(s[k] + (base + jv) * 16);
    }
  }
  float *mas = a.master[c], *m1 = a.m1[c], *m2 = a.m2[c];
#pragma unroll
  for (int j = 0; j < ILP; ++j) {
    if (!live[j]) continue;
    const uint64_t jv = j0 + (uint64_t)j * kNT + threadIdx.x;
    const uint64_t e = jv * VEC;  // element in the shard
    float th[VEC], mo[VEC], vo[VEC];
    load_state<VEC>(mas + e, th);
    load_state<VEC>(m1 + e, mo);
    load_state<VEC>(m2 + e, vo);
    float g[VEC];
    unpack<TG>(raw[j][0], g);
#pragma unroll
    for (int k = 1; k < PMAX; ++k) {
      if (k < p) {
        float x[VEC];
        unpack<TG>(raw[j][k], x);
#pragma unroll
        for (int q = 0; q < VEC; ++q) g[q] = combine<kSum>(g[q], x[q]);
      }
    }
#pragma unroll
    for (int q = 0; q < VEC; ++q) {
      g[q] = finish<kSum>(g[q], a.scale);
      adamw_elem(th[q], mo[q], vo[q], g[q], a.k);
    }
    store_state<VEC>(mas + e, th);
    store_state<VEC>(m1 + e, mo);
    store_state<VEC>(m2 + e, vo);
    const uint64_t off = ((base + jv) * VEC) * (uint64_t)TP::kBytes;
#pragma unroll
    for (int r = 0; r < PMAX; ++r)
      if (r < p) store_vec<TP, VEC>(a.param[r] + off, th);
  }
}

// Element path (buffers not 16-byte aligned, or a shard length that is not a
// whole number of vectors): grid-stride over the n elements.
template <int PMAX, class TG, class TP>
__global__ void __launch_bounds__(kNT) rc_zero1_elem_kernel(const __grid_constant__ Zero1Params a) {
  pdl_wait();
  const int p = a.p;
  for (uint64_t i = blockIdx.x * (uint64_t)kNT + threadIdx.x; i < a.n; i += (uint64_t)gridDim.x * kNT) {
    const uint64_t c = i / a.m, j = i - c * a.m;
    float g = load_elem<TG>(a.grad[rot(c, 0, p)], i);
    for (int k = 1; k < p; ++k) g = combine<kSum>(g, (float)load_elem<TG>(a.grad[rot(c, k, p)], i));
    g = finish<kSum>(g, a.scale);
    float th = a.master[c][j], mo = a.m1[c][j], vo = a.m2[c][j];
    adamw_elem(th, mo, vo, g, a.k);
    a.master[c][j] = th;
    a.m1[c][j] = mo;
    a.m2[c][j] = vo;
    for (int r = 0; r < p; ++r) store_elem<TP>(a.param[r], i, th);
  }
}

// Plain AdamW on one array (the unfused step and the owner-broadcast form).
struct AdamwParams {
  float *th, *m1, *m2;
  const char *grad;
  uint64_t n;
  AdamwConsts k;
  int vector;
};

template <class TG>
__global__ void __launch_bounds__(kNT) rc_adamw_kernel(const __grid_constant__ AdamwParams a) {
  constexpr int VEC = kVec<TG>;
  pdl_wait();
  const uint64_t stride = (uint64_t)gridDim.x * kNT;
  uint64_t done = 0;
  if (a.vector) {
    const uint64_t nv = a.n / VEC;
    for (uint64_t v = blockIdx.x * (uint64_t)kNT + threadIdx.x; v < nv; v += stride) {
      const uint64_t e = v * VEC;
      float th[VEC], mo[VEC], vo[VEC], g[VEC];
      unpack<TG>(ld_stream_v4(a.grad + v * 16), g);
      load_state<VEC>(a.th + e, th);
      load_state<VEC>(a.m1 + e, mo);
      load_state<VEC>(a.m2 + e, vo);
#pragma unroll
      for (int q = 0; q < VEC; ++q) adamw_elem(th[q], mo[q], vo[q], g[q], a.k);
      store_state<VEC>(a.th + e, th);
      store_state<VEC>(a.m1 + e, mo);
      store_state<VEC>(a.m2 + e, vo);
    }
    done = nv * VEC;
  }
  for (uint64_t i = done + blockIdx.x * (uint64_t)kNT + threadIdx.x; i < a.n; i += stride) {
    float th = a.th[i], mo = a.m1[i], vo = a.m2[i];
    adamw_elem(th, mo, vo, load_elem<TG>(a.grad, i), a.k);
    a.th[i] = th;
    a.m1[i] = mo;
    a.m2[i] = vo;
  }
}

AdamwConsts make_consts(const AdamwHyper &h) {
  AdamwConsts k;
  k.lr = h.lr;
  k.beta1 = h.beta1;
  k.beta2 = h.beta2;
  k.eps = h.eps;
  k.decay = (float)(1.0 - (double)h.lr * (double)h.weight_decay);
  k.omb1 = (float)(1.0 - (double)h.beta1);
  k.omb2 = (float)(1.0 - (double)h.beta2);
  k.bc1 = (float)(1.0 - std::pow((double)h.beta1, (double)h.step));
  k.bc2 = (float)(1.0 - std::pow((double)h.beta2, (double)h.step));
  return k;
}

template <int PMAX, class TG, class TP>
cudaError_t run_zero1(const Zero1Job &job, cudaStream_t s) {
  Zero1Params a{};
  const int p = job.p;
  a.p = p;
  a.n = job.n;
  a.m = job.n / p;
  a.scale = job.scale;
  a.k = make_consts(job.hp);
  constexpr int VEC = kVec<TG>;
  bool aligned = a.m % VEC == 0;
  for (int r = 0; r < p; ++r) {
    a.grad[r] = static_cast<const char *>(job.grad[r]);
    a.param[r] = static_cast<char *>(job.param[r]);
    a.master[r] = job.master[r];
    a.m1[r] = job.exp_avg[r];
    a.m2[r] = job.exp_avg_sq[r];
    aligned = aligned && reinterpret_cast<uintptr_t>(job.grad[r]) % 16 == 0 &&
              reinterpret_cast<uintptr_t>(job.param[r]) % 16 == 0 &&
              reinterpret_cast<uintptr_t>(job.master[r]) % 16 == 0 &&
              reinterpret_cast<uintptr_t>(job.exp_avg[r]) % 16 == 0 &&
              reinterpret_cast<uintptr_t>(job.exp_avg_sq[r]) % 16 == 0;
  }
  if (aligned) {
    const uint64_t mvec = a.m / VEC;
    auto go = [&](auto ilp_tag) -> cudaError_t {
      constexpr int ILP = decltype(ilp_tag)::value;
      const uint64_t tps = (mvec + kNT * ILP - 1) / (kNT * ILP);
      const uint64_t grid = tps * (uint64_t)p;
      if (grid == 0) return cudaSuccess;
      if (grid > 0x7fffffffull) return cudaErrorInvalidValue;
      return launch_kernel(rc_zero1_front_kernel<PMAX, TG, TP, ILP>, dim3((unsigned)grid), dim3(kNT), 0, s,
                           a, tps);
    };
    // one vector per thread (52 registers, 4 blocks per SM) measured 2.19 ms
    // against 2.52 ms for two (95 registers, 2 blocks) on a Llama-2-7B layer
    // with bf16 parameters; RC_ZERO1_ILP=2 selects two
    if (env_int("RC_ZERO1_ILP", 1) == 2) return go(std::integral_constant<int, 2>());
    return go(std::integral_constant<int, 1>());
  }
  const uint64_t grid = std::max<uint64_t>(
      1, std::min<uint64_t>((a.n + kNT - 1) / kNT, (uint64_t)device_sm_count() * 8));
  return launch_kernel(rc_zero1_elem_kernel<PMAX, TG, TP>, dim3((unsigned)grid), dim3(kNT), 0, s, a);
}

template <class TG, class TP>
cudaError_t zero1_by_p(const Zero1Job &job, cudaStream_t s) {
  if (job.p <= 2) return run_zero1<2, TG, TP>(job, s);
  if (job.p <= 4) return run_zero1<4, TG, TP>(job, s);
  if (job.p <= 8) return run_zero1<8, TG, TP>(job, s);
  return run_zero1<16, TG, TP>(job, s);
}

}  // namespace

cudaError_t launch_zero1(const Zero1Job &job, cudaStream_t s) {
  const int g = job.grad_dt, q = job.param_dt;
  if (g == kF32 && q == kF32) return zero1_by_p<F32, F32>(job, s);
  if (g == kF32 && q == kBF16) return zero1_by_p<F32, BF16>(job, s);
  if (g == kBF16 && q == kF32) return zero1_by_p<BF16, F32>(job, s);
  if (g == kBF16 && q == kBF16) return zero1_by_p<BF16, BF16>(job, s);
  return cudaErrorInvalidValue;
}

cudaError_t launch_adamw(float *param, float *exp_avg, float *exp_avg_sq, const void *grad, int grad_dt,
                         uint64_t n, const AdamwHyper &hp, cudaStream_t s) {
  if (n == 0) return cudaSuccess;
  AdamwParams a{};
  a.th = param;
  a.m1 = exp_avg;
  a.m2 = exp_avg_sq;
  a.grad = static_cast<const char *>(grad);
  a.n = n;
  a.k = make_consts(hp);
  a.vector = reinterpret_cast<uintptr_t>(param) % 16 == 0 && reinterpret_cast<uintptr_t>(exp_avg) % 16 == 0 &&
             reinterpret_cast<uintptr_t>(exp_avg_sq) % 16 == 0 && reinterpret_cast<uintptr_t>(grad) % 16 == 0;
  const int vec = grad_dt == kBF16 ? 8 : 4;
  const uint64_t units = a.vector ? std::max<uint64_t>(1, n / vec) : n;
  const uint64_t grid = std::max<uint64_t>(
      1, std::min<uint64_t>((units + kNT - 1) / kNT, (uint64_t)device_sm_count() * 8));
  if (grad_dt == kF32) return launch_kernel(rc_adamw_kernel<F32>, dim3((unsigned)grid), dim3(kNT), 0, s, a);
  if (grad_dt == kBF16) return launch_kernel(rc_adamw_kernel<BF16>, dim3((unsigned)grid), dim3(kNT), 0, s, a);
  return cudaErrorInvalidValue;
}

}  // namespace rc
