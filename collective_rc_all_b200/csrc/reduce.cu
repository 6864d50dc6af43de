// reduce.cu -- the flat p-source reduction with register loads: reduce to
// root and reduce-scatter (fused with the scale and the output cast), the
// one-shot all-reduce when the shared-memory-staged fold (fold.cu) does not
// apply, the scalar path for unaligned buffers, and the scalar tail.
//
// Pages: "分布式训练/推理", section "通信原语：rank、world size 和 collective
// operations" (y = sum_r x_r, reduce-scatter keeps one slice of it), section
// "FSDP 的执行顺序" ((1/N_d) sum of gradients, reduce-scattered), and
// "LLM Parallelism 基础", section "Ring AllReduce" for the fold order.
//
// Design (HBM-bound: (p-1) adds per element, 0.1 flop/byte at p = 8):
//  * One thread owns whole 16-byte vectors: it issues all p 128-bit loads of
//    its ILP vectors (1 by default) before folding, so each thread keeps
//    p*ILP*16 bytes in flight (128 B at p = 8) with no shared memory and no
//    barriers.
//  * The fold order of element i depends only on its chunk c = i / C:
//    ranks (c+1)%p, ..., c.  Vectors never straddle a chunk (C % VEC == 0 is
//    required for the vector path), so the rotated rank list is computed once
//    per chunk segment and the p loads land in statically indexed registers.
//  * Vector path: one block per tile of 256*ILP vectors inside one chunk, so
//    the blocks sweep the ranks' buffers as a front (DRAM row locality; for
//    a read-heavy reduce-scatter this measured 16.4 us at p = 8, 8 MiB per
//    rank, against 20.5 us for the shared-memory-staged fold).
//  * Scalar path (unaligned buffers): persistent grid, CTA b owns the
//    contiguous element range [b*N/G, (b+1)*N/G).
//  * Results are written once per destination with 16-byte stores (8-byte for
//    an fp32 -> bf16 reduce-scatter).
#include <algorithm>
#include <type_traits>

#include "common.cuh"
#include "internal.h"
#include "launch.cuh"

namespace rc {
namespace {

constexpr int kNT = 256;

struct ReduceParams {
  const char *src[kMaxRanks];
  char *dst[kMaxRanks];  // kModeScatter: dst[c] already offset by -c*C elements
  uint64_t n;            // elements per rank
  uint64_t C;            // chunk length ceil(n/p)
  uint64_t nvec;         // number of units the grid splits (vectors or elements)
  float scale;
  int p;
  int mode;
  int ndst;  // outputs in kModeAll
  int c0;    // first chunk of the launch (chunk range [c0, c1))
};

__device__ __forceinline__ int rot(uint64_t c, int k, int p) {
  int r = (int)c + 1 + k;  // c < p, k < p  ->  r < 2p
  return r >= p ? r - p : r;
}

// Scalar path for buffers that are not 16-byte aligned (or chunks that do not
// keep 16-byte alignment): element by element, persistent grid, CTA b owns
// the contiguous element range [b*N/G, (b+1)*N/G).
template <int PMAX, class TI, class TO, int OP>
__global__ void __launch_bounds__(kNT) rc_reduce_scalar_kernel(const __grid_constant__ ReduceParams a) {
  using Acc = typename TI::Acc;
  pdl_wait();
  const int p = a.p;
  const uint64_t G = gridDim.x;
  // a.nvec elements starting at element c0 * C (the launch's chunk range)
  const uint64_t lo = (uint64_t)a.c0 * a.C;
  uint64_t u0 = lo + a.nvec * blockIdx.x / G;
  const uint64_t u1 = lo + a.nvec * (blockIdx.x + 1) / G;
  while (u0 < u1) {
    // all elements in [u0, useg) share chunk c, hence one fold order
    const uint64_t c = u0 / a.C;
    const uint64_t cend = (c + 1) * a.C;
    const uint64_t useg = u1 < cend ? u1 : cend;
    const char *s[PMAX];
#pragma unroll
    for (int k = 0; k < PMAX; ++k) s[k] = (k < p) ? a.src[rot(c, k, p)] : nullptr;
    char *d1 = a.dst[a.mode == kModeScatter ? c : 0];
    for (uint64_t e = u0 + threadIdx.x; e < useg; e += kNT) {
      Acc acc = load_elem<TI>(s[0], e);
#pragma unroll
      for (int k = 1; k < PMAX; ++k)
        if (k < p) acc = combine<OP>(acc, load_elem<TI>(s[k], e));
      acc = finish<OP>(acc, a.scale);
      if (a.mode == kModeAll) {
#pragma unroll
        for (int r = 0; r < PMAX; ++r)
          if (r < a.ndst) store_elem<TO>(a.dst[r], e, acc);
      } else {
        store_elem<TO>(d1, e, acc);
      }
    }
    u0 = useg;
  }
}

// Vector path: block t handles vectors [v0, v0 + 256*ILP) of chunk c.
template <int PMAX, class TI, class TO, int OP, int ILP>
__global__ void __launch_bounds__(kNT) rc_reduce_front_kernel(const __grid_constant__ ReduceParams a,
                                                              uint64_t tiles_per_chunk) {
  using Acc = typename TI::Acc;
  pdl_wait();
  constexpr int VEC = kVec<TI>;
  const int p = a.p;
  const uint64_t cvec = a.C / VEC;
  const uint64_t cl = blockIdx.x / tiles_per_chunk;  // chunk within the launch's range
  const uint64_t c = a.c0 + cl;
  const uint64_t v0 = c * cvec + (blockIdx.x - cl * tiles_per_chunk) * (uint64_t)(kNT * ILP);
  const uint64_t cend = (c + 1) * cvec;
  const uint64_t vend = cend < a.nvec ? cend : a.nvec;
  if (v0 >= vend) return;

  const char *s[PMAX];
#pragma unroll
  for (int k = 0; k < PMAX; ++k) s[k] = (k < p) ? a.src[rot(c, k, p)] : nullptr;
  uint4 raw[ILP][PMAX];
  bool live[ILP];
#pragma unroll
  for (int j = 0; j < ILP; ++j) {
    const uint64_t v = v0 + (uint64_t)j * kNT + threadIdx.x;
    live[j] = v < vend;
    if (live[j]) {
#pragma unroll
      for (int k = 0; k < PMAX; ++k)
        if (k < p) raw[j][k] = ld_stream_v4(s[k] + v * 16);
    }
  }
  char *d1 = a.dst[a.mode == kModeScatter ? c : 0];
#pragma unroll
  for (int j = 0; j < ILP; ++j) {
    if (!live[j]) continue;
    const uint64_t e = (v0 + (uint64_t)j * kNT + threadIdx.x) * VEC;
    Acc acc[VEC];
    unpack<TI>(raw[j][0], acc);
#pragma unroll
    for (int k = 1; k < PMAX; ++k) {
      if (k < p) {
        Acc v[VEC];
        unpack<TI>(raw[j][k], v);
#pragma unroll
        for (int q = 0; q < VEC; ++q) acc[q] = combine<OP>(acc[q], v[q]);
      }
    }
#pragma unroll
    for (int q = 0; q < VEC; ++q) acc[q] = finish<OP>(acc[q], a.scale);
    if (a.mode == kModeAll) {
#pragma unroll
      for (int r = 0; r < PMAX; ++r)
        if (r < a.ndst) store_vec<TO, VEC, true>(a.dst[r] + e * TO::kBytes, acc);
    } else if (a.mode == kModeOne) {
      store_vec<TO, VEC, true>(d1 + e * TO::kBytes, acc);
    } else {
      store_vec<TO, VEC>(d1 + e * TO::kBytes, acc);
    }
  }
}

// Elements past the last whole vector (n % VEC of them, all in the last
// chunk) -- one small CTA, scalar.
template <int PMAX, class TI, class TO, int OP>
__global__ void __launch_bounds__(32) rc_reduce_tail_kernel(const __grid_constant__ ReduceParams a,
                                                          uint64_t first, uint64_t last) {
  using Acc = typename TI::Acc;
  pdl_wait();
  const int p = a.p;
  for (uint64_t e = first + threadIdx.x; e < last; e += blockDim.x) {
    const uint64_t c = e / a.C;
    Acc acc = load_elem<TI>(a.src[rot(c, 0, p)], e);
    for (int k = 1; k < p; ++k) acc = combine<OP>(acc, load_elem<TI>(a.src[rot(c, k, p)], e));
    acc = finish<OP>(acc, a.scale);
    if (a.mode == kModeAll) {
      for (int r = 0; r < a.ndst; ++r) store_elem<TO>(a.dst[r], e, acc);
    } else {
      store_elem<TO>(a.dst[a.mode == kModeScatter ? c : 0], e, acc);
    }
  }
}

template <int PMAX, class TI, class TO, int OP>
cudaError_t run(const ReduceJob &job, cudaStream_t s) {
  ReduceParams a{};
  const int p = job.p;
  const uint64_t n = job.n;
  const uint64_t C = (n + p - 1) / p;
  a.n = n;
  a.C = C;
  a.p = p;
  a.mode = job.mode;
  a.scale = job.scale;
  a.ndst = job.mode == kModeAll ? (job.ndst > 0 ? job.ndst : p) : 1;
  const int c0 = job.c0, c1 = job.c1 > 0 ? job.c1 : p;
  if (c0 < 0 || c0 >= c1 || c1 > p) return cudaErrorInvalidValue;
  a.c0 = c0;
  const bool whole = (c0 == 0 && c1 == p);
  const uint64_t e_lo = std::min<uint64_t>(n, (uint64_t)c0 * C);  // the range's elements
  const uint64_t e_hi = std::min<uint64_t>(n, (uint64_t)c1 * C);
  bool aligned = true;
  for (int r = 0; r < p; ++r) {
    a.src[r] = static_cast<const char *>(job.src[r]);
    aligned = aligned && (reinterpret_cast<uintptr_t>(job.src[r]) % 16 == 0);
  }
  const int ndst = job.mode == kModeOne ? 1 : (job.mode == kModeAll ? a.ndst : p);
  for (int r = 0; r < ndst; ++r) {
    uintptr_t d = reinterpret_cast<uintptr_t>(job.dst[r]);
    aligned = aligned && (d % 16 == 0);
    if (job.mode == kModeScatter) d -= (uintptr_t)(r * C * TO::kBytes);  // index by global element
    a.dst[r] = reinterpret_cast<char *>(d);
  }
  constexpr int VEC = kVec<TI>;
  const bool vector = aligned && (C % VEC == 0);

  const int sms = device_sm_count();
  cudaError_t err;
  FoldJob f{};
  f.p = p;
  f.G = p;
  f.n = n;
  f.CG = C;
  f.CL = n;
  f.in_dt = job.in_dt;
  f.out_dt = job.out_dt;
  f.op = job.op;
  f.scale = job.scale;
  f.mode = job.mode;
  f.ndst = a.ndst;
  for (int r = 0; r < p; ++r) f.src[r] = job.src[r];
  for (int r = 0; r < ndst; ++r) f.dst[r] = job.dst[r];
  // The shared-memory-staged fold is the all-reduce's alternative path
  // (RC_AR_FOLD=1): with one vector per thread the register front kernel
  // measured faster for the p = 8 x 8 MiB fp32 all-reduce (23.4 vs 25.3 us
  // back to back, 20.5 vs 23.6 us alone).
  if (whole && vector && job.mode == kModeAll && env_int("RC_AR_FOLD", 0) && fold_tma_eligible(f)) {
    // the staged fold covers whole vectors; the tail (n % VEC elements) is scalar
    if ((err = launch_fold_tma(f, s)) != cudaSuccess) return err;
    a.nvec = n / VEC;
    if (a.nvec * VEC < n) {
      if ((err = launch_kernel(rc_reduce_tail_kernel<PMAX, TI, TO, OP>, dim3(1), dim3(32), 0, s, a,
                               a.nvec * VEC, n)) != cudaSuccess)
        return err;
    }
    return cudaSuccess;
  }
  if (e_lo == e_hi) return cudaSuccess;  // the range holds no element
  if (vector) {
    a.nvec = n / VEC;
    // whole vectors of the range: chunks are whole vectors, so only the last
    // chunk of the vector can end in a partial one
    if (std::min<uint64_t>(a.nvec * VEC, e_hi) > e_lo) {
      const uint64_t cvec = C / VEC;
      auto go = [&](auto ilp_tag) -> cudaError_t {
        constexpr int ILP = decltype(ilp_tag)::value;
        const uint64_t tpc = (cvec + kNT * ILP - 1) / (kNT * ILP);
        const uint64_t grid = tpc * (uint64_t)(c1 - c0);
        if (grid > 0x7fffffffull) return cudaErrorInvalidValue;
        return launch_kernel(rc_reduce_front_kernel<PMAX, TI, TO, OP, ILP>, dim3((unsigned)grid), dim3(kNT), 0,
                             s, a, tpc);
      };
      // one vector per thread: 12.0 vs 12.3 us for the p = 8 x 8 MiB fp32 ->
      // bf16 reduce-scatter replayed back to back (more blocks per SM, fewer
      // registers); RC_FRONT_ILP=2 selects two
      const int ilp = env_int("RC_FRONT_ILP", 1);
      err = ilp == 1 ? go(std::integral_constant<int, 1>()) : go(std::integral_constant<int, 2>());
      if (err != cudaSuccess) return err;
    }
    const uint64_t t0 = std::max<uint64_t>(a.nvec * VEC, e_lo);
    if (t0 < e_hi) {
      if ((err = launch_kernel(rc_reduce_tail_kernel<PMAX, TI, TO, OP>, dim3(1), dim3(32), 0, s, a, t0,
                               e_hi)) != cudaSuccess)
        return err;
    }
  } else {
    auto kern = rc_reduce_scalar_kernel<PMAX, TI, TO, OP>;
    int occ = 0;
    err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, kNT, 0);
    if (err != cudaSuccess) return err;
    a.nvec = e_hi - e_lo;  // elements, from c0 * C
    uint64_t grid = std::min<uint64_t>((uint64_t)sms * std::max(occ, 1), (a.nvec + kNT - 1) / kNT);
    grid = std::max<uint64_t>(grid, 1);
    if ((err = launch_kernel(kern, dim3((unsigned)grid), dim3(kNT), 0, s, a)) != cudaSuccess) return err;
  }
  return cudaSuccess;
}

template <class TI, class TO, int OP>
cudaError_t by_p(const ReduceJob &job, cudaStream_t s) {
  // PMAX bounds both the sources and (for kModeAll) the outputs
  const int w = std::max(job.p, job.mode == kModeAll && job.ndst > 0 ? job.ndst : job.p);
  if (w <= 2) return run<2, TI, TO, OP>(job, s);
  if (w <= 4) return run<4, TI, TO, OP>(job, s);
  if (w <= 8) return run<8, TI, TO, OP>(job, s);
  return run<16, TI, TO, OP>(job, s);
}

template <class TI, class TO>
cudaError_t by_op(const ReduceJob &job, cudaStream_t s) {
  switch (job.op) {
    case kSum: return by_p<TI, TO, kSum>(job, s);
    case kMax: return by_p<TI, TO, kMax>(job, s);
    case kMin: return by_p<TI, TO, kMin>(job, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_reduce(const ReduceJob &job, cudaStream_t s) {
  const int i = job.in_dt, o = job.out_dt;
  if (i == kF32 && o == kF32) return by_op<F32, F32>(job, s);
  if (i == kBF16 && o == kBF16) return by_op<BF16, BF16>(job, s);
  if (i == kI32 && o == kI32) return by_op<I32, I32>(job, s);
  if (i == kF32 && o == kBF16) return by_op<F32, BF16>(job, s);
  if (i == kBF16 && o == kF32) return by_op<BF16, F32>(job, s);
  return cudaErrorInvalidValue;
}

}  // namespace rc
