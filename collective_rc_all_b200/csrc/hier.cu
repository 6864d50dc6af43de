// hier.cu -- two-level (hierarchical) all-reduce.
//
// Page: "大模型并行的最小闭环：集合通信、TP、FSDP/ZeRO-3 到权重分片", log excerpt
// "分层 AllReduce + SHARP": 2 nodes x 4 GPUs; step 1 an AllReduce inside each
// node; step 2 one representative (GPU0) per node; steps 3-5 the
// representatives' vectors go up, the switch computes A + B and sends the
// sum back; step 6 each representative broadcasts inside its node.
//
// Groups are contiguous blocks of G ranks; group g's leader is its local
// rank 0.  Order contract (shared with the CPU oracle):
//   S_g[i] = fold over the group's members in ring order of a G-member ring
//            (chunk length CG = ceil(n/G), member (cg+1)%G first, cg last);
//   T[i]   = fold over S_0..S_{ng-1} in ring order of an ng-member ring
//            (chunk length CL = ceil(n/ng));
//   y[i]   = cast(scale * T[i]) on every rank.
//
// Fused variant: one launch; each thread loads all p values of a 16-byte
// vector, folds each group, then the group results, and writes the result p
// times -- the all-reduce minimum traffic, group partials in registers.
// Staged variant: the page's phases as separate launches over an fp32
// workspace -- per group a reduce to S_g, the leader sum to T, the cast to
// each leader's buffer, then per group a broadcast from its leader.
#include <algorithm>

#include "common.cuh"
#include "internal.h"
#include "launch.cuh"

namespace rc {
namespace {

constexpr int kNT = 256;

struct HierParams {
  const char *x[kMaxRanks];
  char *y[kMaxRanks];
  uint64_t n, CG, CL, units;
  float scale;
  int p, G, ng;
};

template <int PMAX, class T, int OP, bool VECTOR>
__global__ void __launch_bounds__(kNT) rc_hier_reg_kernel(const __grid_constant__ HierParams a) {
  using Acc = typename T::Acc;
  constexpr int VEC = VECTOR ? kVec<T> : 1;
  const int p = a.p, G = a.G, ng = a.ng;
  pdl_wait();
  const uint64_t Gd = gridDim.x;
  uint64_t u0 = a.units * blockIdx.x / Gd;
  const uint64_t u1 = a.units * (blockIdx.x + 1) / Gd;

  while (u0 < u1) {
    // segment with one intra-group chunk index cg and one leader chunk index cl
    const uint64_t e0 = u0 * VEC;
    const uint64_t cg = e0 / a.CG, cl = e0 / a.CL;
    const uint64_t end_g = (cg + 1) * a.CG, end_l = (cl + 1) * a.CL;
    const uint64_t end_u = ((end_g < end_l ? end_g : end_l) + VEC - 1) / VEC;
    const uint64_t useg = u1 < end_u ? u1 : end_u;

    // fold position k = t*G + j: t-th group in leader order, j-th member in
    // group order; first/last flags mark group boundaries
    const char *s[PMAX];
    uint32_t first = 0, lastm = 0;
#pragma unroll
    for (int k = 0; k < PMAX; ++k) {
      s[k] = nullptr;
      if (k < p) {
        const int t = k / G, j = k - t * G;
        int gg = (int)cl + 1 + t;
        gg = gg >= ng ? gg - ng : gg;
        gg = gg >= ng ? gg - ng : gg;
        int m = (int)cg + 1 + j;
        m = m >= G ? m - G : m;
        m = m >= G ? m - G : m;
        s[k] = a.x[gg * G + m];
        if (j == 0) first |= 1u << k;
        if (j == G - 1) lastm |= 1u << k;
      }
    }

    for (uint64_t u = u0 + threadIdx.x; u < useg; u += kNT) {
      const uint64_t e = u * VEC;
      Acc v[PMAX][VEC];
#pragma unroll
      for (int k = 0; k < PMAX; ++k) {
        if (k < p) {
          if constexpr (VECTOR) unpack<T>(ld_stream_v4(s[k] + u * 16), v[k]);
          else v[k][0] = load_elem<T>(s[k], e);
        }
      }
      Acc S[VEC], Tt[VEC];
#pragma unroll
      for (int k = 0; k < PMAX; ++k) {
        if (k < p) {
#pragma unroll
          for (int q = 0; q < VEC; ++q) S[q] = ((first >> k) & 1u) ? v[k][q] : combine<OP>(S[q], v[k][q]);
          if ((lastm >> k) & 1u) {
#pragma unroll
            for (int q = 0; q < VEC; ++q) Tt[q] = (k < G) ? S[q] : combine<OP>(Tt[q], S[q]);
          }
        }
      }
#pragma unroll
      for (int q = 0; q < VEC; ++q) Tt[q] = finish<OP>(Tt[q], a.scale);
#pragma unroll
      for (int r = 0; r < PMAX; ++r) {
        if (r < p) {
          if constexpr (VECTOR) store_vec<T, VEC>(a.y[r] + e * T::kBytes, Tt);
          else store_elem<T>(a.y[r], e, Tt[0]);
        }
      }
    }
    u0 = useg;
  }
}

// Front kernel (default fused path): one 256-thread block per 256 vectors of
// one segment, the segments being the runs of S = min(CG, CL) elements on
// which both chunk indices are constant (used when the larger chunk length is
// a multiple of the smaller, as for every p and G that divide n evenly).
// Each thread loads the p vectors of its offset in the segment's fold order
// -- position k = t*GS + j is rank ((cl+1+t) mod ng)*GS + (cg+1+j) mod GS --
// folds each group of GS, then the group results, and writes the result to
// every rank.  Group size compile-time (GS), so the boundaries cost nothing.
template <int PMAX, class T, int OP, int GS>
__global__ void __launch_bounds__(kNT) rc_hier_front_kernel(const __grid_constant__ HierParams a,
                                                            uint64_t seg_vecs, uint64_t tiles_per_seg) {
  using Acc = typename T::Acc;
  constexpr int VEC = kVec<T>;
  pdl_wait();
  const int p = a.p, ng = a.ng;
  const uint64_t sg = blockIdx.x / tiles_per_seg;
  const uint64_t v0 = sg * seg_vecs + (blockIdx.x - sg * tiles_per_seg) * (uint64_t)kNT;
  const uint64_t vend0 = (sg + 1) * seg_vecs, nv = a.n / VEC;
  const uint64_t vend = vend0 < nv ? vend0 : nv;
  const uint64_t v = v0 + threadIdx.x;
  if (v >= vend) return;
  const uint64_t e0 = sg * seg_vecs * VEC;  // first element of the segment
  const int cg = (int)(e0 / a.CG), cl = (int)(e0 / a.CL);
  uint4 raw[PMAX];
#pragma unroll
  for (int k = 0; k < PMAX; ++k) {
    if (k < p) {
      const int t = k / GS, j = k - t * GS;
      int gg = cl + 1 + t;
      while (gg >= ng) gg -= ng;
      int m = cg + 1 + j;
      while (m >= GS) m -= GS;
      raw[k] = ld_stream_v4(a.x[gg * GS + m] + v * 16);
    }
  }
  Acc tot[VEC], grp[VEC];
#pragma unroll
  for (int k = 0; k < PMAX; ++k) {
    if (k < p) {
      Acc x[VEC];
      unpack<T>(raw[k], x);
      if (k % GS == 0) {
#pragma unroll
        for (int q = 0; q < VEC; ++q) grp[q] = x[q];
      } else {
#pragma unroll
        for (int q = 0; q < VEC; ++q) grp[q] = combine<OP>(grp[q], x[q]);
      }
      if (k % GS == GS - 1) {
        if (k < GS) {
#pragma unroll
          for (int q = 0; q < VEC; ++q) tot[q] = grp[q];
        } else {
#pragma unroll
          for (int q = 0; q < VEC; ++q) tot[q] = combine<OP>(tot[q], grp[q]);
        }
      }
    }
  }
#pragma unroll
  for (int q = 0; q < VEC; ++q) tot[q] = finish<OP>(tot[q], a.scale);
  const uint64_t off = v * VEC * (uint64_t)T::kBytes;
#pragma unroll
  for (int r = 0; r < PMAX; ++r)
    if (r < p) store_vec<T, VEC, true>(a.y[r] + off, tot);
}

template <int PMAX, class T, int OP>
cudaError_t try_front(const HierJob &job, cudaStream_t s, bool *done) {
  *done = false;
  constexpr int VEC = kVec<T>;
  HierParams a{};
  a.p = job.p;
  a.G = job.G;
  a.ng = job.p / job.G;
  a.n = job.n;
  a.CG = (job.n + a.G - 1) / a.G;
  a.CL = (job.n + a.ng - 1) / a.ng;
  a.scale = job.scale;
  bool ok = a.n % VEC == 0 && a.CG % VEC == 0 && a.CL % VEC == 0;
  for (int r = 0; r < job.p; ++r) {
    a.x[r] = static_cast<const char *>(job.x[r]);
    a.y[r] = static_cast<char *>(job.y[r]);
    ok = ok && reinterpret_cast<uintptr_t>(job.x[r]) % 16 == 0 && reinterpret_cast<uintptr_t>(job.y[r]) % 16 == 0;
  }
  const uint64_t S = std::min(a.CG, a.CL), Lg = std::max(a.CG, a.CL);
  ok = ok && S > 0 && Lg % S == 0 && (job.G == 2 || job.G == 4 || job.G == 8);
  if (!ok) return cudaSuccess;
  const uint64_t seg_vecs = S / VEC;
  const uint64_t nseg = (a.n / VEC + seg_vecs - 1) / seg_vecs;
  const uint64_t tps = (seg_vecs + kNT - 1) / kNT;
  const uint64_t grid = nseg * tps;
  if (grid == 0 || grid > 0x7fffffffull) return cudaSuccess;
  *done = true;
  if (job.G == 2) return launch_kernel(rc_hier_front_kernel<PMAX, T, OP, 2>, dim3((unsigned)grid), dim3(kNT), 0, s, a, seg_vecs, tps);
  if (job.G == 4) return launch_kernel(rc_hier_front_kernel<PMAX, T, OP, 4>, dim3((unsigned)grid), dim3(kNT), 0, s, a, seg_vecs, tps);
  return launch_kernel(rc_hier_front_kernel<PMAX, T, OP, 8>, dim3((unsigned)grid), dim3(kNT), 0, s, a, seg_vecs, tps);
}

template <class T, int OP>
cudaError_t front_by_p(const HierJob &job, cudaStream_t s, bool *done) {
  if (job.p <= 4) return try_front<4, T, OP>(job, s, done);
  if (job.p <= 8) return try_front<8, T, OP>(job, s, done);
  return try_front<16, T, OP>(job, s, done);
}

template <class T>
cudaError_t front_by_op(const HierJob &job, cudaStream_t s, bool *done) {
  switch (job.op) {
    case kSum: return front_by_p<T, kSum>(job, s, done);
    case kMax: return front_by_p<T, kMax>(job, s, done);
    case kMin: return front_by_p<T, kMin>(job, s, done);
  }
  *done = false;
  return cudaSuccess;
}

template <int PMAX, class T, int OP>
cudaError_t run_fused(const HierJob &job, cudaStream_t s) {
  HierParams a{};
  a.p = job.p;
  a.G = job.G;
  a.ng = job.p / job.G;
  a.n = job.n;
  a.CG = (job.n + a.G - 1) / a.G;
  a.CL = (job.n + a.ng - 1) / a.ng;
  a.scale = job.scale;
  bool aligned = true;
  for (int r = 0; r < job.p; ++r) {
    a.x[r] = static_cast<const char *>(job.x[r]);
    a.y[r] = static_cast<char *>(job.y[r]);
    aligned = aligned && reinterpret_cast<uintptr_t>(job.x[r]) % 16 == 0 &&
              reinterpret_cast<uintptr_t>(job.y[r]) % 16 == 0;
  }
  constexpr int VEC = kVec<T>;
  const bool vector = aligned && a.CG % VEC == 0 && a.CL % VEC == 0 && a.n % VEC == 0;
  auto kern = vector ? rc_hier_reg_kernel<PMAX, T, OP, true> : rc_hier_reg_kernel<PMAX, T, OP, false>;
  a.units = vector ? a.n / VEC : a.n;
  int occ = 0;
  cudaError_t err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, kNT, 0);
  if (err != cudaSuccess) return err;
  occ = std::max(1, std::min(occ, env_int("RC_CTAS_PER_SM", occ)));
  uint64_t grid = std::min<uint64_t>((uint64_t)device_sm_count() * occ, (a.units + kNT - 1) / kNT);
  grid = std::max<uint64_t>(grid, 1);
  return launch_kernel(kern, dim3((unsigned)grid), dim3(kNT), 0, s, a);
}

template <class T, int OP>
cudaError_t fused_by_p(const HierJob &job, cudaStream_t s) {
  if (job.p <= 4) return run_fused<4, T, OP>(job, s);
  if (job.p <= 8) return run_fused<8, T, OP>(job, s);
  return run_fused<16, T, OP>(job, s);
}

template <class T>
cudaError_t fused_by_op(const HierJob &job, cudaStream_t s) {
  switch (job.op) {
    case kSum: return fused_by_p<T, kSum>(job, s);
    case kMax: return fused_by_p<T, kMax>(job, s);
    case kMin: return fused_by_p<T, kMin>(job, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_hier_fused(const HierJob &job, cudaStream_t s) {
  FoldJob f{};
  f.p = job.p;
  f.G = job.G;
  f.n = job.n;
  f.CG = (job.n + job.G - 1) / job.G;
  f.CL = (job.n + job.p / job.G - 1) / (job.p / job.G);
  f.in_dt = f.out_dt = job.dt;
  f.op = job.op;
  f.scale = job.scale;
  f.mode = kModeAll;
  f.ndst = job.p;
  for (int r = 0; r < job.p; ++r) {
    f.src[r] = job.x[r];
    f.dst[r] = job.y[r];
  }
  // default: the register front kernel; RC_HIER_FOLD=1 selects the
  // shared-memory-staged fold (both give the same bits)
  if (!env_int("RC_HIER_FOLD", 0)) {
    bool done = false;
    cudaError_t err = cudaSuccess;
    switch (job.dt) {
      case kF32: err = front_by_op<F32>(job, s, &done); break;
      case kBF16: err = front_by_op<BF16>(job, s, &done); break;
      case kI32: err = front_by_op<I32>(job, s, &done); break;
    }
    if (done || err != cudaSuccess) return err;
  }
  if (fold_tma_eligible(f)) return launch_fold_tma(f, s);
  switch (job.dt) {
    case kF32: return fused_by_op<F32>(job, s);
    case kBF16: return fused_by_op<BF16>(job, s);
    case kI32: return fused_by_op<I32>(job, s);
  }
  return cudaErrorInvalidValue;
}

// Staged: the page's phases one after another.  Workspace layout (accumulator
// type: fp32, or int32 for int32): [S_0 | S_1 | ... | S_{ng-1} | T], n each.
cudaError_t launch_hier_staged(const HierJob &job, cudaStream_t s) {
  const int p = job.p, G = job.G, ng = p / G;
  const int acc_dt = job.dt == kI32 ? kI32 : kF32;
  const uint64_t n = job.n;
  char *ws = static_cast<char *>(job.ws);
  auto S = [&](int g) { return static_cast<void *>(ws + (uint64_t)g * n * 4); };
  void *T = ws + (uint64_t)ng * n * 4;
  cudaError_t err;

  // step 1: inside each group, fold the members in the group's ring order
  for (int g = 0; g < ng; ++g) {
    ReduceJob j{};
    j.p = G;
    j.n = n;
    for (int m = 0; m < G; ++m) j.src[m] = job.x[g * G + m];
    j.dst[0] = S(g);
    j.in_dt = job.dt;
    j.out_dt = acc_dt;
    j.op = job.op;
    j.scale = 1.0f;
    j.mode = kModeOne;
    if ((err = launch_reduce(j, s)) != cudaSuccess) return err;
  }
  // steps 3-5: the leaders' results are combined in ring order over groups
  {
    ReduceJob j{};
    j.p = ng;
    j.n = n;
    for (int g = 0; g < ng; ++g) j.src[g] = S(g);
    j.dst[0] = T;
    j.in_dt = acc_dt;
    j.out_dt = acc_dt;
    j.op = job.op;
    j.scale = 1.0f;
    j.mode = kModeOne;
    if ((err = launch_reduce(j, s)) != cudaSuccess) return err;
  }
  // step 5 (downlink): scale and cast once into every leader's buffer
  {
    ReduceJob j{};
    j.p = 1;
    j.n = n;
    j.src[0] = T;
    for (int g = 0; g < ng; ++g) j.dst[g] = job.y[g * G];
    j.ndst = ng;
    j.in_dt = acc_dt;
    j.out_dt = job.dt;
    j.op = job.op;
    j.scale = job.scale;
    j.mode = kModeAll;
    if ((err = launch_reduce(j, s)) != cudaSuccess) return err;
  }
  // step 6: each leader broadcasts inside its group
  if (G > 1) {
    const uint32_t esz = job.dt == kBF16 ? 2 : 4;
    for (int g = 0; g < ng; ++g) {
      FanoutJob f{};
      f.nsrc = 1;
      f.p = G - 1;
      f.src[0] = job.y[g * G];
      for (int m = 1; m < G; ++m) f.dst[m - 1] = job.y[g * G + m];
      f.src_bytes = n * esz;
      f.elem_bytes = esz;
      if ((err = launch_fanout(f, s)) != cudaSuccess) return err;
    }
  }
  return cudaSuccess;
}

}  // namespace rc
