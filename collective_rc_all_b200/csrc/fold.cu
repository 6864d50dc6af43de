// fold.cu -- the TMA-staged p-source fold: one-shot all-reduce, reduce,
// reduce-scatter (fused with the scale and the output cast) and the fused
// hierarchical all-reduce.
//
// Pages: "分布式训练/推理", section "通信原语：rank、world size 和 collective
// operations" (y = sum_r x_r; reduce-scatter keeps slice r; all-reduce gives y
// to every rank), section "FSDP 的执行顺序" ((1/N_d) sum of gradients,
// reduce-scattered); "LLM Parallelism 基础", section "Ring AllReduce" (the
// fold order); "大模型并行的最小闭环", log excerpt "分层 AllReduce + SHARP"
// (intra-node fold, the node results added, broadcast).
//
// Fold order.  The vector is cut into segments on which the order is fixed:
// flat folds (G = p) change order at every chunk boundary c*C; the
// hierarchical fold (groups of G, ng = p/G groups) at multiples of
// CG = ceil(n/G) and CL = ceil(n/ng).  On a segment with intra-group chunk cg
// and leader chunk cl, fold position k = t*G + j reads rank
//   gg*G + m,  gg = (cl+1+t) mod ng,  m = (cg+1+j) mod G,
// and the fold restarts at every group start and folds the group results in
// position order.  With G = p this is exactly the flat ring order.
//
// Pipeline (one CTA per SM, persistent, tiles interleaved across CTAs),
// warp-specialised:
//   * a tile is tv 16-byte vectors of every source, inside one segment;
//   * a producer warp (one lane) streams tiles into S shared-memory stages
//     with p bulk copies global -> this CTA's shared memory each, completion
//     counted on the stage's "full" mbarrier; it refills a stage as soon as
//     the stage's "empty" mbarrier says all consumer warps are done with it;
//   * 8 consumer warps fold each tile from shared memory (conflict-free
//     16-byte reads, sources already in fold order) and write the result with
//     16-byte stores (8-byte for fp32 -> bf16), then arrive on "empty".
// No CTA-wide barrier in the loop.  Every wait is bounded (global timer); on
// expiry the thread counts the event and stops; the producer always waits
// (bounded) for its own copies in flight before it leaves.
#include <algorithm>
#include <atomic>
#include <vector>

#include "bulk.cuh"
#include "common.cuh"
#include "internal.h"
#include "launch.cuh"

namespace rc {

// Number of bounded waits of this file's kernels that gave up.
__device__ unsigned int g_wait_timeouts_fold = 0;

namespace {

constexpr int kConsumerWarps = 8;
constexpr int kConsumerThreads = 32 * kConsumerWarps;
constexpr int kFoldNT = kConsumerThreads + 32;  // + one producer warp
constexpr int kDefaultTV = 256;       // vectors per source per tile (4 KiB)
constexpr int kMaxStages = 8;
constexpr int kMaxSeg = 34;           // (G-1) + (ng-1) boundaries + 2
constexpr uint64_t kWaitLimitNs = 2000000000ull;

struct FoldParams {
  const char *src[kMaxRanks];  // rank order
  char *dst[kMaxRanks];        // kModeScatter: dst[c] offset by -c*C elements
  uint64_t seg_vec0[kMaxSeg + 1];   // first vector of each segment, [nseg] = end
  uint64_t seg_tile0[kMaxSeg + 1];  // first tile of each segment, [nseg] = ntiles
  uint8_t seg_cg[kMaxSeg];
  uint8_t seg_cl[kMaxSeg];
  uint64_t ntiles;
  float scale;
  int nseg, p, G, ng, mode, ndst, stages;
  uint32_t tv;           // vectors per source per tile
  uint32_t tile_bytes;   // tv * 16
  uint32_t stage_bytes;  // p * tile_bytes
};

struct TileInfo {
  uint64_t v0;  // first vector
  uint32_t nv;  // vectors in this tile (>= 1)
  int seg;
};

// The segment table lives in shared memory (kernel parameters reached
// through a pointer are slow, dependent loads).  Each thread's tiles only move
// forward, so a per-thread cursor finds the segment in O(1) amortised.
struct SegTable {
  uint64_t vec0[kMaxSeg + 1];
  uint64_t tile0[kMaxSeg + 1];
  uint8_t cg[kMaxSeg];
  uint8_t cl[kMaxSeg];
};

__device__ __forceinline__ TileInfo tile_info(const SegTable &tb, uint64_t t, int &cursor,
                                              uint32_t tv) {
  while (t >= tb.tile0[cursor + 1]) ++cursor;
  TileInfo ti;
  ti.seg = cursor;
  ti.v0 = tb.vec0[cursor] + (t - tb.tile0[cursor]) * tv;
  const uint64_t left = tb.vec0[cursor + 1] - ti.v0;
  ti.nv = (uint32_t)(left < (uint64_t)tv ? left : (uint64_t)tv);
  return ti;
}

__device__ __forceinline__ int fold_rank(int k, int cg, int cl, int G, int ng) {
  const int t = k / G, j = k - t * G;
  int gg = cl + 1 + t;
  gg = gg >= ng ? gg - ng : gg;
  gg = gg >= ng ? gg - ng : gg;
  int m = cg + 1 + j;
  m = m >= G ? m - G : m;
  return gg * G + m;
}

// GROUPED = false: the flat fold (G = p), a plain left-to-right fold;
// GROUPED = true: the hierarchical fold with group boundaries, at fold
// positions that are multiples of G -- compile-time when GS > 0 (GS == G),
// from run-time bit masks when GS == 0.
template <int PMAX, class TI, class TO, int OP, bool GROUPED, int GS = 0>
__global__ void __launch_bounds__(kFoldNT, 1) rc_fold_tma_kernel(const __grid_constant__ FoldParams a) {
  using Acc = typename TI::Acc;
  constexpr int VEC = kVec<TI>;
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ __align__(8) uint64_t full[kMaxStages];   // tile landed (tx bytes)
  __shared__ __align__(8) uint64_t empty[kMaxStages];  // tile consumed (one arrival per consumer warp)
  __shared__ SegTable tb;
  __shared__ const char *s_src[kMaxSeg][PMAX];         // per segment: sources in fold order
  __shared__ char *s_dst[kMaxRanks];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int p = a.p, S = a.stages;

  // Everything the loops index dynamically goes to shared memory once.
  for (int i = threadIdx.x; i <= a.nseg; i += blockDim.x) {
    tb.vec0[i] = a.seg_vec0[i];
    tb.tile0[i] = a.seg_tile0[i];
    if (i < a.nseg) {
      tb.cg[i] = a.seg_cg[i];
      tb.cl[i] = a.seg_cl[i];
    }
  }
  for (int i = threadIdx.x; i < a.nseg * p; i += blockDim.x) {
    const int sg = i / p, q = i - sg * p;
    s_src[sg][q] = a.src[fold_rank(q, a.seg_cg[sg], a.seg_cl[sg], a.G, a.ng)];
  }
  if (threadIdx.x < kMaxRanks) s_dst[threadIdx.x] = a.dst[threadIdx.x];
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumerWarps);
    }
    mbar_init_fence();
  }
  __syncthreads();
  pdl_wait();

  const uint64_t Gd = gridDim.x;
  const int64_t K = a.ntiles > blockIdx.x ? (int64_t)((a.ntiles - blockIdx.x + Gd - 1) / Gd) : 0;
  const uint32_t tv = a.tv, tile_bytes = a.tile_bytes, stage_bytes = a.stage_bytes;
  int cursor = 0;

  if (warp == kConsumerWarps) {
    // ---------------- producer warp: one lane streams the tiles in
    if (lane != 0) return;
    int s = 0;
    uint32_t use = 0;  // how many times stage s was filled before (its phase count)
    int64_t k = 0;
    for (; k < K; ++k) {
      if (use > 0 && !mbar_wait_bounded(&empty[s], (use - 1) & 1, kWaitLimitNs)) {
        atomicAdd(&g_wait_timeouts_fold, 1u);
        break;
      }
      const TileInfo ti = tile_info(tb, blockIdx.x + (uint64_t)k * Gd, cursor, tv);
      unsigned char *st = smem + (size_t)s * stage_bytes;
      const uint32_t bytes = ti.nv * 16u;
      mbar_arrive_expect_tx(&full[s], bytes * (uint32_t)p);
      const char *const *src = s_src[ti.seg];
      for (int q = 0; q < p; ++q)
        bulk_load(st + (size_t)q * tile_bytes, src[q] + ti.v0 * 16, bytes, &full[s]);
      if (++s == S) {
        s = 0;
        ++use;
      }
    }
    // every copy this thread issued has landed before it leaves (bounded)
    for (int64_t j = (k > S ? k - S : 0); j < k; ++j)
      if (!mbar_wait_bounded(&full[j % S], (uint32_t)((j / S) & 1), kWaitLimitNs)) break;
    return;
  }

  // ---------------- consumer warps: fold from shared memory, store
  uint32_t first = 0, lastm = 0;  // group boundaries along the fold positions
  const int G = a.G;
#pragma unroll
  for (int q = 0; q < PMAX; ++q) {
    if (q < p) {
      const int j = q % G;
      if (j == 0) first |= 1u << q;
      if (j == G - 1) lastm |= 1u << q;
    }
  }
  char *dall[PMAX];
#pragma unroll
  for (int r = 0; r < PMAX; ++r) dall[r] = (r < a.ndst) ? a.dst[r] : nullptr;
  const int mode = a.mode, ndst = a.ndst;
  const float scale = a.scale;
  const int ctid = threadIdx.x;  // 0 .. kConsumerThreads-1
  int s = 0;
  uint32_t phase = 0;
  for (int64_t k = 0; k < K; ++k) {
    if (!mbar_wait_bounded(&full[s], phase, kWaitLimitNs)) {
      if (lane == 0) atomicAdd(&g_wait_timeouts_fold, 1u);
      break;
    }
    const TileInfo ti = tile_info(tb, blockIdx.x + (uint64_t)k * Gd, cursor, tv);
    const uint32_t st = smem_addr(smem) + (uint32_t)s * stage_bytes;  // shared address
    char *d1 = (mode == kModeScatter) ? s_dst[tb.cg[ti.seg]] : dall[0];
    for (uint32_t v = ctid; v < ti.nv; v += kConsumerThreads) {
      Acc Sg[VEC], T[VEC];
      const uint32_t col = st + v * 16u;
      if constexpr (!GROUPED) {
        unpack<TI>(lds128(col), T);
#pragma unroll
        for (int q = 1; q < PMAX; ++q) {
          if (q < p) {
            Acc x[VEC];
            unpack<TI>(lds128(col + (uint32_t)q * tile_bytes), x);
#pragma unroll
            for (int e = 0; e < VEC; ++e) T[e] = combine<OP>(T[e], x[e]);
          }
        }
      } else {
#pragma unroll
        for (int q = 0; q < PMAX; ++q) {
          if (q < p) {
            Acc x[VEC];
            unpack<TI>(lds128(col + (uint32_t)q * tile_bytes), x);
            const bool is_first = GS > 0 ? (q % (GS > 0 ? GS : 1) == 0) : (((first >> q) & 1u) != 0);
            if (is_first) {
#pragma unroll
              for (int e = 0; e < VEC; ++e) Sg[e] = x[e];
            } else {
#pragma unroll
              for (int e = 0; e < VEC; ++e) Sg[e] = combine<OP>(Sg[e], x[e]);
            }
            const bool is_last = GS > 0 ? (q % (GS > 0 ? GS : 1) == (GS > 0 ? GS : 1) - 1)
                                        : (((lastm >> q) & 1u) != 0);
            if (is_last) {
              if (GS > 0 ? q < GS : q < G) {
#pragma unroll
                for (int e = 0; e < VEC; ++e) T[e] = Sg[e];
              } else {
#pragma unroll
                for (int e = 0; e < VEC; ++e) T[e] = combine<OP>(T[e], Sg[e]);
              }
            }
          }
        }
      }
#pragma unroll
      for (int e = 0; e < VEC; ++e) T[e] = finish<OP>(T[e], scale);
      const uint64_t off = (ti.v0 + v) * (uint64_t)(VEC * TO::kBytes);
      if (mode == kModeAll) {
#pragma unroll
        for (int r = 0; r < PMAX; ++r)
          if (r < ndst) store_vec<TO, VEC>(dall[r] + off, T);
      } else {
        store_vec<TO, VEC>(d1 + off, T);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);  // this warp is done with stage s
    if (++s == S) {
      s = 0;
      phase ^= 1u;
    }
  }
}

template <int PMAX, class TI, class TO, int OP>
cudaError_t run_fold(const FoldJob &job, cudaStream_t s) {
  FoldParams a{};
  const int p = job.p;
  a.p = p;
  a.G = job.G;
  a.ng = p / job.G;
  a.mode = job.mode;
  a.ndst = job.ndst;
  a.scale = job.scale;
  for (int r = 0; r < p; ++r) a.src[r] = static_cast<const char *>(job.src[r]);
  for (int r = 0; r < kMaxP; ++r) a.dst[r] = static_cast<char *>(job.dst[r]);
  constexpr int VEC = kVec<TI>;
  uint32_t tv = (uint32_t)env_int("RC_FOLD_TV", kDefaultTV);
  if (tv < 32 || tv > 2048 || (tv & (tv - 1))) tv = kDefaultTV;
  // segments on vectors [0, nvec)
  const uint64_t nvec = job.n / VEC;
  std::vector<uint64_t> b;  // boundaries in vectors
  b.push_back(0);
  for (int c = 1; c < a.G; ++c) b.push_back(c * job.CG / VEC);
  for (int c = 1; c < a.ng; ++c) b.push_back(c * job.CL / VEC);
  std::sort(b.begin(), b.end());
  b.erase(std::unique(b.begin(), b.end()), b.end());
  int ns = 0;
  uint64_t tiles = 0;
  for (size_t i = 0; i < b.size(); ++i) {
    const uint64_t lo = b[i], hi = std::min<uint64_t>(i + 1 < b.size() ? b[i + 1] : nvec, nvec);
    if (lo >= hi) continue;
    if (ns >= kMaxSeg) return cudaErrorInvalidValue;
    a.seg_vec0[ns] = lo;
    a.seg_tile0[ns] = tiles;
    a.seg_cg[ns] = (uint8_t)(lo * VEC / job.CG);
    a.seg_cl[ns] = (uint8_t)(lo * VEC / job.CL);
    tiles += (hi - lo + tv - 1) / tv;
    ++ns;
  }
  a.nseg = ns;
  a.seg_vec0[ns] = nvec;
  a.seg_tile0[ns] = tiles;
  a.ntiles = tiles;
  if (tiles == 0) return cudaSuccess;
  if (job.mode == kModeScatter) {
    for (int c = 0; c < p; ++c)
      a.dst[c] = reinterpret_cast<char *>(reinterpret_cast<uintptr_t>(job.dst[c]) -
                                          (uintptr_t)(c * job.CG * TO::kBytes));
  }

  a.tv = tv;
  a.tile_bytes = tv * 16;
  a.stage_bytes = (uint32_t)p * a.tile_bytes;
  // default: 4 stages of 4 KiB per source (one CTA per SM at p = 8); measured
  // best of tile sizes 1-8 KiB x 1-8 stages x 1-3 CTAs per SM for p = 8
  int stages = (int)std::min<uint64_t>(4, (192u * 1024u) / a.stage_bytes);
  stages = std::max(2, std::min(stages, env_int("RC_FOLD_STAGES", stages)));
  if ((uint64_t)stages * a.stage_bytes > 200u * 1024u) stages = (int)((200u * 1024u) / a.stage_bytes);
  if (stages < 1) return cudaErrorInvalidValue;
  a.stages = stages;
  const size_t smem = (size_t)stages * a.stage_bytes;

  // flat, grouped with groups of 4 (compile-time boundaries), other groups
  const int variant = job.G == job.p ? 0 : (job.G == 4 && PMAX >= 8 ? 1 : 2);
  auto kern = variant == 0 ? rc_fold_tma_kernel<PMAX, TI, TO, OP, false>
            : variant == 1 ? rc_fold_tma_kernel<PMAX, TI, TO, OP, true, 4>
                           : rc_fold_tma_kernel<PMAX, TI, TO, OP, true, 0>;
  static std::atomic<uint64_t> attr_set[3];  // [variant], one bit per device
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  std::atomic<uint64_t> &flag = attr_set[variant];
  if (!(flag.load() & (1ull << (dev & 63)))) {
    err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
    if (err != cudaSuccess) return err;
    flag.fetch_or(1ull << (dev & 63));
  }
  int occ = 0;
  err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, kFoldNT, smem);
  if (err != cudaSuccess) return err;
  occ = std::max(1, std::min(occ, env_int("RC_FOLD_CTAS", occ)));
  const uint64_t grid = std::max<uint64_t>(1, std::min<uint64_t>((uint64_t)device_sm_count() * occ, tiles));
  return launch_kernel(kern, dim3((unsigned)grid), dim3(kFoldNT), smem, s, a);
}

template <class TI, class TO, int OP>
cudaError_t fold_by_p(const FoldJob &job, cudaStream_t s) {
  const int w = std::max(job.p, job.ndst);
  if (w <= 2) return run_fold<2, TI, TO, OP>(job, s);
  if (w <= 4) return run_fold<4, TI, TO, OP>(job, s);
  if (w <= 8) return run_fold<8, TI, TO, OP>(job, s);
  return run_fold<16, TI, TO, OP>(job, s);
}

template <class TI, class TO>
cudaError_t fold_by_op(const FoldJob &job, cudaStream_t s) {
  switch (job.op) {
    case kSum: return fold_by_p<TI, TO, kSum>(job, s);
    case kMax: return fold_by_p<TI, TO, kMax>(job, s);
    case kMin: return fold_by_p<TI, TO, kMin>(job, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

bool fold_tma_eligible(const FoldJob &job) {
  if (env_int("RC_NO_TMA_FOLD", 0)) return false;
  const int vec = 16 / (job.in_dt == kBF16 ? 2 : 4);
  if (job.CG % vec || job.CL % vec) return false;
  if (job.G != job.p && job.n % vec) return false;  // the scalar tail handles flat order only
  for (int r = 0; r < job.p; ++r)
    if (reinterpret_cast<uintptr_t>(job.src[r]) % 16) return false;
  const int nd = job.mode == kModeAll ? job.ndst : (job.mode == kModeOne ? 1 : job.p);
  for (int r = 0; r < nd; ++r)
    if (reinterpret_cast<uintptr_t>(job.dst[r]) % 16) return false;
  return job.n / vec > 0;
}

cudaError_t launch_fold_tma(const FoldJob &job, cudaStream_t s) {
  const int i = job.in_dt, o = job.out_dt;
  if (i == kF32 && o == kF32) return fold_by_op<F32, F32>(job, s);
  if (i == kBF16 && o == kBF16) return fold_by_op<BF16, BF16>(job, s);
  if (i == kI32 && o == kI32) return fold_by_op<I32, I32>(job, s);
  if (i == kF32 && o == kBF16) return fold_by_op<F32, BF16>(job, s);
  if (i == kBF16 && o == kF32) return fold_by_op<BF16, F32>(job, s);
  return cudaErrorInvalidValue;
}

cudaError_t read_and_clear_fold_timeouts(unsigned int *count) {
  unsigned int zero = 0;
  cudaError_t err = cudaMemcpyFromSymbol(count, g_wait_timeouts_fold, sizeof(unsigned int));
  if (err != cudaSuccess) return err;
  if (*count) err = cudaMemcpyToSymbol(g_wait_timeouts_fold, &zero, sizeof(unsigned int));
  return err;
}

}  // namespace rc
