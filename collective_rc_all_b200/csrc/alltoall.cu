// alltoall.cu -- all-to-all over p simulated ranks, with equal or per-pair
// split counts (MoE dispatch and combine).
//
// Page: "分布式训练/推理", primitive table (all-to-all: every rank sends a
// different slice to every rank; used to route MoE tokens to the rank of
// their expert), section "从路由结果到专家输出" (dispatch is the exchange
// towards the experts, combine the way back; split counts tell a receiver
// how much arrives) and section "为什么 top-k 和 EP degree 会直接放大通信" (a rank's
// payload per phase is t*k*h*b, of which t*k*h*b*(p-1)/p leaves the rank
// under balanced routing).
//
// counts[r][q] elements go from rank r to rank q.  Rank r's send buffer holds
// its outgoing blocks in destination order, rank q's receive buffer its
// incoming blocks in source order, so block (r, q) is one contiguous copy
//   send[r] + sum_{q'<q} counts[r][q']  ->  recv[q] + sum_{r'<r} counts[r'][q].
// The kernel copies the non-empty blocks as segments: one 256-thread CTA per
// 16 KiB tile of one segment (4 loads of 16 bytes in flight per thread), the
// CTAs sweeping the segments as a front like the copy roofline kernel.  A
// segment whose addresses or length are not 16-byte multiples is copied
// element by element by the CTAs of its tiles.
#include <algorithm>
#include <vector>

#include "common.cuh"
#include "internal.h"
#include "launch.cuh"

namespace rc {
namespace {

constexpr int kNT = 256;
constexpr int kILP = 4;
constexpr uint64_t kTile = (uint64_t)kNT * kILP * 16;  // 16 KiB
constexpr int kMaxSegs = kMaxRanks * kMaxRanks;

struct A2aParams {
  const char *src[kMaxSegs];
  char *dst[kMaxSegs];
  uint64_t bytes[kMaxSegs];
  uint64_t tile0[kMaxSegs + 1];  // first tile of each segment; [nseg] = total tiles
  uint32_t vec_mask[kMaxSegs / 32];  // bit s: segment s is copied in 16-byte vectors
  int nseg;
  int esz;
};

__global__ void __launch_bounds__(kNT) rc_a2a_kernel(const __grid_constant__ A2aParams a) {
  pdl_wait();
  const uint64_t t = blockIdx.x;
  // the segment holding tile t: the last s with tile0[s] <= t
  int lo = 0, hi = a.nseg - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (a.tile0[mid] <= t) lo = mid;
    else hi = mid - 1;
  }
  const int s = lo;
  const uint64_t off = (t - a.tile0[s]) * kTile;
  const uint64_t len = a.bytes[s] - off < kTile ? a.bytes[s] - off : kTile;
  const char *src = a.src[s] + off;
  char *dst = a.dst[s] + off;
  if ((a.vec_mask[s >> 5] >> (s & 31)) & 1u) {
    const uint64_t nv = len / 16;
    uint4 v[kILP];
#pragma unroll
    for (int j = 0; j < kILP; ++j) {
      const uint64_t u = (uint64_t)j * kNT + threadIdx.x;
      if (u < nv) v[j] = ld_stream_v4(src + u * 16);
    }
#pragma unroll
    for (int j = 0; j < kILP; ++j) {
      const uint64_t u = (uint64_t)j * kNT + threadIdx.x;
      if (u < nv) st_v4(dst + u * 16, v[j]);
    }
  } else if (a.esz == 4) {
    for (uint64_t i = threadIdx.x; i < len / 4; i += kNT)
      reinterpret_cast<uint32_t *>(dst)[i] = reinterpret_cast<const uint32_t *>(src)[i];
  } else {  // 2-byte elements
    for (uint64_t i = threadIdx.x; i < len / 2; i += kNT)
      reinterpret_cast<uint16_t *>(dst)[i] = reinterpret_cast<const uint16_t *>(src)[i];
  }
}

}  // namespace

cudaError_t launch_all_to_all(const A2aJob &job, cudaStream_t s) {
  const int p = job.p;
  if (p < 1 || p > kMaxRanks || (job.esz != 2 && job.esz != 4)) return cudaErrorInvalidValue;
  A2aParams a{};
  a.esz = job.esz;
  int ns = 0;
  uint64_t tiles = 0;
  for (int r = 0; r < p; ++r) {
    uint64_t soff = 0;
    for (int q = 0; q < p; ++q) {
      const uint64_t c = job.counts[r * p + q];
      uint64_t roff = 0;
      for (int k = 0; k < r; ++k) roff += job.counts[k * p + q];
      if (c > 0) {
        const char *src = static_cast<const char *>(job.send[r]) + soff * job.esz;
        char *dst = static_cast<char *>(job.recv[q]) + roff * job.esz;
        const uint64_t bytes = c * job.esz;
        a.src[ns] = src;
        a.dst[ns] = dst;
        a.bytes[ns] = bytes;
        a.tile0[ns] = tiles;
        if (reinterpret_cast<uintptr_t>(src) % 16 == 0 && reinterpret_cast<uintptr_t>(dst) % 16 == 0 &&
            bytes % 16 == 0)
          a.vec_mask[ns >> 5] |= 1u << (ns & 31);
        tiles += (bytes + kTile - 1) / kTile;
        ++ns;
      }
      soff += c;
    }
  }
  a.nseg = ns;
  a.tile0[ns] = tiles;
  if (ns == 0) return cudaSuccess;
  if (tiles > 0x7fffffffull) return cudaErrorInvalidValue;
  return launch_kernel(rc_a2a_kernel, dim3((unsigned)tiles), dim3(kNT), 0, s, a);
}

}  // namespace rc
