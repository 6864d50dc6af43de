// copy.cu -- the copy roofline: dst = src with 16-byte loads and stores.
//
// This is the denominator every collective is measured against: the same
// HBM read+write traffic pattern with no arithmetic.  Balanced contiguous
// partition (CTA b owns vectors [b*NV/G, (b+1)*NV/G)), 4 loads in flight per
// thread, streaming cache hints.
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace rc {
namespace {

constexpr int kNT = 256;
constexpr int kILP = 4;

__global__ void __launch_bounds__(kNT) copy_v4_kernel(const char *__restrict__ src,
                                                      char *__restrict__ dst, uint64_t nvec) {
  const uint64_t G = gridDim.x;
  const uint64_t u0 = nvec * blockIdx.x / G, u1 = nvec * (blockIdx.x + 1) / G;
  for (uint64_t u = u0 + threadIdx.x; u < u1; u += (uint64_t)kNT * kILP) {
    uint4 v[kILP];
#pragma unroll
    for (int j = 0; j < kILP; ++j) {
      const uint64_t uj = u + (uint64_t)j * kNT;
      if (uj < u1) v[j] = ld_stream_v4(src + uj * 16);
    }
#pragma unroll
    for (int j = 0; j < kILP; ++j) {
      const uint64_t uj = u + (uint64_t)j * kNT;
      if (uj < u1) st_v4(dst + uj * 16, v[j]);
    }
  }
}

__global__ void copy_bytes_kernel(const unsigned char *src, unsigned char *dst, uint64_t n) {
  for (uint64_t i = blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; i < n;
       i += (uint64_t)gridDim.x * blockDim.x)
    dst[i] = src[i];
}

}  // namespace

cudaError_t launch_copy(const void *src, void *dst, size_t bytes, cudaStream_t s) {
  if (bytes == 0) return cudaSuccess;
  const int sms = device_sm_count();
  const char *sp = static_cast<const char *>(src);
  char *dp = static_cast<char *>(dst);
  uint64_t head = 0;
  if (reinterpret_cast<uintptr_t>(sp) % 16 == 0 && reinterpret_cast<uintptr_t>(dp) % 16 == 0) {
    const uint64_t nvec = bytes / 16;
    if (nvec) {
      int occ = 0;
      cudaError_t err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, copy_v4_kernel, kNT, 0);
      if (err != cudaSuccess) return err;
      uint64_t grid = std::min<uint64_t>((uint64_t)sms * std::max(occ, 1), (nvec + kNT - 1) / kNT);
      copy_v4_kernel<<<(unsigned)std::max<uint64_t>(grid, 1), kNT, 0, s>>>(sp, dp, nvec);
      note_launches(1);
      if ((err = cudaGetLastError()) != cudaSuccess) return err;
    }
    head = nvec * 16;
  }
  if (head < bytes) {
    const uint64_t rest = bytes - head;
    const unsigned grid = (unsigned)std::max<uint64_t>(1, std::min<uint64_t>((rest + 255) / 256, (uint64_t)sms * 8));
    copy_bytes_kernel<<<grid, 256, 0, s>>>(reinterpret_cast<const unsigned char *>(sp + head),
                                           reinterpret_cast<unsigned char *>(dp + head), rest);
    note_launches(1);
    return cudaGetLastError();
  }
  return cudaSuccess;
}

}  // namespace rc
