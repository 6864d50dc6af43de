// copy.cu -- the copy roofline: dst = src with 16-byte loads and stores.
//
// This is the denominator every collective is measured against: the same
// HBM read+write traffic pattern with no arithmetic.  4 loads of 16 bytes in
// flight per thread, read-only streaming loads.
#include <algorithm>

#include "common.cuh"
#include "internal.h"
#include "launch.cuh"

namespace rc {
namespace {

constexpr int kNT = 256;
constexpr int kILP = 4;
constexpr uint64_t kBlockVecs = (uint64_t)kNT * kILP;  // 16 KiB per block

// One block per 16 KiB: the blocks sweep memory as a front, which keeps DRAM
// row locality (a persistent grid with a private contiguous range per CTA
// measured 4.6-5.5 TB/s on 1 GiB; this schedule 6.9 TB/s).
__global__ void __launch_bounds__(kNT) rc_copy_kernel(const char *__restrict__ src,
                                                      char *__restrict__ dst, uint64_t nvec) {
  pdl_wait();
  const uint64_t base = (uint64_t)blockIdx.x * kBlockVecs;
  uint4 v[kILP];
#pragma unroll
  for (int j = 0; j < kILP; ++j) {
    const uint64_t u = base + (uint64_t)j * kNT + threadIdx.x;
    if (u < nvec) v[j] = ld_stream_v4(src + u * 16);
  }
#pragma unroll
  for (int j = 0; j < kILP; ++j) {
    const uint64_t u = base + (uint64_t)j * kNT + threadIdx.x;
    if (u < nvec) st_v4(dst + u * 16, v[j]);
  }
}

__global__ void rc_copy_bytes_kernel(const unsigned char *src, unsigned char *dst, uint64_t n) {
  pdl_wait();
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
      const uint64_t grid = (nvec + kBlockVecs - 1) / kBlockVecs;
      if (grid > 0x7fffffffull) return cudaErrorInvalidValue;
      cudaError_t err = launch_kernel(rc_copy_kernel, dim3((unsigned)grid), dim3(kNT), 0, s, sp, dp, nvec);
      if (err != cudaSuccess) return err;
    }
    head = nvec * 16;
  }
  if (head < bytes) {
    const uint64_t rest = bytes - head;
    const unsigned grid = (unsigned)std::max<uint64_t>(1, std::min<uint64_t>((rest + 255) / 256, (uint64_t)sms * 8));
    return launch_kernel(rc_copy_bytes_kernel, dim3(grid), dim3(256), 0, s,
                         reinterpret_cast<const unsigned char *>(sp + head),
                         reinterpret_cast<unsigned char *>(dp + head), rest);
  }
  return cudaSuccess;
}

}  // namespace rc
