// fanout.cu -- all-gather and broadcast as a fan-out: a register kernel
// (default) and a bulk-copy kernel.
//
// Pages: "分布式训练/推理", section "通信原语：rank、world size 和 collective
// operations" (broadcast copies one rank's tensor to every rank; all-gather
// hands every rank the concatenation of all shards) and section
// "FSDP 的执行顺序" (parameter shards all-gathered before the module runs).
//
// Register kernel: every thread loads its 16-byte vectors of one source once
// and stores them to each destination (one block per 8 KiB of a source, the
// blocks sweeping the sources as a front).
//
// Bulk-copy kernel: each source tile is read from HBM ONCE into the CTA's own shared memory by
// a bulk copy (TMA engine, completion on an mbarrier) and written out p times
// by bulk stores -- minimum traffic n*s read + p*n*s written.  One elected
// thread per CTA drives a STAGES-deep ring of shared-memory tiles: loads run
// LOOKAHEAD tiles ahead of the stores, and a stage is refilled only after the
// stores that read it have finished reading (bulk wait_group.read).  Plain
// (non-multicast) copies only: every load targets this CTA's own shared
// memory from this GPU's own memory.
//
// Every wait is bounded (2 s on the global timer).  On expiry the kernel
// counts the event in a device word, drains its own copies (again bounded)
// and returns; rc_stream_status() reports RC_ERR_TIMEOUT.
#include <algorithm>
#include <atomic>
#include <type_traits>

#include "bulk.cuh"
#include "common.cuh"
#include "internal.h"
#include "launch.cuh"

namespace rc {

// Number of bounded waits that gave up since the host last looked.
__device__ unsigned int g_wait_timeouts = 0;

namespace {

constexpr uint32_t kMaxTile = 32 * 1024;  // bytes per stage, at most
constexpr uint32_t kMinTile = 4 * 1024;
constexpr int kStages = 6;
constexpr int kLookahead = 4;             // loads in flight ahead of the stores
constexpr uint64_t kWaitLimitNs = 2000000000ull;
static_assert(kLookahead <= kStages - 1, "a stage must be free when its load is issued");

struct FanoutParams {
  const char *src[kMaxRanks];
  char *dst[kMaxRanks];
  uint32_t skip[kMaxRanks];  // bit r of skip[q]: do not write source r to rank q
  uint64_t src_bytes;
  uint64_t tiles_per_src;
  uint64_t units;            // nsrc * tiles_per_src
  uint32_t tile;             // bytes per unit (a power of two in [4 KiB, 32 KiB])
  int p;
};

__global__ void __launch_bounds__(32) rc_fanout_bulk_kernel(const __grid_constant__ FanoutParams a) {
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ __align__(8) uint64_t bars[kStages];
  if (threadIdx.x != 0) return;

  for (int s = 0; s < kStages; ++s) mbar_init(&bars[s], 1);
  mbar_init_fence();
  pdl_wait();

  const uint64_t G = gridDim.x;
  const uint64_t u0 = a.units * blockIdx.x / G;
  const uint64_t u1 = a.units * (blockIdx.x + 1) / G;
  const int64_t K = (int64_t)(u1 - u0);

  const uint32_t tile = a.tile;
  auto unit_bytes = [&](uint64_t u, uint64_t &src_idx, uint64_t &off) -> uint32_t {
    src_idx = u / a.tiles_per_src;
    off = (u - src_idx * a.tiles_per_src) * tile;
    const uint64_t rem = a.src_bytes - off;
    return (uint32_t)(rem < tile ? rem : tile);
  };

  const uint64_t pol = l2_policy_evict_first();
  bool failed = false;
  int64_t loads_issued = 0, loads_seen = 0;
  for (int64_t k = 0; k < K + kLookahead && !failed; ++k) {
    if (k < K) {  // refill stage k % S with unit u0 + k
      const int s = (int)(k % kStages);
      if (k >= kStages) bulk_wait_read<kStages - kLookahead - 1>();
      uint64_t r, off;
      const uint32_t bytes = unit_bytes(u0 + k, r, off);
      mbar_arrive_expect_tx(&bars[s], bytes);
      bulk_load(smem + (size_t)s * tile, a.src[r] + off, bytes, &bars[s]);
      ++loads_issued;
    }
    const int64_t j = k - kLookahead;
    if (j >= 0 && j < K) {  // write unit u0 + j to every destination
      const int s = (int)(j % kStages);
      if (!mbar_wait_bounded(&bars[s], (uint32_t)((j / kStages) & 1), kWaitLimitNs)) {
        failed = true;
        break;
      }
      ++loads_seen;
      fence_proxy_async_smem();
      uint64_t r, off;
      const uint32_t bytes = unit_bytes(u0 + j, r, off);
      const unsigned char *buf = smem + (size_t)s * tile;
      for (int q = 0; q < a.p; ++q) {
        if ((a.skip[q] >> r) & 1u) continue;
        bulk_store_hint(a.dst[q] + r * a.src_bytes + off, buf, bytes, pol);
      }
      bulk_commit();
    }
  }
  if (failed) {
    atomicAdd(&g_wait_timeouts, 1u);
    // drain loads still in flight into this CTA's shared memory (bounded)
    for (int64_t j = loads_seen; j < loads_issued; ++j) {
      const int s = (int)(j % kStages);
      if (!mbar_wait_bounded(&bars[s], (uint32_t)((j / kStages) & 1), kWaitLimitNs)) break;
    }
  }
  bulk_wait_all();
}

// Register fan-out (aligned buffers): one 256-thread block per tile of
// 256*kRegILP 16-byte vectors of one source; every thread loads its vectors
// once and stores them to each destination rank.  Blocks sweep the sources as
// a front.
constexpr int kRegNT = 256;

template <int kRegILP>
__global__ void __launch_bounds__(kRegNT) rc_fanout_reg_kernel(const __grid_constant__ FanoutParams a,
                                                               uint64_t tiles_per_src) {
  pdl_wait();
  const uint64_t r = blockIdx.x / tiles_per_src;
  const uint64_t v0 = (blockIdx.x - r * tiles_per_src) * (uint64_t)(kRegNT * kRegILP);
  const uint64_t nv = a.src_bytes / 16;
  const char *src = a.src[r];
  uint4 v[kRegILP];
#pragma unroll
  for (int j = 0; j < kRegILP; ++j) {
    const uint64_t u = v0 + (uint64_t)j * kRegNT + threadIdx.x;
    if (u < nv) v[j] = ld_stream_v4(src + u * 16);
  }
  const uint64_t base = r * a.src_bytes;
  for (int q = 0; q < a.p; ++q) {
    if ((a.skip[q] >> r) & 1u) continue;
    char *dst = a.dst[q] + base;
#pragma unroll
    for (int j = 0; j < kRegILP; ++j) {
      const uint64_t u = v0 + (uint64_t)j * kRegNT + threadIdx.x;
      if (u < nv) st_v4_cs(dst + u * 16, v[j]);
    }
  }
}

// Fallback for buffers that are not 16-byte aligned (or sizes not a multiple
// of 16 bytes): element copies, blockIdx.y = destination rank, x grid-stride.
template <typename E>
__global__ void rc_fanout_elem_kernel(const __grid_constant__ FanoutParams a, int nsrc) {
  pdl_wait();
  const int q = blockIdx.y;
  const uint64_t per_src = a.src_bytes / sizeof(E);
  const uint64_t total = per_src * nsrc;
  E *out = reinterpret_cast<E *>(a.dst[q]);
  for (uint64_t i = blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; i < total;
       i += (uint64_t)gridDim.x * blockDim.x) {
    const uint64_t r = i / per_src;
    if ((a.skip[q] >> r) & 1u) continue;
    out[i] = reinterpret_cast<const E *>(a.src[r])[i - r * per_src];
  }
}

// Exercises the bounded-wait path: waits on a barrier phase that nothing will
// complete, gives up after limit_ns and records the timeout like any other
// wait of this library.  No copy is in flight, so returning is safe.
__global__ void rc_wait_probe_kernel(uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x != 0) return;
  mbar_init(&bar, 1);
  mbar_init_fence();
  if (!mbar_wait_bounded(&bar, 0, limit_ns)) atomicAdd(&g_wait_timeouts, 1u);
}

}  // namespace

cudaError_t launch_wait_probe(uint64_t limit_ns, cudaStream_t s) {
  rc_wait_probe_kernel<<<1, 32, 0, s>>>(limit_ns);
  note_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_fanout(const FanoutJob &job, cudaStream_t s) {
  FanoutParams a{};
  a.p = job.p;
  a.src_bytes = job.src_bytes;
  bool aligned = (job.src_bytes % 16 == 0);
  for (int r = 0; r < job.nsrc; ++r) {
    a.src[r] = static_cast<const char *>(job.src[r]);
    aligned = aligned && reinterpret_cast<uintptr_t>(job.src[r]) % 16 == 0;
  }
  for (int q = 0; q < job.p; ++q) {
    a.dst[q] = static_cast<char *>(job.dst[q]);
    a.skip[q] = job.skip[q];
    aligned = aligned && reinterpret_cast<uintptr_t>(job.dst[q]) % 16 == 0;
  }
  if (job.src_bytes == 0) return cudaSuccess;
  cudaError_t err;
  const int sms = device_sm_count();
  // default: the register kernel (faster alone: 7.6 vs 8.1 us for an
  // 8 x 512 KiB bf16 all-gather and 12.1 vs 12.4 us for an 8 MiB fp32
  // broadcast replayed back to back, 6.1 vs 5.5 TB/s on 64 MiB sources; and in
  // a sequence of seven different collectives in one graph, 130-133 vs
  // 133-134 us, with dependent launches off).  RC_FANOUT_BULK=1 selects the
  // bulk-copy kernel.
  if (aligned && !env_int("RC_FANOUT_BULK", 0)) {
    const uint64_t nv = job.src_bytes / 16;
    auto go = [&](auto ilp_tag) -> cudaError_t {
      constexpr int ILP = decltype(ilp_tag)::value;
      const uint64_t tps = (nv + kRegNT * ILP - 1) / (kRegNT * ILP);
      const uint64_t grid = tps * (uint64_t)job.nsrc;
      if (grid > 0x7fffffffull) return cudaErrorInvalidValue;
      return launch_kernel(rc_fanout_reg_kernel<ILP>, dim3((unsigned)grid), dim3(kRegNT), 0, s, a, tps);
    };
    // vectors per thread: 2 measured best in the one-graph sequence of seven
    // collectives (131.0 us against 131.5 for 1 and 132.0 for 4); alone, the
    // all-gather prefers 4 (7.9 vs 8.2 us) and the broadcast 2 (12.4 vs 12.6)
    const int ilp = env_int("RC_FANOUT_ILP", 2);
    if (ilp == 1) return go(std::integral_constant<int, 1>());
    if (ilp == 2) return go(std::integral_constant<int, 2>());
    return go(std::integral_constant<int, 4>());
  }
  if (aligned) {
    // tile: the largest power of two <= 32 KiB that still gives every SM about
    // four units, so small fan-outs still pipeline
    const uint64_t total = job.src_bytes * job.nsrc;
    uint32_t tile = kMaxTile;
    while (tile > kMinTile && total / tile < 4ull * sms) tile >>= 1;
    tile = (uint32_t)env_int("RC_FANOUT_TILE", (int)tile);
    if (tile < 16 || tile % 16 || tile > kMaxTile) tile = kMaxTile;
    a.tile = tile;
    a.tiles_per_src = (job.src_bytes + tile - 1) / tile;
    a.units = a.tiles_per_src * job.nsrc;
    const size_t smem = (size_t)kStages * tile;
    static std::atomic<uint64_t> attr_set{0};  // one bit per device
    int dev = 0;
    if ((err = cudaGetDevice(&dev)) != cudaSuccess) return err;
    const uint64_t bit = 1ull << (dev & 63);
    if (!(attr_set.load() & bit)) {
      err = cudaFuncSetAttribute(rc_fanout_bulk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)(kStages * kMaxTile));
      if (err != cudaSuccess) return err;
      attr_set.fetch_or(bit);
    }
    int occ = 0;
    if ((err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, rc_fanout_bulk_kernel, 32, smem)) !=
        cudaSuccess)
      return err;
    occ = std::max(1, std::min(occ, env_int("RC_FANOUT_CTAS_PER_SM", 8)));
    const uint64_t grid = std::max<uint64_t>(1, std::min<uint64_t>((uint64_t)sms * occ, a.units));
    return launch_kernel(rc_fanout_bulk_kernel, dim3((unsigned)grid), dim3(32), smem, s, a);
  } else {
    const uint64_t per_src = job.src_bytes / job.elem_bytes;
    const uint64_t total = per_src * job.nsrc;
    const unsigned gx = (unsigned)std::max<uint64_t>(
        1, std::min<uint64_t>((total + 255) / 256, (uint64_t)sms * 4));
    dim3 grid(gx, job.p);
    if (job.elem_bytes == 2) return launch_kernel(rc_fanout_elem_kernel<uint16_t>, grid, dim3(256), 0, s, a, job.nsrc);
    return launch_kernel(rc_fanout_elem_kernel<uint32_t>, grid, dim3(256), 0, s, a, job.nsrc);
  }
}

cudaError_t read_and_clear_wait_timeouts(unsigned int *count) {
  unsigned int zero = 0;
  cudaError_t err = cudaMemcpyFromSymbol(count, g_wait_timeouts, sizeof(unsigned int));
  if (err != cudaSuccess) return err;
  if (*count) err = cudaMemcpyToSymbol(g_wait_timeouts, &zero, sizeof(unsigned int));
  return err;
}

}  // namespace rc
