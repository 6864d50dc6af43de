// ring.cu -- the literal ring all-reduce, executed step by step.
//
// Page: "LLM Parallelism 基础", section "Ring AllReduce": the data is cut into
// N chunks; in the reduce-scatter phase (N-1 steps) every card sends one
// chunk to the next card on the ring, which accumulates it into its own
// matching chunk, so that card 0 ends up with the finished chunk 0; in the
// all-gather phase (N-1 steps) every card forwards its finished chunk to the
// next card, which overwrites its copy.  2(N-1) steps in all.  The bandwidth
// model is in "分布式训练/推理", section "Ring all-reduce 的带宽账".
//
// Schedule executed here, for p simulated ranks held in one GPU's memory:
//   reduce-scatter step k = 0..p-2, every rank r:
//     c = (r-k-1) mod p, d = r+1 mod p
//     msg = (k == 0) ? x_r[chunk c] : partial_r[chunk c]       (the send)
//     partial_d[chunk c] = msg (+) x_d[chunk c]                (the receive)
//     at k = p-2 the receiver owns chunk c == d: y_d[chunk d] = cast(scale*acc)
//   all-gather step k = 0..p-2, every rank r:
//     c = (r-k) mod p:  y_{r+1}[chunk c] = y_r[chunk c]
// Every send and receive is a real load / store in device memory.  Partials
// are fp32 (int32 for int32): they live in the receiver's own y buffer for
// fp32/int32 and in a workspace [2 parities][p][C] for bf16 (the parity
// double-buffers consecutive steps).
//
// Tile-outer / step-inner: each thread owns fixed offsets o inside the
// chunks and runs all 2(p-1) steps on them.  Step k+1 reads exactly what
// the same thread stored at step k, so program order is the only
// synchronisation -- no grid barrier, no flags, nothing can wait forever.
// Within one step the ranks' reads and writes touch disjoint locations, so a
// thread issues all loads of a step before its stores, and it loads the next
// step's x values (independent of the partials) while the current step folds:
// only the partials' round trip through L2 stays on the dependent chain.  The
// per-(step, rank) chunk addresses come from a table in shared memory.
//
// Three kernels execute this schedule:
//  * rc_ring_link_kernel (default for 16-byte aligned buffers): the ranks are
//    thread groups of one thread block and every message crosses a link
//    buffer in shared memory -- a store by the sender, a block barrier, a
//    load by the receiver.  Device memory sees x once and y once.
//  * rc_ring_chain_kernel: the messages are partials in device memory (the
//    receivers' y, or a workspace for bf16), one thread per chunk chain.
//  * rc_ring_literal_kernel: element-wise form for unaligned buffers.
#include <algorithm>
#include <atomic>
#include <mutex>
#include <type_traits>

#include "common.cuh"
#include "internal.h"
#include "launch.cuh"

namespace rc {
namespace {

constexpr int kRingNT = 128;

struct RingParams {
  const char *x[kMaxRanks];
  char *y[kMaxRanks];
  char *ws;
  uint64_t n, C;
  uint64_t units;  // units (vectors or elements) per chunk
  float scale;
  int p;
};

// Coherent loads at L2 (partials are written and read back in this kernel).
__device__ __forceinline__ uint4 ld_cg_v4(const void *p) {
  uint4 v;
  asm volatile("ld.global.cg.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p)
               : "memory");
  return v;
}
// Default-cached (L1) loads: a thread's load after its own store to the same
// address returns the stored value under either caching mode.
__device__ __forceinline__ uint4 ld_ca_v4(const void *p) {
  uint4 v;
  asm volatile("ld.global.ca.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p)
               : "memory");
  return v;
}
__device__ __forceinline__ uint32_t ld_cg_u32(const void *p) {
  uint32_t v;
  asm volatile("ld.global.cg.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ uint32_t ld_cg_u16(const void *p) {
  unsigned short v;
  asm volatile("ld.global.cg.u16 %0, [%1];" : "=h"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_u32(void *p, uint32_t v) {
  asm volatile("st.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ void st_u16(void *p, uint32_t v) {
  asm volatile("st.global.u16 [%0], %1;" ::"l"(p), "h"((unsigned short)v) : "memory");
}

// input element(s) of type T -> accumulators
template <class T, int VEC>
__device__ __forceinline__ void load_in(const char *p, typename T::Acc (&a)[VEC]) {
  if constexpr (VEC == 1) {
    if constexpr (std::is_same<T, BF16>::value) a[0] = bf16_bits_to_f32(ld_cg_u16(p));
    else if constexpr (std::is_same<T, F32>::value) a[0] = __uint_as_float(ld_cg_u32(p));
    else a[0] = (int32_t)ld_cg_u32(p);
  } else {
    unpack<T>(ld_cg_v4(p), a);
  }
}

// input element(s) of type T in their stored form (16-byte vector or one element)
template <class T, int VEC>
__device__ __forceinline__ typename std::conditional<(VEC > 1), uint4, uint32_t>::type load_raw(
    const char *p) {
  if constexpr (VEC > 1) return ld_cg_v4(p);
  else if constexpr (T::kBytes == 2) return ld_cg_u16(p);
  else return ld_cg_u32(p);
}
template <class T, int VEC>
__device__ __forceinline__ void unpack_raw(const uint4 &raw, typename T::Acc (&a)[VEC]) {
  unpack<T>(raw, a);
}
template <class T, int VEC>
__device__ __forceinline__ void unpack_raw(uint32_t raw, typename T::Acc (&a)[VEC]) {
  if constexpr (std::is_same<T, BF16>::value) a[0] = bf16_bits_to_f32(raw);
  else if constexpr (std::is_same<T, F32>::value) a[0] = __uint_as_float(raw);
  else a[0] = (int32_t)raw;
}

// partial (raw 32-bit accumulators) load / store
template <class Acc, int VEC, bool L1>
__device__ __forceinline__ void load_part(const char *p, Acc (&a)[VEC]) {
  uint32_t w[VEC];
  if constexpr (VEC == 1) {
    w[0] = ld_cg_u32(p);
  } else {
#pragma unroll
    for (int h = 0; h < VEC / 4; ++h) {
      const uint4 v = L1 ? ld_ca_v4(p + 16 * h) : ld_cg_v4(p + 16 * h);
      w[4 * h] = v.x;
      w[4 * h + 1] = v.y;
      w[4 * h + 2] = v.z;
      w[4 * h + 3] = v.w;
    }
  }
#pragma unroll
  for (int j = 0; j < VEC; ++j) {
    if constexpr (std::is_same<Acc, float>::value) a[j] = __uint_as_float(w[j]);
    else a[j] = (int32_t)w[j];
  }
}
__device__ __forceinline__ uint32_t acc_bits(float v) { return __float_as_uint(v); }
__device__ __forceinline__ uint32_t acc_bits(int32_t v) { return (uint32_t)v; }

template <class Acc, int VEC>
__device__ __forceinline__ void store_part(char *p, const Acc (&a)[VEC]) {
  if constexpr (VEC == 1) {
    st_u32(p, acc_bits(a[0]));
  } else {
#pragma unroll
    for (int h = 0; h < VEC / 4; ++h)
      st_v4(p + 16 * h, make_uint4(acc_bits(a[4 * h]), acc_bits(a[4 * h + 1]),
                                   acc_bits(a[4 * h + 2]), acc_bits(a[4 * h + 3])));
  }
}

template <class T, int VEC>
__device__ __forceinline__ void store_out(char *p, const typename T::Acc (&a)[VEC]) {
  if constexpr (VEC == 1) {
    if constexpr (std::is_same<T, BF16>::value) st_u16(p, f32_to_bf16_bits(a[0]));
    else st_u32(p, acc_bits(a[0]));
  } else {
    store_vec<T, VEC>(p, a);
  }
}

__device__ __forceinline__ int mod_p(int v, int p) { return v < 0 ? v + p : v; }

// Chunk addresses of every (step, rank) of the schedule, computed once per
// thread block; a thread adds its own offset inside the chunk.
struct RsEntry {      // reduce-scatter step k, sender r -> receiver d = r+1
  const char *msg;    // k == 0: x_r at chunk c (input stride); else r's partial (4-byte stride)
  const char *own;    // x_d at chunk c (input stride)
  char *dst;          // d's partial (4-byte stride), or y_d at chunk d on the last step
  uint64_t len;       // elements in chunk c
};
struct AgEntry {      // all-gather step k, r -> d = r+1, chunk c = r-k
  const char *src;
  char *dst;
  uint64_t len;
};

// Registers are capped so that at least 4 (PMAX <= 8) or 2 (PMAX = 16) thread
// blocks fit per SM: a typical launch then keeps every offset resident at
// once, instead of running a second full 2(p-1)-step chain for a few blocks.
template <class T, int OP, bool VECTOR, int PMAX, bool L1>
__global__ void __launch_bounds__(kRingNT, (PMAX <= 8 ? 4 : 2))
    rc_ring_literal_kernel(const __grid_constant__ RingParams a) {
  using Acc = typename T::Acc;
  constexpr int VEC = VECTOR ? kVec<T> : 1;
  using Raw = typename std::conditional<VECTOR, uint4, uint32_t>::type;
  constexpr int RG = 4;  // ranks folded together (register budget)
  constexpr bool kWs = std::is_same<T, BF16>::value;  // bf16: fp32 partials in workspace
  constexpr int kIn = T::kBytes;
  __shared__ RsEntry rs[kMaxRanks - 1][PMAX];
  __shared__ AgEntry ag[kMaxRanks - 1][PMAX];
  const int p = a.p;
  const uint64_t C = a.C;

  for (int i = threadIdx.x; i < (p - 1) * p; i += blockDim.x) {
    const int k = i / p, r = i - k * p;
    const int d = (r + 1 < p) ? r + 1 : 0;
    // reduce-scatter entry
    {
      const int c = mod_p(r - k - 1, p);
      const uint64_t b = (uint64_t)c * C;
      RsEntry e;
      e.len = b >= a.n ? 0 : (a.n - b < C ? a.n - b : C);
      e.own = a.x[d] + b * kIn;
      if (k == 0) e.msg = a.x[r] + b * kIn;
      else if (kWs) e.msg = a.ws + ((uint64_t)(((k - 1) & 1) * p + r)) * C * 4;
      else e.msg = a.y[r] + b * 4;
      if (k == p - 2) e.dst = a.y[d] + b * kIn;
      else if (kWs) e.dst = a.ws + ((uint64_t)((k & 1) * p + d)) * C * 4;
      else e.dst = a.y[d] + b * 4;
      rs[k][r] = e;
    }
    // all-gather entry
    {
      const int c = mod_p(r - k, p);
      const uint64_t b = (uint64_t)c * C;
      AgEntry e;
      e.len = b >= a.n ? 0 : (a.n - b < C ? a.n - b : C);
      e.src = a.y[r] + b * kIn;
      e.dst = a.y[d] + b * kIn;
      ag[k][r] = e;
    }
  }
  __syncthreads();
  pdl_wait();

  const uint64_t G = gridDim.x;
  const uint64_t o0 = a.units * blockIdx.x / G;
  const uint64_t o1 = a.units * (blockIdx.x + 1) / G;

  for (uint64_t o = o0 + threadIdx.x; o < o1; o += blockDim.x) {
    const uint64_t oe = o * VEC;                 // element offset inside every chunk
    const uint64_t oin = oe * kIn, o4 = oe * 4;  // byte offsets: input / partial

    // ---- phase 1: reduce-scatter, p-1 steps.  own[] holds the receivers' x_d
    // of the current step in input form, loaded one step ahead.
    Raw own[PMAX], nxt[PMAX];
#pragma unroll
    for (int r = 0; r < PMAX; ++r)
      if (r < p && oe < rs[0][r].len) own[r] = load_raw<T, VEC>(rs[0][r].own + oin);
    for (int k = 0; k + 1 < p; ++k) {
      const bool last = (k + 2 == p);
      if (!last) {  // next step's x_d, in flight while this step folds
#pragma unroll
        for (int r = 0; r < PMAX; ++r)
          if (r < p && oe < rs[k + 1][r].len) nxt[r] = load_raw<T, VEC>(rs[k + 1][r].own + oin);
      }
#pragma unroll
      for (int r0 = 0; r0 < PMAX; r0 += RG) {
        if (r0 >= p) break;
        Acc msg[RG][VEC];
#pragma unroll
        for (int g = 0; g < RG; ++g) {  // the sends of this group of ranks
          const int r = r0 + g;
          if (r < p && oe < rs[k][r].len) {
            if (k == 0) unpack_raw<T, VEC>(load_raw<T, VEC>(rs[0][r].msg + oin), msg[g]);
            else load_part<Acc, VEC, L1>(rs[k][r].msg + o4, msg[g]);
          }
        }
#pragma unroll
        for (int g = 0; g < RG; ++g) {  // the receives
          const int r = r0 + g;
          if (r < p && oe < rs[k][r].len) {
            Acc x[VEC];
            unpack_raw<T, VEC>(own[r], x);
#pragma unroll
            for (int j = 0; j < VEC; ++j) msg[g][j] = combine<OP>(msg[g][j], x[j]);
            if (last) {  // receiver d now owns the finished chunk c (== d)
#pragma unroll
              for (int j = 0; j < VEC; ++j) msg[g][j] = finish<OP>(msg[g][j], a.scale);
              store_out<T, VEC>(rs[k][r].dst + oin, msg[g]);
            } else {
              store_part<Acc, VEC>(rs[k][r].dst + o4, msg[g]);
            }
          }
        }
      }
      if (!last) {
#pragma unroll
        for (int r = 0; r < PMAX; ++r) own[r] = nxt[r];
      }
    }

    // ---- phase 2: all-gather, p-1 steps, the receiver overwrites
    for (int k = 0; k + 1 < p; ++k) {
      uint4 v16[PMAX];
      uint32_t v4[PMAX];
#pragma unroll
      for (int r = 0; r < PMAX; ++r) {
        if (r < p && oe < ag[k][r].len) {
          const char *src = ag[k][r].src + oin;
          if constexpr (VECTOR) v16[r] = L1 ? ld_ca_v4(src) : ld_cg_v4(src);
          else if constexpr (kIn == 2) v4[r] = ld_cg_u16(src);
          else v4[r] = ld_cg_u32(src);
        }
      }
#pragma unroll
      for (int r = 0; r < PMAX; ++r) {
        if (r < p && oe < ag[k][r].len) {
          char *dst = ag[k][r].dst + oin;
          if constexpr (VECTOR) st_v4(dst, v16[r]);
          else if constexpr (kIn == 2) st_u16(dst, v4[r]);
          else st_u32(dst, v4[r]);
        }
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Chain kernel (16-byte aligned buffers, chunks a whole number of vectors).
//
// The schedule above, regrouped: follow one chunk c through the ring.  Its
// partial starts at rank c+1 (step 0 sends x_{c+1}[chunk c] to c+2), gains
// x_d[chunk c] at each receiver d = c+k+2 (reduce-scatter step k), ends at
// rank c after p-1 steps (d = c at step p-2, where it is scaled and cast
// into y_c), and is then forwarded c -> c+1 -> ... -> c-1 by the all-gather
// steps (step k: y_{c+k+1}[chunk c] = y_{c+k}[chunk c]).  Every message of
// the schedule belongs to exactly one such chain, and different chunks'
// chains never touch the same memory: the partial of chunk c at receiver d
// lives in y_d[chunk c] (fp32 / int32), or for bf16 in the workspace slot
// [k & 1][c] (two parities: the send buffer of step k-1 and the receive buffer
// of step k are different memory).  So a thread can own CH chains of one
// vector offset and run their 2(p-1) steps in program order, with no
// synchronisation with the threads that own the other chains; the sends and
// receives are real loads and stores of device memory as above.
//
// Each warp holds 32 consecutive offsets of the same chains, so every access
// is a coalesced 512-byte row; the receivers' x values are loaded PF steps
// ahead of the step that adds them.  The ranks of a step are warp-uniform:
// their base pointers come from the kernel parameters.
constexpr int kChainNT = 128;

struct RingChainParams {
  const char *x[kMaxRanks];
  char *y[kMaxRanks];
  char *ws;
  uint64_t cv;  // vectors per chunk (C / VEC)
  uint64_t nv;  // vectors in the whole per-rank vector (n / VEC)
  float scale;
  int p, ngroups;
};

template <class T, int OP, int CH, int PF>
__global__ void __launch_bounds__(kChainNT) rc_ring_chain_kernel(const __grid_constant__ RingChainParams a) {
  using Acc = typename T::Acc;
  constexpr int VEC = kVec<T>;
  constexpr int kIn = T::kBytes;
  constexpr bool kWs = std::is_same<T, BF16>::value;
  pdl_wait();
  const int p = a.p;
  const uint64_t tile = blockIdx.x / (uint32_t)a.ngroups;
  const int grp = (int)(blockIdx.x - tile * (uint32_t)a.ngroups);
  const uint64_t o = tile * kChainNT + threadIdx.x;  // vector offset inside every chunk
  const uint64_t cv = a.cv, C = cv * VEC;
  const uint64_t oin = o * 16, o4 = o * (uint64_t)(VEC * 4);

  int c[CH];          // this thread's chunks
  bool on[CH];
  uint64_t cin[CH];   // byte offset of chunk c in an input / output buffer
  bool any = false;
#pragma unroll
  for (int i = 0; i < CH; ++i) {
    c[i] = grp * CH + i;
    const uint64_t b = (uint64_t)c[i] * cv;
    const uint64_t len = (c[i] >= p || b >= a.nv) ? 0 : (a.nv - b < cv ? a.nv - b : cv);
    on[i] = o < len;
    any = any || on[i];
    cin[i] = (uint64_t)c[i] * C * kIn;
  }
  if (!any) return;
  auto wrap = [p](int v) { return v >= p ? v - p : v; };  // v < 2p
  // partial of chunk c after step k, as received by d
  auto part_at = [&](int i, int k, int d) -> char * {
    if constexpr (kWs) return a.ws + ((uint64_t)((k & 1) * p + c[i])) * C * 4 + o4;
    else return a.y[d] + cin[i] + o4;
  };

  // ---- reduce-scatter: p-1 steps; own[j][i] holds x of receiver c+k+2+j
  uint4 own[PF][CH];
  Acc acc[CH][VEC];
#pragma unroll
  for (int j = 0; j < PF; ++j) {
#pragma unroll
    for (int i = 0; i < CH; ++i)
      if (on[i] && j < p - 1) own[j][i] = ld_cg_v4(a.x[wrap(wrap(c[i] + 2 + j))] + cin[i] + oin);
  }
#pragma unroll
  for (int i = 0; i < CH; ++i)  // step 0's sends: x_{c+1}[chunk c]
    if (on[i]) unpack<T>(ld_cg_v4(a.x[wrap(c[i] + 1)] + cin[i] + oin), acc[i]);
  for (int k = 0; k + 1 < p; ++k) {
    const bool last = (k + 2 == p);
    if (k > 0) {
#pragma unroll
      for (int i = 0; i < CH; ++i)  // receive: the partial the previous step stored
        if (on[i]) load_part<Acc, VEC, true>(part_at(i, k - 1, wrap(wrap(c[i] + k + 1))), acc[i]);
    }
    uint4 cur[CH];
#pragma unroll
    for (int i = 0; i < CH; ++i) {
      cur[i] = own[0][i];
#pragma unroll
      for (int j = 0; j + 1 < PF; ++j) own[j][i] = own[j + 1][i];
      if (on[i] && k + PF < p - 1)  // x of the receiver PF steps ahead
        own[PF - 1][i] = ld_cg_v4(a.x[wrap(wrap(c[i] + k + PF + 2))] + cin[i] + oin);
    }
#pragma unroll
    for (int i = 0; i < CH; ++i) {
      if (!on[i]) continue;
      Acc x[VEC];
      unpack<T>(cur[i], x);
#pragma unroll
      for (int e = 0; e < VEC; ++e) acc[i][e] = combine<OP>(acc[i][e], x[e]);
      if (last) {  // the receiver is c itself: the finished chunk
#pragma unroll
        for (int e = 0; e < VEC; ++e) acc[i][e] = finish<OP>(acc[i][e], a.scale);
        store_out<T, VEC>(a.y[c[i]] + cin[i] + oin, acc[i]);
      } else {
        store_part<Acc, VEC>(part_at(i, k, wrap(wrap(c[i] + k + 2))), acc[i]);
      }
    }
  }

  // ---- all-gather: p-1 steps, y_{c+k+1}[chunk c] = y_{c+k}[chunk c]
  for (int k = 0; k + 1 < p; ++k) {
    uint4 v[CH];
#pragma unroll
    for (int i = 0; i < CH; ++i)
      if (on[i]) v[i] = ld_ca_v4(a.y[wrap(c[i] + k)] + cin[i] + oin);
#pragma unroll
    for (int i = 0; i < CH; ++i)
      if (on[i]) st_v4(a.y[wrap(wrap(c[i] + k + 1))] + cin[i] + oin, v[i]);
  }
}

template <class T, int OP, int CH, int PF>
cudaError_t launch_ring_chain(const RingJob &job, uint64_t C, cudaStream_t s) {
  RingChainParams a{};
  const int p = job.p;
  if (p < 2) return cudaErrorInvalidValue;  // no steps; the API never sends p = 1 here
  constexpr int VEC = kVec<T>;
  a.p = p;
  a.cv = C / VEC;
  a.nv = job.n / VEC;
  a.scale = job.scale;
  a.ws = static_cast<char *>(job.ws);
  a.ngroups = (p + CH - 1) / CH;
  for (int r = 0; r < p; ++r) {
    a.x[r] = static_cast<const char *>(job.x[r]);
    a.y[r] = static_cast<char *>(job.y[r]);
  }
  const uint64_t tiles = (a.cv + kChainNT - 1) / kChainNT;
  const uint64_t grid = tiles * (uint64_t)a.ngroups;
  if (grid == 0) return cudaSuccess;
  if (grid > 0x7fffffffull) return cudaErrorInvalidValue;
  return launch_kernel(rc_ring_chain_kernel<T, OP, CH, PF>, dim3((unsigned)grid), dim3(kChainNT), 0, s, a);
}

// ---------------------------------------------------------------------------
// Link kernel (16-byte aligned buffers, chunks a whole number of vectors).
//
// One thread block owns one tile of L vector offsets [t*L, t*L + L) inside
// every chunk, and holds all p ranks of the ring for that tile: thread group
// r (threads r*L .. r*L + L-1) is rank r, and its thread l works on offset
// o = t*L + l of rank r's chunks.  The ring's links are buffers in shared
// memory: at each of the 2(p-1) steps every rank stores its message into its
// outgoing link, the block synchronises, and every rank loads the message of
// its predecessor from that link.  So each step is still a real send (a
// store) and a real receive (a load) between different threads, in the
// schedule's order, while device memory sees only the inputs, read once
// (rank r reads x_r[chunk c][o] for every c), and the outputs, written once
// (y_r[chunk c][o] when rank r receives finished chunk c).
//
// Rank r meets its own chunks in the order c_j = (r-1-j) mod p: j = 0 is the
// chunk it sends at reduce-scatter step 0 (its own input as the message),
// j = k+1 the chunk it receives at step k, whose partial it folds with its
// own x (acc = msg (+) x_r, the ring order).  At step p-2 the received chunk
// is c = r: finished, scaled and cast once, stored to y_r[chunk r].  The
// all-gather steps then forward the finished vectors in their stored form:
// at step k rank r sends chunk (r-k) mod p and receives chunk (r-1-k) mod p,
// which it stores to y_r.  Partials stay in the accumulator type (fp32 for
// fp32 and bf16, int32 for int32).  The links alternate between two buffers
// by step parity: a link written at step s is read at step s after the
// barrier and rewritten at step s+2, after the barrier of step s+1, by which
// time every reader of step s is done.  One barrier per step.
//
// All of rank r's inputs are requested at the start, in the order of use.
// By default (XS) they are asynchronous 16-byte copies into the thread's own
// slots of shared memory (cp.async, one commit group per slot), so no
// register is tied up while they are in flight and more thread blocks fit on
// an SM; the thread waits for slot j only when a step needs it.  Measured on
// 8 ranks x 8 MiB fp32, back to back: 23.9 us against 25.2 us with the
// inputs held in registers (RC_RING_XSMEM=0), and 13.9 against 15.9 us in
// bf16.  Either way every input is read before the thread's first store (the
// first store follows the wait for the last slot), so an in-place call
// (y_r == x_r) is safe, and no other thread touches x_r[.][o] or y_r[.][o].
//
// At p > 8 only a window of 4 slots per thread is staged (slot j + 4 is
// requested into slot j's buffer once slot j is consumed), so that blocks of
// 16 ranks still fit several to an SM.
//
// Lanes per rank: 16 for p > 4 (128-thread blocks at p = 8), 32 for p <= 4:
// measured at p = 8, 16 lanes gave 25.2 us against 25.6 for 32 and 27.3 for
// 64 (inputs in registers).
template <class Acc>
__device__ __forceinline__ uint4 acc4_bits(const Acc *a) {
  return make_uint4(acc_bits(a[0]), acc_bits(a[1]), acc_bits(a[2]), acc_bits(a[3]));
}
template <class Acc>
__device__ __forceinline__ void bits_acc4(const uint4 &v, Acc *a) {
  if constexpr (std::is_same<Acc, float>::value) {
    a[0] = __uint_as_float(v.x); a[1] = __uint_as_float(v.y);
    a[2] = __uint_as_float(v.z); a[3] = __uint_as_float(v.w);
  } else {
    a[0] = (int32_t)v.x; a[1] = (int32_t)v.y; a[2] = (int32_t)v.z; a[3] = (int32_t)v.w;
  }
}
__device__ __forceinline__ uint4 ld_x_v4(const void *p) {
  // volatile: the compiler keeps every input load ahead of the thread's
  // first output store (in-place calls)
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// Asynchronous 16-byte copy global -> this thread's shared memory (no
// register holds the data in flight), one commit group per call site, and a
// wait until at most N of this thread's groups are still pending.
__device__ __forceinline__ void cp_async16(void *smem, const void *gmem) {
  const unsigned sa = (unsigned)__cvta_generic_to_shared(smem);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(sa), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
template <int PMAX>
__device__ __forceinline__ void cp_async_wait_rt(int n) {  // n in [0, PMAX): unrolled callers fold it
  if constexpr (PMAX > 0) {
    if (n >= PMAX - 1) { cp_async_wait<PMAX - 1>(); return; }
    if constexpr (PMAX > 1) cp_async_wait_rt<PMAX - 1>(n);
    else cp_async_wait<0>();
  }
}

struct RingLinkParams {
  const char *x[kMaxRanks];
  char *y[kMaxRanks];
  uint64_t cv;  // vectors per chunk (C / VEC)
  uint64_t nv;  // vectors in the whole per-rank vector (n / VEC)
  float scale;
  int p;
};

template <class T, int OP, int PMAX, int L, int MINB, bool XS, int XD = 0>
__global__ void __launch_bounds__(PMAX * L, MINB) rc_ring_link_kernel(const __grid_constant__ RingLinkParams a) {
  using Acc = typename T::Acc;
  constexpr int VEC = kVec<T>;
  constexpr int W = VEC / 4;  // 16-byte words per partial message (1, or 2 for bf16)
  // [2 parities][p senders][W][L] links; with XS, then [p ranks][p slots][L]
  // staged inputs (each thread's own: written by its cp.async, read by it)
  extern __shared__ uint4 link[];
  const int p = a.p;
  const int r = threadIdx.x / L;
  const int l = threadIdx.x - r * L;
  const uint64_t cv = a.cv;
  const uint64_t o = (uint64_t)blockIdx.x * L + l;  // vector offset inside every chunk
  auto wrap = [p](int v) { return v < 0 ? v + p : v; };  // v > -p
  auto live = [&](int c) -> bool {  // chunk c has an element vector at offset o
    const uint64_t b = (uint64_t)c * cv;
    return o < cv && b + o < a.nv;
  };
  const int prev = wrap(r - 1);
  pdl_wait();

  // rank r's inputs, chunk c_j = (r-1-j) mod p in slot j, loaded in order of
  // use: into registers, or (XS) by asynchronous copies into shared memory,
  // one commit group per slot (PMAX groups, the ones past p empty), so that
  // slot j is ready once at most PMAX-1-j groups are pending
  // With a window (XD > 0) only XD slots per thread exist: slot j lives in
  // buffer j % XD, slot j + XD is requested as soon as slot j has been
  // consumed, and every wait allows XD - 1 pending groups.
  constexpr int NS = (XS && XD > 0) ? XD : PMAX;  // staged slots per thread
  uint4 xr[XS ? 1 : PMAX];
  uint4 *xs = link + (size_t)2 * p * W * L + (size_t)r * (XD > 0 ? XD : p) * L + l;
  const char *xb = a.x[r];
  auto request = [&](int j) {  // slot j (one commit group, empty past p or off the data)
    if (j < p) {
      const int c = wrap(r - 1 - j);
      if (live(c)) {
        if constexpr (XS) cp_async16(xs + (j % NS) * L, xb + ((uint64_t)c * cv + o) * 16);
        else xr[j] = ld_x_v4(xb + ((uint64_t)c * cv + o) * 16);
      }
    }
    if constexpr (XS) cp_async_commit();
  };
#pragma unroll
  for (int j = 0; j < NS; ++j) request(j);
  auto xslot = [&](int j) -> uint4 {
    if constexpr (XS && XD > 0) {
      cp_async_wait<XD - 1>();
      return xs[(j % NS) * L];
    } else if constexpr (XS) {
      cp_async_wait_rt<PMAX>(PMAX - 1 - j);
      return xs[j * L];
    } else {
      return xr[j];
    }
  };
  auto consumed = [&](int j) {  // slot j's buffer is free: request slot j + XD
    if constexpr (XS && XD > 0) request(j + XD);
  };
  char *yb = a.y[r];

  // ---- reduce-scatter: p-1 steps
  Acc msg[VEC];
  if (live(prev)) unpack<T>(xslot(0), msg);  // step 0 sends x_r[chunk r-1]
  consumed(0);
#pragma unroll
  for (int k = 0; k < PMAX - 1; ++k) {
    if (k + 1 >= p) break;
    uint4 *out = link + ((size_t)((k & 1) * p + r) * W) * L + l;
    const uint4 *in = link + ((size_t)((k & 1) * p + prev) * W) * L + l;
    const int cs = wrap(r - 1 - k), cr = wrap(r - 2 - k);
    if (live(cs)) {
#pragma unroll
      for (int h = 0; h < W; ++h) out[h * L] = acc4_bits(msg + 4 * h);
    }
    __syncthreads();
    if (live(cr)) {
#pragma unroll
      for (int h = 0; h < W; ++h) bits_acc4(in[h * L], msg + 4 * h);
      Acc xv[VEC];
      unpack<T>(xslot(k + 1), xv);
#pragma unroll
      for (int e = 0; e < VEC; ++e) msg[e] = combine<OP>(msg[e], xv[e]);
    }
    consumed(k + 1);
  }
  // the received chunk of the last step is r itself: finished
  uint4 fwd = make_uint4(0, 0, 0, 0);
  if (live(r)) {
#pragma unroll
    for (int e = 0; e < VEC; ++e) msg[e] = finish<OP>(msg[e], a.scale);
    char *dst = yb + ((uint64_t)r * cv + o) * 16;
    store_vec<T, VEC, true>(dst, msg);
    if constexpr (std::is_same<T, BF16>::value)
      fwd = make_uint4(pack_bf16x2(msg[0], msg[1]), pack_bf16x2(msg[2], msg[3]),
                       pack_bf16x2(msg[4], msg[5]), pack_bf16x2(msg[6], msg[7]));
    else
      fwd = acc4_bits(msg);
  }

  // ---- all-gather: p-1 steps, finished vectors in their stored form
#pragma unroll
  for (int k = 0; k < PMAX - 1; ++k) {
    if (k + 1 >= p) break;
    const int par = (p - 1 + k) & 1;
    const int cs = wrap(r - k), cr = wrap(r - 1 - k);
    if (live(cs)) link[((size_t)(par * p + r) * W) * L + l] = fwd;
    __syncthreads();
    if (live(cr)) {
      fwd = link[((size_t)(par * p + prev) * W) * L + l];
      st_v4_cs(yb + ((uint64_t)cr * cv + o) * 16, fwd);
    }
  }
}

template <class T, int OP, int PMAX, int L, int MINB = 1, bool XS = false, int XD = 0>
cudaError_t launch_ring_link_t(const RingJob &job, uint64_t C, cudaStream_t s) {
  RingLinkParams a{};
  const int p = job.p;
  if (p < 2 || p > PMAX) return cudaErrorInvalidValue;
  constexpr int VEC = kVec<T>;
  a.p = p;
  a.cv = C / VEC;
  a.nv = job.n / VEC;
  a.scale = job.scale;
  for (int r = 0; r < p; ++r) {
    a.x[r] = static_cast<const char *>(job.x[r]);
    a.y[r] = static_cast<char *>(job.y[r]);
  }
  const uint64_t grid = (a.cv + L - 1) / L;
  if (grid == 0) return cudaSuccess;
  if (grid > 0x7fffffffull) return cudaErrorInvalidValue;
  const size_t slots = XS ? (XD > 0 ? (size_t)XD : (size_t)p) : 0;  // staged slots per thread
  const size_t smem = ((size_t)2 * p * (VEC / 4) + (size_t)p * slots) * L * 16;
  auto kern = rc_ring_link_kernel<T, OP, PMAX, L, MINB, XS, XD>;
  if (smem > 48 * 1024) {  // opt in to the larger shared-memory carve-out, once per device
    static std::atomic<uint64_t> attr_set{0};
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    const uint64_t bit = 1ull << (dev & 63);
    if (!(attr_set.load() & bit)) {
      const int most = (int)(((size_t)2 * PMAX * (VEC / 4) + (size_t)PMAX * (XD > 0 ? XD : PMAX)) * L * 16);
      err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, most);
      if (err != cudaSuccess) return err;
      attr_set.fetch_or(bit);
    }
  }
  return launch_kernel(kern, dim3((unsigned)grid), dim3(p * L), smem, s, a);
}

template <class T, int OP>
cudaError_t launch_ring_link(const RingJob &job, uint64_t C, cudaStream_t s) {
  // Lanes per rank: 16 for p > 4, 32 for p <= 4 (blocks of 128-256 threads).
  const int lanes = env_int("RC_RING_LANES", 0);
  const bool xs = env_int("RC_RING_XSMEM", 1) != 0;
  if (job.p <= 4) {
    if (xs) return launch_ring_link_t<T, OP, 4, 32, 1, true>(job, C, s);
    if (lanes == 64) return launch_ring_link_t<T, OP, 4, 64>(job, C, s);
    return launch_ring_link_t<T, OP, 4, 32>(job, C, s);
  }
  // staged-input window (RC_RING_XWIN): all p slots by default for p <= 8
  // (a window of 4 or 6 measured no faster there); 4 slots for p > 8, where
  // 16 slots per thread would hold the block to 2 per SM in bf16 (16 ranks x
  // 8 MiB: 47.4 vs 52.1 us bf16, 46.2 vs 46.6 us fp32); 0 keeps every slot
  const int win = env_int("RC_RING_XWIN", -1);
  if (job.p <= 8) {
    if (xs && win == 4) return launch_ring_link_t<T, OP, 8, 16, 1, true, 4>(job, C, s);
    if (xs && win == 6) return launch_ring_link_t<T, OP, 8, 16, 1, true, 6>(job, C, s);
    if (xs) return launch_ring_link_t<T, OP, 8, 16, 1, true>(job, C, s);
    if (lanes == 32) return launch_ring_link_t<T, OP, 8, 32>(job, C, s);
    return launch_ring_link_t<T, OP, 8, 16>(job, C, s);
  }
  if (xs && win == 0) return launch_ring_link_t<T, OP, 16, 16, 1, true>(job, C, s);
  if (xs && win == 8) return launch_ring_link_t<T, OP, 16, 16, 1, true, 8>(job, C, s);
  if (xs) return launch_ring_link_t<T, OP, 16, 16, 1, true, 4>(job, C, s);
  return launch_ring_link_t<T, OP, 16, 16>(job, C, s);
}

template <class T, int OP, int PMAX>
cudaError_t run_ring(const RingJob &job, cudaStream_t s) {
  RingParams a{};
  const int p = job.p;
  a.p = p;
  a.n = job.n;
  a.C = (job.n + p - 1) / p;
  a.scale = job.scale;
  a.ws = static_cast<char *>(job.ws);
  bool aligned = reinterpret_cast<uintptr_t>(job.ws) % 16 == 0;
  for (int r = 0; r < p; ++r) {
    a.x[r] = static_cast<const char *>(job.x[r]);
    a.y[r] = static_cast<char *>(job.y[r]);
    aligned = aligned && reinterpret_cast<uintptr_t>(job.x[r]) % 16 == 0 &&
              reinterpret_cast<uintptr_t>(job.y[r]) % 16 == 0;
  }
  constexpr int VEC = kVec<T>;
  const bool vector = aligned && a.C % VEC == 0 && a.n % VEC == 0;
  // RC_RING_KERNEL: 2 (default) the link kernel, 1 the chain kernel, 0 the
  // element-register kernel; a job that brings its own partial buffer
  // (job.partials_in_ws) runs the chain kernel.
  const int kern_sel = job.partials_in_ws ? 1 : env_int("RC_RING_KERNEL", 2);
  if (vector && kern_sel == 2) return launch_ring_link<T, OP>(job, a.C, s);
  if (vector && kern_sel == 1) {
    // default: 4 chains per thread, x one step ahead (72 registers, so that
    // at p = 8 every offset's chains are resident at once); measured against
    // 2 and 8 chains and a two-step prefetch.  RC_RING_KERNEL=0 selects the
    // register kernel above on this path too.
    const int ch = env_int("RC_RING_CH", 4), pf = env_int("RC_RING_PF", 1);
    if (ch == 2) return pf == 1 ? launch_ring_chain<T, OP, 2, 1>(job, a.C, s) : launch_ring_chain<T, OP, 2, 2>(job, a.C, s);
    if (ch == 8) return pf == 1 ? launch_ring_chain<T, OP, 8, 1>(job, a.C, s) : launch_ring_chain<T, OP, 8, 2>(job, a.C, s);
    return pf == 1 ? launch_ring_chain<T, OP, 4, 1>(job, a.C, s) : launch_ring_chain<T, OP, 4, 2>(job, a.C, s);
  }
  const int sms = device_sm_count();
  const bool l1 = env_int("RC_RING_L1", 1) != 0;
  auto kern = vector ? (l1 ? rc_ring_literal_kernel<T, OP, true, PMAX, true>
                           : rc_ring_literal_kernel<T, OP, true, PMAX, false>)
                     : rc_ring_literal_kernel<T, OP, false, PMAX, false>;
  a.units = vector ? a.C / VEC : a.C;
  int occ = 0;
  cudaError_t err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, kRingNT, 0);
  if (err != cudaSuccess) return err;
  occ = std::max(1, std::min(occ, env_int("RC_CTAS_PER_SM", occ)));
  uint64_t grid = std::min<uint64_t>((uint64_t)sms * occ, (a.units + kRingNT - 1) / kRingNT);
  grid = std::max<uint64_t>(grid, 1);
  return launch_kernel(kern, dim3((unsigned)grid), dim3(kRingNT), 0, s, a);
}

template <class T, int OP>
cudaError_t ring_by_p(const RingJob &job, cudaStream_t s) {
  if (job.p <= 4) return run_ring<T, OP, 4>(job, s);
  if (job.p <= 8) return run_ring<T, OP, 8>(job, s);
  return run_ring<T, OP, 16>(job, s);
}

template <class T>
cudaError_t ring_by_op(const RingJob &job, cudaStream_t s) {
  switch (job.op) {
    case kSum: return ring_by_p<T, kSum>(job, s);
    case kMax: return ring_by_p<T, kMax>(job, s);
    case kMin: return ring_by_p<T, kMin>(job, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

// ---------------------------------------------------------------------------
// Fixed scratch for rc_ring_all_reduce_noalloc: the bf16 ring's fp32
// partials, [2 parities][p][ceil(n/p)] floats, in a file-scope device array
// instead of an allocation.  Every GPU that loads this library holds it until
// the process exits.  Calls that use it and overlap on the GPU race on it.
// Nothing in it needs clearing: every partial is written before it is read.
constexpr size_t kNoallocScratchFloats = size_t(4) << 20;  // 16 MiB
static __device__ __align__(256) float g_noalloc_scratch[kNoallocScratchFloats];

size_t noalloc_scratch_floats() { return kNoallocScratchFloats; }

// Device address of the array for the current device.  In host code the
// symbol's name is only a host-side handle, so the address is looked up once
// per device (with that device current) and cached until rc_finalize, which
// forgets the cache (a device reset reloads the module, so it must come after
// rc_finalize).
std::mutex g_noalloc_mu;
void *g_noalloc_ptrs[64] = {};

void noalloc_scratch_forget() {
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  for (void *&q : g_noalloc_ptrs) q = nullptr;
}

cudaError_t noalloc_scratch_ptr(void **out) {
  std::mutex &mu = g_noalloc_mu;
  void **ptrs = g_noalloc_ptrs;
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (!ptrs[dev]) {
    void *p = nullptr;
    err = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (err != cudaSuccess) return err;
    ptrs[dev] = p;
  }
  *out = ptrs[dev];
  return cudaSuccess;
}

bool ring_needs_workspace(const RingJob &job) {
  if (job.dt != kBF16) return false;  // fp32 / int32 partials live in y
  bool aligned = true;
  for (int r = 0; r < job.p; ++r)
    aligned = aligned && reinterpret_cast<uintptr_t>(job.x[r]) % 16 == 0 &&
              reinterpret_cast<uintptr_t>(job.y[r]) % 16 == 0;
  const uint64_t C = (job.n + job.p - 1) / job.p;
  const bool vector = aligned && C % 8 == 0 && job.n % 8 == 0;
  const int kern_sel = job.partials_in_ws ? 1 : env_int("RC_RING_KERNEL", 2);
  return !(vector && kern_sel == 2);  // the link kernel keeps its partials on chip
}

cudaError_t launch_ring_literal(const RingJob &job, cudaStream_t s) {
  switch (job.dt) {
    case kF32: return ring_by_op<F32>(job, s);
    case kBF16: return ring_by_op<BF16>(job, s);
    case kI32: return ring_by_op<I32>(job, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace rc
