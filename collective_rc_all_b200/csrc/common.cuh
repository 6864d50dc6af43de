// common.cuh -- device helpers shared by the librankcoll kernels (sm_100a).
//
// Arithmetic contract of every reducing kernel (see include/rankcoll.h):
// fp32 accumulate with IEEE round-to-nearest-even adds (the library is built
// with -fmad=false and without fast-math, so no contraction and no flush to
// zero), compare-select MAX/MIN, wrapping int32 adds, one fp32 multiply by
// `scale` after the fold, bf16 narrowing with the round-to-nearest-even
// conversion intrinsics.
#pragma once

#include <cstdint>
#include <type_traits>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace rc {

enum Dtype : int { kF32 = 0, kBF16 = 1, kI32 = 2 };
enum Op : int { kSum = 0, kMax = 1, kMin = 2 };

constexpr int kMaxRanks = 16;

// ---------------------------------------------------------------- dependent launch
// See launch.cuh.  pdl_wait(): block until the kernels this grid depends on
// have completed and their writes are visible; it must precede the first
// global-memory access of every thread.  No kernel releases its dependents
// early (griddepcontrol.launch_dependents): they are released as this
// kernel's blocks exit, so the next kernel's launch overlaps only this
// kernel's drain, and its blocks never take SM slots that this kernel's later
// waves still need.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// ---------------------------------------------------------------- type traits
// Storage tags.  Each has: bytes per element, the accumulator type, and
// widen / narrow conversions.
struct F32 {
  static constexpr int kBytes = 4;
  using Acc = float;
};
struct BF16 {
  static constexpr int kBytes = 2;
  using Acc = float;
};
struct I32 {
  static constexpr int kBytes = 4;
  using Acc = int32_t;
};

// ---------------------------------------------------------------- reductions
template <int OP>
__device__ __forceinline__ float combine(float acc, float v) {
  if constexpr (OP == kSum) {
    return __fadd_rn(acc, v);
  } else if constexpr (OP == kMax) {
    return (v > acc) ? v : acc;
  } else {
    return (v < acc) ? v : acc;
  }
}

template <int OP>
__device__ __forceinline__ int32_t combine(int32_t acc, int32_t v) {
  if constexpr (OP == kSum) {
    return (int32_t)((uint32_t)acc + (uint32_t)v);
  } else if constexpr (OP == kMax) {
    return (v > acc) ? v : acc;
  } else {
    return (v < acc) ? v : acc;
  }
}

// One multiply by scale for floating SUM; other ops carry scale == 1 and the
// value is passed through unchanged.
template <int OP>
__device__ __forceinline__ float finish(float acc, float scale) {
  if constexpr (OP == kSum) {
    return __fmul_rn(acc, scale);
  } else {
    return acc;
  }
}
template <int OP>
__device__ __forceinline__ int32_t finish(int32_t acc, float) {
  return acc;
}

// ---------------------------------------------------------------- conversions
__device__ __forceinline__ float bf16_bits_to_f32(uint32_t h16) {
  return __uint_as_float(h16 << 16);
}

// two fp32 -> packed bf16x2 (lo in the low half), round to nearest even
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&v);
}

__device__ __forceinline__ uint16_t f32_to_bf16_bits(float f) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}

// Scalar element load/store in a storage type, widened to the accumulator.
template <class T>
__device__ __forceinline__ typename T::Acc load_elem(const char *base, uint64_t i);
template <>
__device__ __forceinline__ float load_elem<F32>(const char *base, uint64_t i) {
  return reinterpret_cast<const float *>(base)[i];
}
template <>
__device__ __forceinline__ float load_elem<BF16>(const char *base, uint64_t i) {
  return bf16_bits_to_f32(reinterpret_cast<const uint16_t *>(base)[i]);
}
template <>
__device__ __forceinline__ int32_t load_elem<I32>(const char *base, uint64_t i) {
  return reinterpret_cast<const int32_t *>(base)[i];
}

template <class T>
__device__ __forceinline__ void store_elem(char *base, uint64_t i, typename T::Acc v);
template <>
__device__ __forceinline__ void store_elem<F32>(char *base, uint64_t i, float v) {
  reinterpret_cast<float *>(base)[i] = v;
}
template <>
__device__ __forceinline__ void store_elem<BF16>(char *base, uint64_t i, float v) {
  reinterpret_cast<uint16_t *>(base)[i] = f32_to_bf16_bits(v);
}
template <>
__device__ __forceinline__ void store_elem<I32>(char *base, uint64_t i, int32_t v) {
  reinterpret_cast<int32_t *>(base)[i] = v;
}

// ---------------------------------------------------------------- 16-byte vectors
// A 16-byte vector of input type T holds kVec<T> elements.
template <class T>
constexpr int kVec = 16 / T::kBytes;

// Read-only streaming load: non-coherent path, no L1 allocation.  Only for
// data no thread writes before this thread's own read of it in the kernel.
__device__ __forceinline__ uint4 ld_stream_v4(const void *p) {
  uint4 v;
  asm("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
      : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
      : "l"(p));
  return v;
}

__device__ __forceinline__ void st_v4(void *p, uint4 v) {
  asm volatile("st.global.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}
__device__ __forceinline__ void st_v2(void *p, uint2 v) {
  asm volatile("st.global.v2.u32 [%0], {%1,%2};" ::"l"(p), "r"(v.x), "r"(v.y) : "memory");
}
// Streaming stores (cache-streaming, .cs: the line is likely written once and
// not read again here, so L2 evicts it first).  Used for the outputs of the
// collectives with many destinations, which no kernel of the call reads back:
// they leave fewer dirty lines in L2 for the next kernel to write back.
// Measured in a sequence of seven collectives (8 ranks x 8 MiB fp32), each
// collective back to back with itself: all-gather 8.17 -> 7.73 us, broadcast
// 12.8 -> 12.3, hierarchical all-reduce 23.96 -> 23.56, all-reduce 24.1 ->
// 23.8; the reduce-scatter (one small output per rank) was 3% slower with
// them and keeps ordinary stores.
__device__ __forceinline__ void st_v4_cs(void *p, uint4 v) {
  asm volatile("st.global.cs.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}
__device__ __forceinline__ void st_v2_cs(void *p, uint2 v) {
  asm volatile("st.global.cs.v2.u32 [%0], {%1,%2};" ::"l"(p), "r"(v.x), "r"(v.y) : "memory");
}
template <bool CS>
__device__ __forceinline__ void st16(void *p, uint4 v) {
  if constexpr (CS) st_v4_cs(p, v);
  else st_v4(p, v);
}
template <bool CS>
__device__ __forceinline__ void st8(void *p, uint2 v) {
  if constexpr (CS) st_v2_cs(p, v);
  else st_v2(p, v);
}

// Unpack a raw 16-byte vector of T into kVec<T> accumulators.
template <class T>
__device__ __forceinline__ void unpack(const uint4 &raw, typename T::Acc (&a)[kVec<T>]);
template <>
__device__ __forceinline__ void unpack<F32>(const uint4 &raw, float (&a)[4]) {
  a[0] = __uint_as_float(raw.x);
  a[1] = __uint_as_float(raw.y);
  a[2] = __uint_as_float(raw.z);
  a[3] = __uint_as_float(raw.w);
}
template <>
__device__ __forceinline__ void unpack<I32>(const uint4 &raw, int32_t (&a)[4]) {
  a[0] = (int32_t)raw.x;
  a[1] = (int32_t)raw.y;
  a[2] = (int32_t)raw.z;
  a[3] = (int32_t)raw.w;
}
template <>
__device__ __forceinline__ void unpack<BF16>(const uint4 &raw, float (&a)[8]) {
  const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    a[2 * j] = __uint_as_float(w[j] << 16);
    a[2 * j + 1] = __uint_as_float(w[j] & 0xffff0000u);
  }
}

// Store VEC accumulated values (already scaled) as type TO at address p.
// VEC * TO::kBytes is 8, 16 or 32 bytes.  CS: streaming stores (st16 / st8).
template <class TO, int VEC, bool CS = false>
__device__ __forceinline__ void store_vec(char *p, const typename TO::Acc (&y)[VEC]) {
  if constexpr (std::is_same<TO, F32>::value && VEC == 4) {
    st16<CS>(p, make_uint4(__float_as_uint(y[0]), __float_as_uint(y[1]), __float_as_uint(y[2]),
                           __float_as_uint(y[3])));
  } else if constexpr (std::is_same<TO, I32>::value && VEC == 4) {
    st16<CS>(p, make_uint4((uint32_t)y[0], (uint32_t)y[1], (uint32_t)y[2], (uint32_t)y[3]));
  } else if constexpr (std::is_same<TO, BF16>::value && VEC == 8) {
    st16<CS>(p, make_uint4(pack_bf16x2(y[0], y[1]), pack_bf16x2(y[2], y[3]), pack_bf16x2(y[4], y[5]),
                           pack_bf16x2(y[6], y[7])));
  } else if constexpr (std::is_same<TO, BF16>::value && VEC == 4) {
    st8<CS>(p, make_uint2(pack_bf16x2(y[0], y[1]), pack_bf16x2(y[2], y[3])));
  } else {
    static_assert(std::is_same<TO, F32>::value && VEC == 8, "unsupported output vector");
    st16<CS>(p, make_uint4(__float_as_uint(y[0]), __float_as_uint(y[1]), __float_as_uint(y[2]),
                           __float_as_uint(y[3])));
    st16<CS>(p + 16, make_uint4(__float_as_uint(y[4]), __float_as_uint(y[5]), __float_as_uint(y[6]),
                                __float_as_uint(y[7])));
  }
}

}  // namespace rc
