// Shared device helpers of the MoE layer library (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "moe.h"

namespace moe {

using bf16 = __nv_bfloat16;

// Device error word bits (kept in the first bytes of a workspace).
constexpr unsigned kErrNonfiniteLogit = MOE_DEVERR_NONFINITE_LOGIT;
constexpr unsigned kErrTimeout = MOE_DEVERR_TIMEOUT;

// Number of bytes reserved at the head of every workspace for the error word
// (256 keeps what follows aligned for TMA and vector access).
constexpr size_t kWsHeader = 256;

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(bf16 v) { return __bfloat162float(v); }

template <typename T>
__device__ __forceinline__ T from_f32(float v);
template <>
__device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ bf16 from_f32<bf16>(float v) { return __float2bfloat16_rn(v); }

// 16-byte vector of elements: 8 bf16 or 4 fp32.
template <typename T>
struct Vec16 {
  static constexpr int N = 16 / sizeof(T);
  uint4 raw;
  __device__ __forceinline__ float get(int i) const {
    const T* p = reinterpret_cast<const T*>(&raw);
    return to_f32(p[i]);
  }
  __device__ __forceinline__ void set(int i, float v) {
    T* p = reinterpret_cast<T*>(&raw);
    p[i] = from_f32<T>(v);
  }
};

template <typename T>
__device__ __forceinline__ Vec16<T> ld16(const T* p) {
  Vec16<T> v;
  v.raw = __ldg(reinterpret_cast<const uint4*>(p));
  return v;
}
// Streaming load for data read exactly once.
template <typename T>
__device__ __forceinline__ Vec16<T> ld16_stream(const T* p) {
  Vec16<T> v;
  v.raw = __ldcs(reinterpret_cast<const uint4*>(p));
  return v;
}
template <typename T>
__device__ __forceinline__ void st16(T* p, const Vec16<T>& v) {
  *reinterpret_cast<uint4*>(p) = v.raw;
}

// sigmoid and silu with the fast exponential and fast division intrinsics:
// a few ulp in fp32, far below the bf16 rounding of the values they feed, and
// correct in the limits (for u << 0 the denominator overflows to +inf and the
// quotient is 0).
__device__ __forceinline__ float sigmoid_f(float u) { return __fdividef(1.0f, 1.0f + __expf(-u)); }
__device__ __forceinline__ float silu_f(float u) { return u * sigmoid_f(u); }

__device__ __forceinline__ void raise_error(unsigned* err, unsigned bit) {
  if (err) atomicOr(err, bit);
}

}  // namespace moe
