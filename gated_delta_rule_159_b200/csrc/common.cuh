// common.cuh -- small device helpers shared by the libgdn2 kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/gdn2.h"

namespace gdn2 {

constexpr float kLog2e = 1.4426950408889634f;

// exp(x) via the hardware base-2 exponential: exp(x) = 2^(x * log2(e)).
__device__ __forceinline__ float exp_fast(float x) { return exp2f(x * kLog2e); }

// Fused prologue (GDN2_FUSED_PROLOGUE): sigmoid gates and the L2 normalisation
// of q and k, x / sqrt(|x|^2 + kNormEps).
constexpr float kNormEps = 1e-6f;

__device__ __forceinline__ float sigmoid_f(float x) { return __fdividef(1.f, 1.f + exp_fast(-x)); }

// log sigmoid(x) = min(x, 0) - log(1 + e^{-|x|}); the argument of the log lies in [1, 2].
__device__ __forceinline__ float log_sigmoid_f(float x) { return fminf(x, 0.f) - __logf(1.f + exp_fast(-fabsf(x))); }

template <typename T>
__device__ __forceinline__ float to_f32(T v);
template <>
__device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }

template <typename T>
__device__ __forceinline__ T from_f32(float v);
template <>
__device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&h);
}

__device__ __forceinline__ float2 unpack_bf16x2(uint32_t u) {
  __nv_bfloat162 h = *reinterpret_cast<__nv_bfloat162 *>(&u);
  return __bfloat1622float2(h);
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

}  // namespace gdn2
