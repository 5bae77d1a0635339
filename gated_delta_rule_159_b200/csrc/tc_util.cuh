// tc_util.cuh -- shared-memory access helpers, the 128-byte swizzle and the bounded
// mbarrier waits shared by the tensor-core kernels (chunk_tc.cu, bwd_tc.cu).
#pragma once

#include "common.cuh"
#include "internal.h"
#include "sm100_ptx.cuh"

namespace gdn2 {
namespace tc {

__device__ __forceinline__ void named_bar(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}
__device__ __forceinline__ uint2 lds_v2(uint32_t a) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
  return v;
}
__device__ __forceinline__ void sts_v2(uint32_t a, uint2 v) {
  asm volatile("st.shared.v2.u32 [%0], {%1, %2};" ::"r"(a), "r"(v.x), "r"(v.y) : "memory");
}
__device__ __forceinline__ void sts_u16(uint32_t a, uint16_t v) {
  asm volatile("st.shared.u16 [%0], %1;" ::"r"(a), "h"(v) : "memory");
}
__device__ __forceinline__ uint16_t lds_u16(uint32_t a) {
  uint16_t v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ void sts_u32(uint32_t a, uint32_t v) {
  asm volatile("st.shared.u32 [%0], %1;" ::"r"(a), "r"(v) : "memory");
}
__device__ __forceinline__ uint16_t bf16_bits(float v) {
  const __nv_bfloat16 h = __float2bfloat16_rn(v);
  return *reinterpret_cast<const uint16_t *>(&h);
}
__device__ __forceinline__ float bf16_value(uint16_t bits) {
  return __uint_as_float((uint32_t)bits << 16);
}
__device__ __forceinline__ void sts_f32(uint32_t a, float v) {
  asm volatile("st.shared.f32 [%0], %1;" ::"r"(a), "f"(v) : "memory");
}
__device__ __forceinline__ void sts_v4(uint32_t a, uint4 v) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}
__device__ __forceinline__ uint4 lds_v4(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
  return v;
}

// Byte offset of (row r, 16-byte chunk `chunk`) in a 128B-swizzled tile: the tiles are stacks
// of 8-row x 128-byte atoms whose 16-byte chunks are permuted by the row's low three bits.
__device__ __forceinline__ uint32_t swz(int r, uint32_t chunk) {
  return (uint32_t)r * 128u + (((chunk ^ (uint32_t)(r & 7))) << 4);
}
// Byte offset of bf16 element (row r, column c) of a [rows][128] bf16 matrix stored as two
// swizzled column blocks of 64 (one 128-byte row each) `block_stride` bytes apart.
__device__ __forceinline__ uint32_t swz_elem(int r, int c, uint32_t block_stride) {
  return (uint32_t)(c >> 6) * block_stride + swz(r, (uint32_t)((c & 63) >> 3)) + (uint32_t)(c & 7) * 2u;
}

// mbarrier wait bounded by `limit_ns`: on timeout it sets the CTA's abort flag and the status
// word (kStatusTimeout) and returns false; it also returns false at once once another thread
// of the CTA has aborted.
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                         int32_t *status, uint64_t limit_ns) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  if (*abort_flag) return false;
  const uint64_t t0 = global_timer_ns();
  uint32_t it = 0;
  while (!ptx::mbar_try_wait(bar, parity)) {
    if ((++it & 255u) == 0) {
      if (*abort_flag) return false;
      if (global_timer_ns() - t0 > limit_ns) {
        *abort_flag = 1;
        if (status) atomicExch(status, kStatusTimeout);
        return false;
      }
    }
  }
  return true;
}

// Bounded wait that ignores the abort flag: the wind-down after a timed-out wait uses it to let
// the copies and MMAs a CTA issued land before it frees its memory.
__device__ __forceinline__ void drain_bar(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
  const uint64_t t0 = global_timer_ns();
  uint32_t it = 0;
  while (!ptx::mbar_try_wait(bar, parity))
    if ((++it & 255u) == 0 && global_timer_ns() - t0 > limit_ns) return;
}

__device__ __forceinline__ uint4 pack8(const float *f, float s) {
  uint4 v;
  v.x = pack_bf16x2(f[0] * s, f[1] * s);
  v.y = pack_bf16x2(f[2] * s, f[3] * s);
  v.z = pack_bf16x2(f[4] * s, f[5] * s);
  v.w = pack_bf16x2(f[6] * s, f[7] * s);
  return v;
}
__device__ __forceinline__ float4 unpack4(uint2 u) {
  const float2 a = unpack_bf16x2(u.x), b = unpack_bf16x2(u.y);
  return make_float4(a.x, a.y, b.x, b.y);
}
__device__ __forceinline__ uint2 pack4(float a, float b, float c, float d) {
  return make_uint2(pack_bf16x2(a, b), pack_bf16x2(c, d));
}

// First checkpoint slot of unit (n, h) in the chunk-start state buffer: sequence n owns
// nchunks_n * H consecutive slots from ckpt_off[n] * H (n * nchunks * H for equal lengths,
// ckpt_off == NULL), head h the nchunks_n of them from h * nchunks_n; slot c holds chunk c's
// start state.
__device__ __forceinline__ int64_t ckpt_first_slot(const int64_t *ckpt_off, int n, int h, int H, int nchunks) {
  const int64_t base = ckpt_off ? ckpt_off[n] : (int64_t)n * nchunks;
  return base * H + (int64_t)h * nchunks;
}

}  // namespace tc
}  // namespace gdn2
