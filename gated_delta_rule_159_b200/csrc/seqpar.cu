// seqpar.cu -- sequence-parallel chunked forward: long sequences split into
// segments that run side by side.
//
// The recurrence is affine in its state (neelmishra.github.io, "What makes the
// architecture more than a recurrence": the affine-composition view of DeltaNet
// still holds once each transition includes decay).  For a segment with start
// state S_s the end state is S_e = F S_s + G, and every output splits as
// o_t = o_t(S_s = 0) + o_t(S_s, v = 0).  With d_k = d_v the transition F is the
// end state of the segment run from S_s = I with v = 0.  Hence three passes of
// the chunk kernel over all segments at once, with one serial combine:
//
//   1. S_s = 0 (the first segment of a sequence keeps S0): o and G per segment;
//   2. S_s = I, v = 0: F per segment;
//   3. combine per (sequence, head): S_s(j+1) = F_j S_s(j) + G_j, S_T = the last;
//   4. S_s = the combined starts, v = 0, for every segment but the first: the
//      correction o(S_s, v = 0), added to o.
//
// The work is about three forwards, spread over n_split times as many units.
#include "common.cuh"
#include "internal.h"

namespace gdn2 {
namespace {

constexpr int kComb = 512;  // threads of the combine kernel: 4 per row, 32 columns each
constexpr int kIntBlock = 960;  // int32 values per plan-upload launch (a 3.8 KB parameter block)

// Segment boundaries of N sequences of T tokens cut every L tokens.
__global__ void seg_bounds_kernel(int32_t *cu, int N, int T, int L, int ns) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i > N * ns) return;
  const int n = i / ns, j = i % ns;
  int v;
  if (i == N * ns) v = N * T;
  else v = n * T + (j * L < T ? j * L : T);
  cu[i] = v;
}

// Start states of pass 1 (S0 in each sequence's first segment, 0 elsewhere) or
// identities for pass 2.  One CTA per (segment, head), 128 x 128 floats.
__global__ void seg_states_kernel(float *dst, const float *S0, int ns, int H, bool identity) {
  const int sh = blockIdx.x;  // seg * H + h
  const int seg = sh / H, h = sh % H, n = seg / ns, j = seg % ns;
  float *d = dst + (size_t)sh * 128 * 128;
  for (int e = threadIdx.x; e < 128 * 128; e += blockDim.x) {
    float v = 0.f;
    if (identity) v = (e / 128 == e % 128) ? 1.f : 0.f;
    else if (j == 0 && S0) v = S0[((size_t)n * H + h) * 128 * 128 + e];
    d[e] = v;
  }
}

// Serial combine per (sequence, head): S <- F_j S + G_j over the segments.
// starts[(n, j)] receives the start state of segment j (zero for j = 0, whose
// outputs already include S0); S_T[n] the final state.
__global__ void __launch_bounds__(kComb) combine_kernel(const float *F, const float *G, float *starts, float *S_T,
                                                        int ns, int H) {
  extern __shared__ float Ss[];  // [128][128] current state
  const int unit = blockIdx.x, n = unit / H, h = unit % H;
  const int t = threadIdx.x, r = t >> 2, c0 = (t & 3) * 32;
  auto at = [&](const float *base, int j) { return base + (((size_t)n * ns + j) * H + h) * 128 * 128; };
  auto start = [&](int j) { return starts + (((size_t)n * ns + j) * H + h) * 128 * 128; };
  // segment 0 ends in G_0 (its start, S0, is already folded in)
  for (int e = t; e < 128 * 128; e += kComb) {
    Ss[e] = at(G, 0)[e];
    start(0)[e] = 0.f;
  }
  __syncthreads();
  for (int j = 1; j < ns; ++j) {
    for (int e = t; e < 128 * 128; e += kComb) start(j)[e] = Ss[e];
    const float *Fr = at(F, j) + (size_t)r * 128;
    float acc[32];
#pragma unroll
    for (int c = 0; c < 32; ++c) acc[c] = at(G, j)[(size_t)r * 128 + c0 + c];
    for (int kk = 0; kk < 128; ++kk) {
      const float f = Fr[kk];
#pragma unroll
      for (int c = 0; c < 32; ++c) acc[c] += f * Ss[kk * 128 + c0 + c];
    }
    __syncthreads();  // everyone has read the old state
#pragma unroll
    for (int c = 0; c < 32; ++c) Ss[r * 128 + c0 + c] = acc[c];
    __syncthreads();
  }
  if (S_T) {
    float *d = S_T + ((size_t)n * H + h) * 128 * 128;
    for (int e = t; e < 128 * 128; e += kComb) d[e] = Ss[e];
  }
}

// Start state of segment `upto` and, when S_T is given, the end state after all n_segs
// segments, for one (sequence, head) per CTA, from per-segment maps laid out with element
// strides (in 128 x 128 matrices) seg_stride between segments and seq_stride between
// sequences: S <- F_j S + G_j from S = 0 (segment 0's map already carries the true S0).
__global__ void __launch_bounds__(kComb) prefix_kernel(const float *F, const float *G, size_t seg_stride,
                                                       size_t seq_stride, float *start, float *S_T, int upto,
                                                       int n_segs, int H) {
  extern __shared__ float Ss[];  // [128][128] current state
  const int unit = blockIdx.x, n = unit / H, h = unit % H;
  const int t = threadIdx.x, r = t >> 2, c0 = (t & 3) * 32;
  auto at = [&](const float *base, int j) { return base + ((size_t)j * seg_stride + (size_t)n * seq_stride + h) * 128 * 128; };
  for (int e = t; e < 128 * 128; e += kComb) Ss[e] = 0.f;
  __syncthreads();
  const int last = S_T ? n_segs : upto;
  for (int j = 0; j <= last; ++j) {
    if (j == upto && start) {
      float *d = start + (size_t)unit * 128 * 128;
      for (int e = t; e < 128 * 128; e += kComb) d[e] = Ss[e];
    }
    if (j == last) break;
    const float *Fr = at(F, j) + (size_t)r * 128;
    float acc[32];
#pragma unroll
    for (int c = 0; c < 32; ++c) acc[c] = at(G, j)[(size_t)r * 128 + c0 + c];
    if (j > 0) {  // S = 0 before segment 0
      for (int kk = 0; kk < 128; ++kk) {
        const float f = Fr[kk];
#pragma unroll
        for (int c = 0; c < 32; ++c) acc[c] += f * Ss[kk * 128 + c0 + c];
      }
    }
    __syncthreads();  // everyone has read the old state
#pragma unroll
    for (int c = 0; c < 32; ++c) Ss[r * 128 + c0 + c] = acc[c];
    __syncthreads();
  }
  if (S_T) {
    float *d = S_T + (size_t)unit * 128 * 128;
    for (int e = t; e < 128 * 128; e += kComb) d[e] = Ss[e];
  }
}

// ---- packed varlen split (gdn2_chunk_fwd_split_varlen)

// A block of host-planned int32 values written to device memory by a launch parameter (no
// host-side copy, no stream synchronisation).
struct IntBlock {
  int32_t n;
  int32_t v[kIntBlock];
};
__global__ void write_ints_kernel(int32_t *dst, const __grid_constant__ IntBlock b) {
  for (int i = threadIdx.x; i < b.n; i += blockDim.x) dst[i] = b.v[i];
}

// Start states, one CTA per (unit, head): src[unit] = -2 identity, -1 zeros, n >= 0 S0[n, h].
__global__ void fill_starts_kernel(float *dst, const int32_t *src, const float *S0, int H) {
  const int uh = blockIdx.x, u = uh / H, h = uh % H;
  const int s = src[u];
  float *d = dst + (size_t)uh * 128 * 128;
  const float *from = (s >= 0 && S0) ? S0 + ((size_t)s * H + h) * 128 * 128 : nullptr;
  for (int e = threadIdx.x; e < 128 * 128; e += blockDim.x)
    d[e] = s == -2 ? ((e / 128 == e % 128) ? 1.f : 0.f) : (from ? from[e] : 0.f);
}

// Per (sequence, head), serial over its m segments (seq_info[n] = {m, first segment in the
// pass-1 list, first in the pass-2 list, first in the pass-3 list}).  m == 1: the pass-1 end
// state is S_T.  m > 1: with G_j the segment's end state from 0 (pass 1) and E_j from the
// identity (pass 2), F_j = E_j - G_j; S <- F_j S + G_j from S = S0 (or 0), recording the start
// of every segment that pass 3 re-runs (all of them with S0, else j >= 1).
__global__ void __launch_bounds__(kComb) combine_varlen_kernel(const int32_t *seq_info, const float *E,
                                                               const float *G, float *starts3, const float *S0,
                                                               float *S_T, int H) {
  extern __shared__ float Ss[];  // [128][128] current state
  const int unit = blockIdx.x, n = unit / H, h = unit % H;
  const int t = threadIdx.x, r = t >> 2, c0 = (t & 3) * 32;
  const int m = seq_info[4 * n], g0 = seq_info[4 * n + 1], e0 = seq_info[4 * n + 2], c3 = seq_info[4 * n + 3];
  auto mat = [&](const float *base, int idx) { return base + ((size_t)idx * H + h) * 128 * 128; };
  auto mat_w = [&](float *base, int idx) { return base + ((size_t)idx * H + h) * 128 * 128; };
  if (m == 1) {
    if (S_T) {
      float *d = S_T + (size_t)unit * 128 * 128;
      for (int e = t; e < 128 * 128; e += kComb) d[e] = mat(G, g0)[e];
    }
    return;
  }
  const float *s0 = S0 ? S0 + (size_t)unit * 128 * 128 : nullptr;
  for (int e = t; e < 128 * 128; e += kComb) Ss[e] = s0 ? s0[e] : 0.f;
  __syncthreads();
  int k3 = c3;
  for (int j = 0; j < m; ++j) {
    if (j > 0 || S0) {
      float *d = mat_w(starts3, k3++);
      for (int e = t; e < 128 * 128; e += kComb) d[e] = Ss[e];
    }
    const float *Er = mat(E, e0 + j) + (size_t)r * 128, *Gr = mat(G, g0 + j) + (size_t)r * 128;
    float acc[32];
#pragma unroll
    for (int c = 0; c < 32; ++c) acc[c] = Gr[c0 + c];
    for (int kk = 0; kk < 128; ++kk) {
      const float f = Er[kk] - Gr[kk];
#pragma unroll
      for (int c = 0; c < 32; ++c) acc[c] += f * Ss[kk * 128 + c0 + c];
    }
    __syncthreads();  // everyone has read the old state
#pragma unroll
    for (int c = 0; c < 32; ++c) Ss[r * 128 + c0 + c] = acc[c];
    __syncthreads();
  }
  if (S_T) {
    float *d = S_T + (size_t)unit * 128 * 128;
    for (int e = t; e < 128 * 128; e += kComb) d[e] = Ss[e];
  }
}

template <typename T>
__global__ void add_kernel(T *o, const T *d, size_t n) {
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x)
    o[i] = from_f32<T>(to_f32(o[i]) + to_f32(d[i]));
}

size_t up256(size_t x) { return (x + 255) / 256 * 256; }

}  // namespace

SplitPlan split_plan(int N, int T, int H, int n_split, int dtype_in, int dtype_out, size_t inner_bytes) {
  SplitPlan s;
  const int nc = (T + 63) / 64;
  const int per = (nc + n_split - 1) / n_split;
  s.seg_len = per * 64;
  s.n_per_seq = (T + s.seg_len - 1) / s.seg_len;
  if (s.n_per_seq < 1) s.n_per_seq = 1;
  s.n_segs = N * s.n_per_seq;
  const size_t state = (size_t)s.n_segs * H * 128 * 128 * sizeof(float);
  const size_t tok = (size_t)N * T * H * 128;
  const size_t in_e = dtype_in == GDN2_BF16 ? 2 : 4, out_e = dtype_out == GDN2_BF16 ? 2 : 4;
  // the inner forwards' workspace comes first: its status word is word 0 of the whole workspace
  s.off_inner = 0;
  s.off_cu = up256(inner_bytes);
  s.off_start = s.off_cu + up256((size_t)(s.n_segs + 1) * sizeof(int32_t));
  s.off_F = s.off_start + up256(state);
  s.off_G = s.off_F + up256(state);
  s.off_zero_v = s.off_G + up256(state);
  s.off_o2 = s.off_zero_v + up256(tok * in_e);
  s.total = s.off_o2 + up256(tok * out_e);
  return s;
}

cudaError_t write_ints(int32_t *dst, const int32_t *vals, size_t n, cudaStream_t stream) {
  for (size_t i = 0; i < n; i += kIntBlock) {
    IntBlock b;
    b.n = (int32_t)(n - i < (size_t)kIntBlock ? n - i : (size_t)kIntBlock);
    for (int j = 0; j < b.n; ++j) b.v[j] = vals[i + j];
    write_ints_kernel<<<1, 256, 0, stream>>>(dst + i, b);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t launch_fill_starts(float *dst, const int32_t *src, const float *S0, int units, int H,
                               cudaStream_t stream) {
  if (units == 0) return cudaSuccess;
  fill_starts_kernel<<<units * H, 256, 0, stream>>>(dst, src, S0, H);
  return cudaGetLastError();
}

cudaError_t launch_combine_varlen(const int32_t *seq_info, const float *E, const float *G, float *starts3,
                                  const float *S0, float *S_T, int N, int H, cudaStream_t stream) {
  const int smem = 128 * 128 * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(combine_varlen_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  combine_varlen_kernel<<<N * H, kComb, smem, stream>>>(seq_info, E, G, starts3, S0, S_T, H);
  return cudaGetLastError();
}

cudaError_t launch_identities(float *dst, int units, cudaStream_t stream) {
  seg_states_kernel<<<units, 256, 0, stream>>>(dst, nullptr, 1, 1, true);
  return cudaGetLastError();
}

cudaError_t launch_add(void *o, const void *o2, size_t n, int dtype_out, cudaStream_t stream) {
  if (dtype_out == GDN2_BF16)
    add_kernel<__nv_bfloat16><<<592, 256, 0, stream>>>(static_cast<__nv_bfloat16 *>(o),
                                                       static_cast<const __nv_bfloat16 *>(o2), n);
  else
    add_kernel<float><<<592, 256, 0, stream>>>(static_cast<float *>(o), static_cast<const float *>(o2), n);
  return cudaGetLastError();
}

cudaError_t launch_prefix(const float *F, const float *G, size_t seg_stride, size_t seq_stride, float *start,
                          float *S_T, int upto, int n_segs, int N, int H, cudaStream_t stream) {
  const int smem = 128 * 128 * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(prefix_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  prefix_kernel<<<N * H, kComb, smem, stream>>>(F, G, seg_stride, seq_stride, start, S_T, upto, n_segs, H);
  return cudaGetLastError();
}

cudaError_t launch_split_helpers(int what, const SplitArgs &a, cudaStream_t stream) {
  const int segs = a.plan.n_segs;
  switch (what) {
    case 0:  // segment bounds, zero v
      seg_bounds_kernel<<<(segs + 1 + 255) / 256, 256, 0, stream>>>(a.cu, a.N, a.T, a.plan.seg_len, a.plan.n_per_seq);
      break;
    case 1:  // pass 1 starts
      seg_states_kernel<<<segs * a.H, 256, 0, stream>>>(a.starts, a.S0, a.plan.n_per_seq, a.H, false);
      break;
    case 2:  // pass 2 starts: identities
      seg_states_kernel<<<segs * a.H, 256, 0, stream>>>(a.starts, nullptr, a.plan.n_per_seq, a.H, true);
      break;
    case 3: {  // combine
      const int smem = 128 * 128 * sizeof(float);
      cudaError_t e = cudaFuncSetAttribute(combine_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
      if (e != cudaSuccess) return e;
      combine_kernel<<<a.N * a.H, kComb, smem, stream>>>(a.F, a.G, a.starts, a.S_T, a.plan.n_per_seq, a.H);
      break;
    }
    case 4: {  // o += correction
      const size_t n = (size_t)a.N * a.T * a.H * 128;
      if (a.dtype_out == GDN2_BF16)
        add_kernel<__nv_bfloat16><<<592, 256, 0, stream>>>(static_cast<__nv_bfloat16 *>(a.o),
                                                           static_cast<const __nv_bfloat16 *>(a.o2), n);
      else
        add_kernel<float><<<592, 256, 0, stream>>>(static_cast<float *>(a.o), static_cast<const float *>(a.o2), n);
      break;
    }
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace gdn2
