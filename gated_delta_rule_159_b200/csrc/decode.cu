// decode.cu -- recurrent Gated DeltaNet-2 decode step (one token per sequence).
//
// One CTA owns one (sequence, head) state S (d_k x d_v fp32) and makes a single
// pass over it: every element is loaded once (128-bit, coalesced along d_v),
// decayed in registers, reduced into the two column sums r = Sbar^T k and
// u = Sbar^T q, then updated and stored once:
//
//   Sbar = Diag(a) S,  S' = Sbar - (b.k) r^T + (w.k) v^T,
//   o    = S'^T q = u - (q.(b.k)) r + (q.(w.k)) v.
//
// The operation is the recurrent inference form of Gated DeltaNet-2
// (alanhou.org "Core Mechanism": inference runs as a pure recurrent network with
// O(1) memory per token; gist.science Methodologie 1 for the gates).  Writing o
// through u, r and two dot products is exact algebra (o_t = S_t^T q_t expanded),
// which lets the kernel read S only once.
#include "common.cuh"
#include "internal.h"

namespace gdn2 {
namespace {

constexpr int kThreads = 256;

template <int DV, typename Tin, typename Tout>
__global__ void __launch_bounds__(kThreads) decode_kernel(DecodeProblem p) {
  constexpr int G = DV / 4;           // float4 column groups per row
  constexpr int R = kThreads / G;     // rows covered per pass
  constexpr int MAXIT = (128 + R - 1) / R;
  const int unit = blockIdx.x;        // n * H + h
  const int dk = p.d_k;
  const int t = threadIdx.x, cg = t % G, rg = t / G;
  const bool scalar_decay = (p.flags & GDN2_SCALAR_DECAY) != 0;
  const bool scalar_gates = (p.flags & GDN2_SCALAR_GATES) != 0;
  const bool tied = (p.flags & GDN2_TIED_GATES) != 0;

  __shared__ float s_a[128], s_k[128], s_x[128], s_p[128], s_q[128];
  __shared__ float s_v[DV];
  __shared__ __align__(16) float red[2][R][DV];
  __shared__ __align__(16) float s_r[DV];
  __shared__ float s_dot[2];

  float *S = p.S + (size_t)unit * dk * DV;

  // Issue the state loads first so their latency overlaps the gate math.
  float4 st[MAXIT];
#pragma unroll
  for (int it = 0; it < MAXIT; ++it) {
    const int i = rg + R * it;
    if (i < dk) st[it] = __ldcs(reinterpret_cast<const float4 *>(S + (size_t)i * DV) + cg);
  }

  const Tin *q = static_cast<const Tin *>(p.q) + (size_t)unit * dk;
  const Tin *k = static_cast<const Tin *>(p.k) + (size_t)unit * dk;
  const Tin *v = static_cast<const Tin *>(p.v) + (size_t)unit * DV;
  const Tin *la = static_cast<const Tin *>(p.log_a);
  const Tin *gb = static_cast<const Tin *>(p.b);
  const Tin *gw = static_cast<const Tin *>(tied ? p.b : p.w);
  if (t < dk) {
    const float kk = to_f32(k[t]);
    const float g = to_f32(scalar_decay ? la[unit] : la[(size_t)unit * dk + t]);
    const float bb = to_f32(scalar_gates ? gb[unit] : gb[(size_t)unit * dk + t]);
    const float ww = to_f32(scalar_gates ? gw[unit] : gw[(size_t)unit * dk + t]);
    s_a[t] = exp_fast(g);
    s_k[t] = kk;
    s_x[t] = bb * kk;
    s_p[t] = ww * kk;
    s_q[t] = to_f32(q[t]);
  }
  if (t < DV) s_v[t] = to_f32(v[t]);
  __syncthreads();

  if (t < 32) {  // q.(b.k) and q.(w.k)
    float dx = 0.f, dp = 0.f;
    for (int i = t; i < dk; i += 32) {
      dx += s_q[i] * s_x[i];
      dp += s_q[i] * s_p[i];
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      dx += __shfl_xor_sync(0xffffffffu, dx, off);
      dp += __shfl_xor_sync(0xffffffffu, dp, off);
    }
    if (t == 0) {
      s_dot[0] = dx;
      s_dot[1] = dp;
    }
  }

  // Decay in registers and accumulate the partial column sums.
  float4 r4 = make_float4(0.f, 0.f, 0.f, 0.f), u4 = r4;
#pragma unroll
  for (int it = 0; it < MAXIT; ++it) {
    const int i = rg + R * it;
    if (i < dk) {
      const float a = s_a[i], kk = s_k[i], qq = s_q[i];
      float4 s = st[it];
      s.x *= a; s.y *= a; s.z *= a; s.w *= a;
      st[it] = s;
      r4.x += s.x * kk; r4.y += s.y * kk; r4.z += s.z * kk; r4.w += s.w * kk;
      u4.x += s.x * qq; u4.y += s.y * qq; u4.z += s.z * qq; u4.w += s.w * qq;
    }
  }
  reinterpret_cast<float4 *>(red[0][rg])[cg] = r4;
  reinterpret_cast<float4 *>(red[1][rg])[cg] = u4;
  __syncthreads();

  if (t < DV) {
    float r = 0.f, u = 0.f;
#pragma unroll
    for (int g = 0; g < R; ++g) {
      r += red[0][g][t];
      u += red[1][g][t];
    }
    s_r[t] = r;
    const float o = u - s_dot[0] * r + s_dot[1] * s_v[t];
    static_cast<Tout *>(p.o)[(size_t)unit * DV + t] = from_f32<Tout>(o);
  }
  __syncthreads();

  const float4 rr = reinterpret_cast<const float4 *>(s_r)[cg];
  const float4 vv = reinterpret_cast<const float4 *>(s_v)[cg];
#pragma unroll
  for (int it = 0; it < MAXIT; ++it) {
    const int i = rg + R * it;
    if (i < dk) {
      const float x = s_x[i], pp = s_p[i];
      float4 s = st[it];
      s.x += pp * vv.x - x * rr.x;
      s.y += pp * vv.y - x * rr.y;
      s.z += pp * vv.z - x * rr.z;
      s.w += pp * vv.w - x * rr.w;
      __stcs(reinterpret_cast<float4 *>(S + (size_t)i * DV) + cg, s);
    }
  }
}

template <int DV>
cudaError_t launch_dv(const DecodeProblem &p, cudaStream_t stream) {
  const unsigned grid = (unsigned)(p.n_seqs * p.n_heads);
  if (grid == 0) return cudaSuccess;
  const bool in_bf = p.dtype_in == GDN2_BF16, out_bf = p.dtype_out == GDN2_BF16;
  if (in_bf && out_bf) decode_kernel<DV, __nv_bfloat16, __nv_bfloat16><<<grid, kThreads, 0, stream>>>(p);
  else if (in_bf) decode_kernel<DV, __nv_bfloat16, float><<<grid, kThreads, 0, stream>>>(p);
  else if (out_bf) decode_kernel<DV, float, __nv_bfloat16><<<grid, kThreads, 0, stream>>>(p);
  else decode_kernel<DV, float, float><<<grid, kThreads, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode(const DecodeProblem &p, cudaStream_t stream) {
  switch (p.d_v) {
    case 16: return launch_dv<16>(p, stream);
    case 32: return launch_dv<32>(p, stream);
    case 64: return launch_dv<64>(p, stream);
    case 128: return launch_dv<128>(p, stream);
    default: return cudaErrorNotSupported;
  }
}

}  // namespace gdn2
