// chunk_simt.cu -- chunked Gated DeltaNet-2 forward for small heads (d_k, d_v <= 64),
// fp32 arithmetic on CUDA cores.
//
// Same chunk algebra as the tensor-core path (alanhou.org "Core Mechanism": a
// chunkwise WY form; gist.science Methodologie 3: a lower-triangular solve
// gives the erase-side auxiliaries), written for one chunk of rows i, j < n
// starting from state S, with y the erase read vector, x the erase outer
// factor, p the write outer factor, V the written values (k, b.k, w.k, v by
// default; b.k, k, k, w.v in the gist.science form) and L the inclusive
// cumulative log-decay inside the chunk:
//
//   A_ij  = sum_c y_ic x_jc e^{L_ic - L_jc}   (j < i)     B_ij  = same with p
//   QX_ij = sum_c q_ic x_jc e^{L_ic - L_jc}   (j <= i)    QP_ij = same with p
//   M     = (I + A)^-1 (Ytilde S + B V),      Ytilde_ic = y_ic e^{L_ic}
//   O     = Qtilde S + QP V - QX M,           Qtilde_ic = q_ic e^{L_ic}
//   S'    = Diag(e^{L_C}) S + sum_j Diag(e^{L_C - L_j}) (p_j v_j^T - x_j M_j^T)
//
// Here the decay factors are formed pairwise and exactly (every exponent is
// <= 0), so this path has no range precondition; (I + A)^-1 is applied by
// forward substitution, one M column per thread.  One CTA per (sequence, head).
#include "common.cuh"
#include "internal.h"

namespace gdn2 {
namespace {

constexpr int kThreads = 256;

template <typename Tin, typename Tout>
__global__ void __launch_bounds__(kThreads) chunk_simt_kernel(ChunkProblem p) {
  extern __shared__ float smem[];
  const int dk = p.d_k, dv = p.d_v, C = p.chunk, H = p.n_heads;
  const int unit = blockIdx.x;
  const int n = unit / H, h = unit % H;
  const int tid = threadIdx.x;
  const bool scalar_decay = (p.flags & GDN2_SCALAR_DECAY) != 0;
  const bool scalar_gates = (p.flags & GDN2_SCALAR_GATES) != 0;
  const bool tied = (p.flags & GDN2_TIED_GATES) != 0;
  const bool p3 = (p.flags & GDN2_GATE_FORM_P3) != 0;
  const bool prolog = (p.flags & GDN2_FUSED_PROLOGUE) != 0;

  int64_t bos, len;
  if (p.cu_seqlens) {
    bos = p.cu_seqlens[n];
    len = p.cu_seqlens[n + 1] - bos;
  } else {
    bos = (int64_t)n * p.seq_len;
    len = p.seq_len;
  }

  float *S = smem;                 // [dk][dv]
  float *sq = S + dk * dv;         // [C][dk]
  float *sk = sq + C * dk;         // [C][dk]
  float *sx = sk + C * dk;         // [C][dk]  b.k
  float *sp = sx + C * dk;         // [C][dk]  w.k
  float *sL = sp + C * dk;         // [C][dk]  cumulative log-decay, then e^{L}
  float *sF = sL + C * dk;         // [C][dk]  log_a, then e^{L_C - L}
  float *sv = sF + C * dk;         // [C][dv]
  float *sA = sv + C * dv;         // [C][C]
  float *sB = sA + C * C;
  float *sQX = sB + C * C;
  float *sQP = sQX + C * C;
  float *sM = sQP + C * C;         // [C][dv]

  const float *S0 = p.S0 ? p.S0 + (size_t)unit * dk * dv : nullptr;
  for (int e = tid; e < dk * dv; e += kThreads) S[e] = S0 ? S0[e] : 0.f;

  const Tin *gq = static_cast<const Tin *>(p.q);
  const Tin *gk = static_cast<const Tin *>(p.k);
  const Tin *gv = static_cast<const Tin *>(p.v);
  const Tin *ga = static_cast<const Tin *>(p.log_a);
  const Tin *gb = static_cast<const Tin *>(p.b);
  const Tin *gw = static_cast<const Tin *>(tied ? p.b : p.w);
  Tout *go = static_cast<Tout *>(p.o);

  for (int64_t c0 = 0; c0 < len; c0 += C) {
    const int nr = (int)((len - c0) < C ? (len - c0) : C);
    __syncthreads();
    // 1. load the chunk (rows >= nr are zero: no decay, no key, no gates)
    for (int e = tid; e < C * dk; e += kThreads) {
      const int r = e / dk, c = e % dk;
      float qq = 0.f, kk = 0.f, g = 0.f, bb = 0.f, ww = 0.f;
      if (r < nr) {
        const int64_t tok = bos + c0 + r;
        const size_t ik = ((size_t)tok * H + h) * dk + c;
        const size_t is = (size_t)tok * H + h;
        qq = to_f32(gq[ik]);
        kk = to_f32(gk[ik]);
        g = to_f32(scalar_decay ? ga[is] : ga[ik]);
        bb = to_f32(scalar_gates ? gb[is] : gb[ik]);
        if (!p3) ww = to_f32(scalar_gates ? gw[is] : gw[ik]);
        if (prolog) {
          g = log_sigmoid_f(g);
          bb = sigmoid_f(bb);
          ww = sigmoid_f(ww);
        }
      }
      // sk: erase read vector, sx: erase outer factor, sp: write outer factor.
      // Default form (k, b.k, w.k); gist.science form (b.k, k, k), whose write
      // gate scales the values below instead.
      sq[e] = qq;
      sk[e] = p3 ? bb * kk : kk;
      sx[e] = p3 ? kk : bb * kk;
      sp[e] = p3 ? kk : ww * kk;
      sF[e] = g;
    }
    for (int e = tid; e < C * dv; e += kThreads) {
      const int r = e / dv, c = e % dv;
      float vv = 0.f;
      if (r < nr) {
        const int64_t tok = bos + c0 + r;
        vv = to_f32(gv[((size_t)tok * H + h) * dv + c]);
        if (p3) {
          float ww = to_f32(scalar_gates ? gw[(size_t)tok * H + h] : gw[((size_t)tok * H + h) * dv + c]);
          if (prolog) ww = sigmoid_f(ww);
          vv *= ww;
        }
      }
      sv[e] = vv;
    }
    __syncthreads();
    if (prolog) {  // L2 norms of the q and k rows (one row per thread); sk, sx, sp are all proportional to k
      const float *kraw = p3 ? sx : sk;
      if (tid < C) {
        float qq = 0.f, kk = 0.f;
        for (int c = 0; c < dk; ++c) {
          qq += sq[tid * dk + c] * sq[tid * dk + c];
          kk += kraw[tid * dk + c] * kraw[tid * dk + c];
        }
        const float iq = rsqrtf(qq + kNormEps), ik = rsqrtf(kk + kNormEps);
        for (int c = 0; c < dk; ++c) {
          sq[tid * dk + c] *= iq;
          sk[tid * dk + c] *= ik;
          sx[tid * dk + c] *= ik;
          sp[tid * dk + c] *= ik;
        }
      }
      __syncthreads();
    }
    // 2. inclusive cumulative log-decay per channel
    if (tid < dk) {
      float acc = 0.f;
      for (int r = 0; r < C; ++r) {
        acc += sF[r * dk + tid];
        sL[r * dk + tid] = acc;
      }
    }
    __syncthreads();
    // 3. pairwise interaction matrices with exact decay factors
    for (int e = tid; e < C * C; e += kThreads) {
      const int i = e / C, j = e % C;
      float a = 0.f, bb = 0.f, qx = 0.f, qp = 0.f;
      if (j <= i) {
        for (int c = 0; c < dk; ++c) {
          const float d = exp_fast(sL[i * dk + c] - sL[j * dk + c]);
          const float kd = sk[i * dk + c] * d, qd = sq[i * dk + c] * d;
          a += kd * sx[j * dk + c];
          bb += kd * sp[j * dk + c];
          qx += qd * sx[j * dk + c];
          qp += qd * sp[j * dk + c];
        }
      }
      sA[e] = j < i ? a : 0.f;
      sB[e] = j < i ? bb : 0.f;
      sQX[e] = qx;
      sQP[e] = qp;
    }
    __syncthreads();
    // decay factors relative to the chunk end (e^{L_C - L}) and to its start (e^{L});
    // two passes, since every row reads the last row's L_C before sL is overwritten
    for (int e = tid; e < C * dk; e += kThreads) {
      const int c = e % dk;
      sF[e] = exp_fast(sL[(C - 1) * dk + c] - sL[e]);
    }
    __syncthreads();
    for (int e = tid; e < C * dk; e += kThreads) sL[e] = exp_fast(sL[e]);
    __syncthreads();
    // 4. right-hand side Ytilde S + B V
    for (int e = tid; e < C * dv; e += kThreads) {
      const int i = e / dv, d = e % dv;
      float acc = 0.f;
      for (int c = 0; c < dk; ++c) acc += sk[i * dk + c] * sL[i * dk + c] * S[c * dv + d];
      for (int j = 0; j < i; ++j) acc += sB[i * C + j] * sv[j * dv + d];
      sM[e] = acc;
    }
    __syncthreads();
    // 5. forward substitution (I + A) M = rhs, one column per thread
    if (tid < dv) {
      for (int i = 1; i < C; ++i) {
        float acc = sM[i * dv + tid];
        for (int j = 0; j < i; ++j) acc -= sA[i * C + j] * sM[j * dv + tid];
        sM[i * dv + tid] = acc;
      }
    }
    __syncthreads();
    // 6. outputs
    for (int e = tid; e < nr * dv; e += kThreads) {
      const int i = e / dv, d = e % dv;
      float acc = 0.f;
      for (int c = 0; c < dk; ++c) acc += sq[i * dk + c] * sL[i * dk + c] * S[c * dv + d];
      for (int j = 0; j <= i; ++j) acc += sQP[i * C + j] * sv[j * dv + d] - sQX[i * C + j] * sM[j * dv + d];
      go[((size_t)(bos + c0 + i) * H + h) * dv + d] = from_f32<Tout>(acc);
    }
    __syncthreads();  // every output has read S before the update below overwrites it
    // 7. state update (each thread reads and writes only its own S elements)
    for (int e = tid; e < dk * dv; e += kThreads) {
      const int c = e / dv, d = e % dv;
      float acc = sL[(C - 1) * dk + c] * S[e];
      for (int j = 0; j < nr; ++j)
        acc += sF[j * dk + c] * (sp[j * dk + c] * sv[j * dv + d] - sx[j * dk + c] * sM[j * dv + d]);
      S[e] = acc;
    }
  }
  __syncthreads();
  if (p.S_T) {
    float *ST = p.S_T + (size_t)unit * dk * dv;
    for (int e = tid; e < dk * dv; e += kThreads) ST[e] = S[e];
  }
}

}  // namespace

cudaError_t launch_chunk_simt(const ChunkProblem &p, cudaStream_t stream) {
  const int dk = p.d_k, dv = p.d_v, C = p.chunk;
  const size_t smem = sizeof(float) * ((size_t)dk * dv + 6 * (size_t)C * dk + 2 * (size_t)C * dv + 4 * (size_t)C * C);
  const unsigned grid = (unsigned)(p.n_seqs * p.n_heads);
  if (grid == 0) return cudaSuccess;
  const bool in_bf = p.dtype_in == GDN2_BF16, out_bf = p.dtype_out == GDN2_BF16;
  auto go = [&](auto kern) -> cudaError_t {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<grid, kThreads, smem, stream>>>(p);
    return cudaGetLastError();
  };
  if (in_bf && out_bf) return go(chunk_simt_kernel<__nv_bfloat16, __nv_bfloat16>);
  if (in_bf) return go(chunk_simt_kernel<__nv_bfloat16, float>);
  if (out_bf) return go(chunk_simt_kernel<float, __nv_bfloat16>);
  return go(chunk_simt_kernel<float, float>);
}

}  // namespace gdn2
