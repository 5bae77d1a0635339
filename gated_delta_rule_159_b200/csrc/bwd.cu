// bwd.cu -- gradients of the Gated DeltaNet-2 recurrence (reverse mode, fp32 on CUDA cores).
//
// The method trains through its chunked form with a gate-aware backward
// (gist.science Methodologie 3; alanhou.org "Core Mechanism"); the pages give
// no formula for it, and the gradient is fixed by the forward.  This file
// computes it token by token in reverse.  With every token in the general form
// (erase read vector y, erase outer factor x, write outer factor p, value z)
//
//   Sbar = Diag(a) S_prev,   r = Sbar^T y,   S = Sbar - x r^T + p z^T,   o = S^T q,
//
// and G the gradient with respect to S (starting from dS_T):
//
//   G += q do^T;  dq = S do;  dp = G z;  dx = -G r;  dz = G^T p;  dr = -G^T x;
//   Gbar = G + y dr^T;  dy = Sbar dr;  dlog_a_i = sum_j Gbar_ij Sbar_ij;  G = Diag(a) Gbar.
//
// Layout of the work: the columns of S evolve independently, so one CTA owns
// a slice of W columns of one (sequence, head) state and thread i owns row i
// of the slice (W fp32 registers).  Row sums over the slice (dq, dp, dx, dy,
// dlog_a) are per-thread; column sums over the rows (r, dz, dr) are warp
// reduce-scatters plus one cross-warp pass through shared memory.
//
// bwd_kernel:    a forward sweep writes the state before every K-th token to
//                the workspace; then, block by block in reverse, the K states
//                of the block are recomputed from their checkpoint into a
//                shared-memory stash and walked backward.  Per-slice row sums
//                go to a partial buffer, dz (complete per slice) to its own.
// finish_kernel: sums the slices and applies the chain rule to the inputs
//                (k, v, log_a, b, w) for both gate placements and the scalar
//                and tied flags, writing the gradients in the output dtype.
#include "common.cuh"
#include "internal.h"

namespace gdn2 {
namespace {

constexpr int kThreads = 128;  // one thread per row of the state (d_k <= 128)
constexpr int kBlock = 4;      // tokens per checkpoint block (the stash holds one block: 2 CTAs per SM)
constexpr int kRows = 5;       // row sums kept per token: dq, dp, dx, dy, dlog_a
#ifndef GDN2_BWD_SLICE
#define GDN2_BWD_SLICE 32
#endif
constexpr int kSlice = GDN2_BWD_SLICE;  // columns of S per CTA (d_v above it is split into slices)
__host__ __device__ constexpr int slice_width(int dv) { return dv < kSlice ? dv : kSlice; }

// Four consecutive floats between memory and a register array without taking
// the array's address (which would move it to local memory).
__device__ __forceinline__ void load4(float *dst, const float *src) {
  const float4 t = *reinterpret_cast<const float4 *>(src);
  dst[0] = t.x; dst[1] = t.y; dst[2] = t.z; dst[3] = t.w;
}
__device__ __forceinline__ void store4(float *dst, const float *src) {
  *reinterpret_cast<float4 *>(dst) = make_float4(src[0], src[1], src[2], src[3]);
}

template <int W>
struct BwdSmem {
  static constexpr int kStride = W + 4;          // row stride of the stash (float4-aligned, conflict-free)
  float stash[kBlock][kThreads * kStride];      // state before each token of the block, [row][col]
  float rowv[kBlock][5][kThreads];              // a, y, x, p, q per token and row
  float z[kBlock][W], r[kBlock][W], dout[kBlock][W];
  float red[kThreads / 32][2 * W];              // per-warp column sums
  float col[2 * W];                             // final column sums
  float ck[kThreads * kStride];                 // next block's checkpoint (cp.async), [row][col]
};

// 16-byte asynchronous global -> shared copy (each thread copies and later reads its own row).
__device__ __forceinline__ void cp_async16(float *dst, const float *src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
               "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// Sum v[0..W) of every thread over the block's rows.  After the warp
// reduce-scatter lane l holds column l % W; warps then meet in shared memory.
// Results land in out[0..W) (and out[W..2W) for the second vector when TWO).
template <int W, bool TWO>
__device__ __forceinline__ void column_sums(float (&v0)[W], float (&v1)[W], BwdSmem<W> &sm, float *out) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int off = W / 2; off >= 1; off >>= 1) {
    const bool up = (lane & off) != 0;
#pragma unroll
    for (int j = 0; j < off; ++j) {
      const float s0 = up ? v0[j] : v0[j + off], k0 = up ? v0[j + off] : v0[j];
      v0[j] = k0 + __shfl_xor_sync(0xffffffffu, s0, off);
      if (TWO) {
        const float s1 = up ? v1[j] : v1[j + off], k1 = up ? v1[j + off] : v1[j];
        v1[j] = k1 + __shfl_xor_sync(0xffffffffu, s1, off);
      }
    }
  }
#pragma unroll
  for (int off = W; off < 32; off <<= 1) {
    v0[0] += __shfl_xor_sync(0xffffffffu, v0[0], off);
    if (TWO) v1[0] += __shfl_xor_sync(0xffffffffu, v1[0], off);
  }
  if (lane < W) {
    sm.red[warp][lane] = v0[0];
    if (TWO) sm.red[warp][W + lane] = v1[0];
  }
  __syncthreads();
  if (threadIdx.x < (TWO ? 2 * W : W)) {
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < kThreads / 32; ++w) s += sm.red[w][threadIdx.x];
    out[threadIdx.x] = s;
  }
  __syncthreads();
}

template <typename Tin>
struct TokenIo {
  const Tin *q, *k, *v, *g, *b, *w;
  bool scalar_decay, scalar_gates, p3;
  int H, dk, dv;
  // Raw inputs of token `tok` (global index) for row i of head h: k, log_a, b, w, q.
  __device__ __forceinline__ void fetch_row(int64_t tok, int h, int i, float (&r)[5]) const {
    const size_t ik = ((size_t)tok * H + h) * dk + i, is = (size_t)tok * H + h;
    r[0] = to_f32(k[ik]);
    r[1] = to_f32(scalar_decay ? g[is] : g[ik]);
    r[2] = to_f32(scalar_gates ? b[is] : b[ik]);
    r[3] = p3 ? 0.f : to_f32(scalar_gates ? w[is] : w[ik]);
    r[4] = to_f32(q[ik]);
  }
  // Row values a, y, x, p, q from the raw inputs.
  __device__ __forceinline__ void row_values(const float (&r)[5], float (&o)[5]) const {
    const float kk = r[0], bb = r[2];
    o[0] = exp_fast(r[1]);
    o[1] = p3 ? bb * kk : kk;
    o[2] = p3 ? kk : bb * kk;
    o[3] = p3 ? kk : r[3] * kk;
    o[4] = r[4];
  }
  // Raw value (and, in the gist.science form, value gate) of column c of token `tok`.
  __device__ __forceinline__ void fetch_col(int64_t tok, int h, int c, float &vv, float &ww) const {
    const size_t iv = ((size_t)tok * H + h) * dv + c;
    vv = to_f32(v[iv]);
    ww = p3 ? to_f32(scalar_gates ? w[(size_t)tok * H + h] : w[iv]) : 1.f;
  }
};

template <int W, typename Tin, typename Tout>
__global__ void __launch_bounds__(kThreads) bwd_kernel(BwdProblem p) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  BwdSmem<W> &sm = *reinterpret_cast<BwdSmem<W> *>(smem_raw);
  constexpr int ST = BwdSmem<W>::kStride;
  const int NS = p.d_v / W;
  const int unit = blockIdx.x / NS, slice = blockIdx.x % NS;
  const int H = p.n_heads, dk = p.d_k, dv = p.d_v;
  const int n = unit / H, h = unit % H;
  const int i = threadIdx.x, c0 = slice * W;
  const bool live = i < dk;
  const bool tied = (p.flags & GDN2_TIED_GATES) != 0;

  TokenIo<Tin> io;
  io.q = static_cast<const Tin *>(p.q);
  io.k = static_cast<const Tin *>(p.k);
  io.v = static_cast<const Tin *>(p.v);
  io.g = static_cast<const Tin *>(p.log_a);
  io.b = static_cast<const Tin *>(p.b);
  io.w = static_cast<const Tin *>(tied ? p.b : p.w);
  io.scalar_decay = (p.flags & GDN2_SCALAR_DECAY) != 0;
  io.scalar_gates = (p.flags & GDN2_SCALAR_GATES) != 0;
  io.p3 = (p.flags & GDN2_GATE_FORM_P3) != 0;
  io.H = H;
  io.dk = dk;
  io.dv = dv;
  const Tout *dO = static_cast<const Tout *>(p.dO);

  int64_t bos, len;
  if (p.cu_seqlens) {
    bos = p.cu_seqlens[n];
    len = p.cu_seqlens[n + 1] - bos;
  } else {
    bos = (int64_t)n * p.seq_len;
    len = p.seq_len;
  }
  const int64_t nblk = (len + kBlock - 1) / kBlock;
  const int64_t slot0 = bos / kBlock + n;  // first checkpoint slot of this sequence
  const size_t D = (size_t)dk * dv;
  auto ckpt = [&](int64_t j) { return p.ckpt + ((size_t)(slot0 + j) * H + h) * D + (size_t)i * dv + c0; };

  float S[W], G[W], t0v[W], t1v[W];
  if (p.S0 && live) {
    const float *s0 = p.S0 + (size_t)unit * D + (size_t)i * dv + c0;
#pragma unroll
    for (int j = 0; j < W; j += 4) load4(S + j, s0 + j);
  } else {
#pragma unroll
    for (int j = 0; j < W; ++j) S[j] = 0.f;
  }

  // One forward token on the registers S; r of the token lands in rout (shared).
  auto fwd_token = [&](float a, float y, float x, float pp, const float *zt, float *rout) {
#pragma unroll
    for (int j = 0; j < W; ++j) {
      S[j] *= a;
      t0v[j] = S[j] * y;
    }
    column_sums<W, false>(t0v, t1v, sm, rout);
#pragma unroll
    for (int j = 0; j < W; ++j) S[j] += pp * zt[j] - x * rout[j];
  };

  // The token values of one block (raw inputs of this thread's row; v, the value
  // gate and dO of this slice's columns) are fetched into registers one block ahead
  // and written to shared memory when the block starts, so the serial token loop
  // waits on no global load.
  float raw[kBlock][5], rvv[kBlock], rww[kBlock], rdo[kBlock];
  auto blk_cnt = [&](int64_t blk) { return (int)((len - blk * kBlock) < kBlock ? (len - blk * kBlock) : kBlock); };
  auto fetch_block = [&](int64_t blk, bool with_dout) {
    const int cnt = blk_cnt(blk);
#pragma unroll
    for (int s = 0; s < kBlock; ++s) {
      raw[s][0] = raw[s][1] = raw[s][2] = raw[s][3] = raw[s][4] = 0.f;
      rvv[s] = rdo[s] = 0.f;
      rww[s] = 1.f;
      if (s < cnt) {
        const int64_t tok = bos + blk * kBlock + s;
        if (live) io.fetch_row(tok, h, i, raw[s]);
        if (i < W) {
          io.fetch_col(tok, h, c0 + i, rvv[s], rww[s]);
          if (with_dout) rdo[s] = to_f32(dO[((size_t)tok * H + h) * dv + c0 + i]);
        }
      }
    }
  };
  auto commit_block = [&]() {
#pragma unroll
    for (int s = 0; s < kBlock; ++s) {
      float o[5];
      io.row_values(raw[s], o);
#pragma unroll
      for (int m = 0; m < 5; ++m) sm.rowv[s][m][i] = o[m];
      if (i < W) {
        sm.z[s][i] = rvv[s] * rww[s];
        sm.dout[s][i] = rdo[s];
      }
    }
  };

  // ---- forward sweep: checkpoints before tokens 0, K, 2K, ...
  if (nblk > 0) fetch_block(0, false);
  for (int64_t blk = 0; blk < nblk; ++blk) {
    if (live) {
      float *cp = ckpt(blk);
#pragma unroll
      for (int j = 0; j < W; j += 4) store4(cp + j, S + j);
    }
    const int cnt = blk_cnt(blk);
    commit_block();
    __syncthreads();
    if (blk + 1 < nblk) fetch_block(blk + 1, false);
    for (int s = 0; s < cnt; ++s)
      fwd_token(sm.rowv[s][0][i], sm.rowv[s][1][i], sm.rowv[s][2][i], sm.rowv[s][3][i], sm.z[s], sm.col);
    __syncthreads();  // the next block rewrites the token values
  }

  // ---- backward, block by block in reverse
  if (p.dS_T && live) {
    const float *g0 = p.dS_T + (size_t)unit * D + (size_t)i * dv + c0;
#pragma unroll
    for (int j = 0; j < W; j += 4) load4(G + j, g0 + j);
  } else {
#pragma unroll
    for (int j = 0; j < W; ++j) G[j] = 0.f;
  }
  // the checkpoint of the next block travels by cp.async into sm.ck (own row only)
  auto fetch_ckpt = [&](int64_t blk) {
    if (live) {
      const float *cp = ckpt(blk);
#pragma unroll
      for (int j = 0; j < W; j += 4) cp_async16(&sm.ck[i * ST + j], cp + j);
    }
    cp_async_commit();
  };
  if (nblk > 0) {
    fetch_block(nblk - 1, true);
    fetch_ckpt(nblk - 1);
  }
  for (int64_t blk = nblk - 1; blk >= 0; --blk) {
    const int cnt = blk_cnt(blk);
    cp_async_wait();
#pragma unroll
    for (int j = 0; j < W; j += 4) load4(S + j, &sm.ck[i * ST + j]);
    commit_block();
    __syncthreads();
    if (blk > 0) {
      fetch_block(blk - 1, true);
      fetch_ckpt(blk - 1);
    }
    // recompute the block, stashing the state before each token (own row only)
    for (int s = 0; s < cnt; ++s) {
#pragma unroll
      for (int j = 0; j < W; j += 4) store4(&sm.stash[s][i * ST + j], S + j);
      fwd_token(sm.rowv[s][0][i], sm.rowv[s][1][i], sm.rowv[s][2][i], sm.rowv[s][3][i], sm.z[s], sm.r[s]);
    }
    // walk it backward
    for (int s = cnt - 1; s >= 0; --s) {
      const int64_t tok = bos + blk * kBlock + s;
      const float a = sm.rowv[s][0][i], y = sm.rowv[s][1][i], x = sm.rowv[s][2][i];
      const float pp = sm.rowv[s][3][i], qq = sm.rowv[s][4][i];
      const float *zt = sm.z[s], *rt = sm.r[s], *dt = sm.dout[s];
      float sbar[W];
      float dq = 0.f, dp = 0.f, dx = 0.f;
#pragma unroll
      for (int j = 0; j < W; j += 4) load4(sbar + j, &sm.stash[s][i * ST + j]);
#pragma unroll
      for (int j = 0; j < W; ++j) {
        sbar[j] *= a;
        const float st = sbar[j] - x * rt[j] + pp * zt[j];  // S after the token
        dq += st * dt[j];
        G[j] += qq * dt[j];
        dp += G[j] * zt[j];
        dx -= G[j] * rt[j];
        t0v[j] = G[j] * pp;   // -> dz
        t1v[j] = -G[j] * x;   // -> dr
      }
      column_sums<W, true>(t0v, t1v, sm, sm.col);
      float dy = 0.f, dg = 0.f;
#pragma unroll
      for (int j = 0; j < W; ++j) {
        const float dr = sm.col[W + j];
        const float gb = G[j] + y * dr;
        dy += sbar[j] * dr;
        dg += gb * sbar[j];
        G[j] = a * gb;
      }
      if (live) {
        float *pr = p.part + (((size_t)slice * p.t_total + tok) * H + h) * kRows * dk + i;
        pr[0 * dk] = dq;
        pr[1 * dk] = dp;
        pr[2 * dk] = dx;
        pr[3 * dk] = dy;
        pr[4 * dk] = dg;
      }
      if (i < W) p.dz[((size_t)tok * H + h) * dv + c0 + i] = sm.col[i];
      // sm.col is next written after the first barrier of the next column sums
    }
    __syncthreads();  // the next block's recompute rewrites the stash and row values
  }
  if (p.dS0 && live) {
    float *g0 = p.dS0 + (size_t)unit * D + (size_t)i * dv + c0;
#pragma unroll
    for (int j = 0; j < W; j += 4) store4(g0 + j, G + j);
  }
}

// Sum of v over the block's 128 threads for NV values at once (result in every thread).
template <int NV>
__device__ __forceinline__ void block_sums(float (&v)[NV], float (*red)[kThreads / 32]) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int u = 0; u < NV; ++u) {
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) v[u] += __shfl_xor_sync(0xffffffffu, v[u], off);
    if (lane == 0) red[u][warp] = v[u];
  }
  __syncthreads();
#pragma unroll
  for (int u = 0; u < NV; ++u) {
    float t = 0.f;
#pragma unroll
    for (int w = 0; w < kThreads / 32; ++w) t += red[u][w];
    v[u] = t;
  }
}

// One CTA per (token, head): sums the slices, applies the chain rule through the
// gate placement (and, with the fused prologue, through the activations).
template <typename Tin, typename Tout>
__global__ void __launch_bounds__(kThreads) finish_kernel(BwdProblem p) {
  __shared__ float red[5][kThreads / 32];
  const int64_t th = blockIdx.x;  // tok * H + h
  const int i = threadIdx.x;
  const int H = p.n_heads, dk = p.d_k, dv = p.d_v, NS = dv / slice_width(dv);
  const bool sd = (p.flags & GDN2_SCALAR_DECAY) != 0, sg = (p.flags & GDN2_SCALAR_GATES) != 0;
  const bool tied = (p.flags & GDN2_TIED_GATES) != 0, p3 = (p.flags & GDN2_GATE_FORM_P3) != 0;
  const bool prolog = p.inv_norm != nullptr;
  (void)H;
  const Tin *k = static_cast<const Tin *>(p.k), *v = static_cast<const Tin *>(p.v);
  const Tin *b = static_cast<const Tin *>(p.b), *w = static_cast<const Tin *>(tied ? p.b : p.w);
  const Tin *q = static_cast<const Tin *>(p.q), *g = static_cast<const Tin *>(p.log_a);
  Tout *dq = static_cast<Tout *>(p.dq), *dkk = static_cast<Tout *>(p.dk), *dvv = static_cast<Tout *>(p.dv);
  Tout *dg = static_cast<Tout *>(p.dlog_a), *db = static_cast<Tout *>(p.db), *dw = static_cast<Tout *>(p.dw);

  float vdq = 0.f, vdp = 0.f, vdx = 0.f, vdy = 0.f, vdg = 0.f;
  if (i < dk) {
    for (int s = 0; s < NS; ++s) {
      const float *pr = p.part + ((size_t)s * p.t_total * p.n_heads + th) * kRows * dk + i;
      vdq += pr[0 * dk];
      vdp += pr[1 * dk];
      vdx += pr[2 * dk];
      vdy += pr[3 * dk];
      vdg += pr[4 * dk];
    }
  }
  // gradients with respect to the (activated) inputs, per row and per column
  float gb = 0.f, gw = 0.f, gdk = 0.f, kk = 0.f, qq = 0.f;
  const size_t ik = (size_t)th * dk + i;
  if (i < dk) {
    kk = to_f32(k[ik]);
    qq = to_f32(q[ik]);
    const float bb = to_f32(sg ? b[th] : b[ik]);
    if (p3) {
      gdk = bb * vdy + vdx + vdp;
      gb = kk * vdy;
    } else {
      const float ww = to_f32(sg ? w[th] : w[ik]);
      gdk = vdy + bb * vdx + ww * vdp;
      gb = kk * vdx;
      gw = kk * vdp;
    }
  }
  float gwv = 0.f;  // P3: v_j dz_j, the value-side write-gate gradient
  if (i < dv) {
    const size_t iv = (size_t)th * dv + i;
    const float dz = p.dz[iv];
    if (p3) {
      const float ww = to_f32(sg ? w[th] : w[iv]);
      dvv[iv] = from_f32<Tout>(ww * dz);
      gwv = to_f32(v[iv]) * dz;
    } else {
      dvv[iv] = from_f32<Tout>(dz);
    }
  }
  // per-channel gate gradient of b (tied gates add the w gradient; P3 tied needs d_k == d_v)
  const float gbt = gb + (tied ? (p3 ? gwv : gw) : 0.f);
  // block sums: channel sums for the scalar flags, q.dq and k.dk for the L2-norm gradient
  float sums[5] = {vdg, gb, p3 ? gwv : gw, qq * vdq, kk * gdk};
  block_sums<5>(sums, red);

  // sigmoid' = s (1 - s) from the activated value s; d/dx log sigmoid(x) = 1 - a
  auto dsig = [&](float s) { return prolog ? s * (1.f - s) : 1.f; };
  if (i < dk) {
    float oq = vdq, ok = gdk;
    if (prolog) {  // y = x / |x|: dx = (dy - y (y . dy)) / |x|
      oq = (vdq - qq * sums[3]) * p.inv_norm[2 * th];
      ok = (gdk - kk * sums[4]) * p.inv_norm[2 * th + 1];
    }
    dq[ik] = from_f32<Tout>(oq);
    dkk[ik] = from_f32<Tout>(ok);
    if (!sd) {
      const float a = prolog ? exp_fast(to_f32(g[ik])) : 0.f;
      dg[ik] = from_f32<Tout>(prolog ? vdg * (1.f - a) : vdg);
    }
    if (!sg) {
      db[ik] = from_f32<Tout>(gbt * dsig(to_f32(b[ik])));
      if (!tied && !p3) dw[ik] = from_f32<Tout>(gw * dsig(to_f32(w[ik])));
    }
  }
  if (!sg && !tied && p3 && i < dv) {
    const size_t iv = (size_t)th * dv + i;
    dw[iv] = from_f32<Tout>(gwv * dsig(to_f32(w[iv])));
  }
  if (i == 0) {
    if (sd) {
      const float a = prolog ? exp_fast(to_f32(g[th])) : 0.f;
      dg[th] = from_f32<Tout>(prolog ? sums[0] * (1.f - a) : sums[0]);
    }
    if (sg) {
      if (tied) {
        db[th] = from_f32<Tout>((sums[1] + sums[2]) * dsig(to_f32(b[th])));
      } else {
        db[th] = from_f32<Tout>(sums[1] * dsig(to_f32(b[th])));
        dw[th] = from_f32<Tout>(sums[2] * dsig(to_f32(w[th])));
      }
    }
  }
}

// Fused prologue: activated fp32 copies of the inputs (and v) for the reverse pass,
// and 1/sqrt(|q|^2 + eps), 1/sqrt(|k|^2 + eps) per (token, head).
template <typename Tin>
__global__ void __launch_bounds__(kThreads) prologue_kernel(BwdProblem p, PrologueCopies c) {
  __shared__ float red[2][kThreads / 32];
  const int64_t th = blockIdx.x;
  const int i = threadIdx.x, dk = p.d_k, dv = p.d_v;
  const bool sd = (p.flags & GDN2_SCALAR_DECAY) != 0, sg = (p.flags & GDN2_SCALAR_GATES) != 0;
  const bool tied = (p.flags & GDN2_TIED_GATES) != 0, p3 = (p.flags & GDN2_GATE_FORM_P3) != 0;
  const Tin *q = static_cast<const Tin *>(p.q), *k = static_cast<const Tin *>(p.k);
  const Tin *v = static_cast<const Tin *>(p.v), *g = static_cast<const Tin *>(p.log_a);
  const Tin *b = static_cast<const Tin *>(p.b), *w = static_cast<const Tin *>(p.w);
  const size_t ik = (size_t)th * dk + i, iv = (size_t)th * dv + i;
  const float qq = i < dk ? to_f32(q[ik]) : 0.f, kk = i < dk ? to_f32(k[ik]) : 0.f;
  float sums[2] = {qq * qq, kk * kk};
  block_sums<2>(sums, red);
  const float iq = rsqrtf(sums[0] + kNormEps), ikn = rsqrtf(sums[1] + kNormEps);
  if (i < dk) {
    c.q[ik] = qq * iq;
    c.k[ik] = kk * ikn;
    if (!sd) c.log_a[ik] = log_sigmoid_f(to_f32(g[ik]));
    if (!sg) {
      c.b[ik] = sigmoid_f(to_f32(b[ik]));
      if (!tied && !p3) c.w[ik] = sigmoid_f(to_f32(w[ik]));
    }
  }
  if (i < dv) {
    c.v[iv] = to_f32(v[iv]);
    if (!sg && !tied && p3) c.w[iv] = sigmoid_f(to_f32(w[iv]));
  }
  if (i == 0) {
    if (sd) c.log_a[th] = log_sigmoid_f(to_f32(g[th]));
    if (sg) {
      c.b[th] = sigmoid_f(to_f32(b[th]));
      if (!tied) c.w[th] = sigmoid_f(to_f32(w[th]));
    }
    c.inv_norm[2 * th] = iq;
    c.inv_norm[2 * th + 1] = ikn;
  }
}

template <int W, typename Tin, typename Tout>
cudaError_t launch_w(const BwdProblem &p, cudaStream_t stream) {
  const unsigned units = (unsigned)(p.n_seqs * p.n_heads);
  if (units > 0) {
    auto kern = bwd_kernel<W, Tin, Tout>;
    const int smem = (int)sizeof(BwdSmem<W>);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    kern<<<units * (unsigned)(p.d_v / W), kThreads, smem, stream>>>(p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  const int64_t rows = p.t_total * p.n_heads;
  if (rows > 0) {
    finish_kernel<Tin, Tout><<<(unsigned)rows, kThreads, 0, stream>>>(p);
    return cudaGetLastError();
  }
  return cudaSuccess;
}

template <typename Tin, typename Tout>
cudaError_t launch_types(const BwdProblem &p, cudaStream_t stream) {
  switch (p.d_v) {
    case 16: return launch_w<slice_width(16), Tin, Tout>(p, stream);
    case 32: return launch_w<slice_width(32), Tin, Tout>(p, stream);
    case 64: return launch_w<slice_width(64), Tin, Tout>(p, stream);
    case 128: return launch_w<slice_width(128), Tin, Tout>(p, stream);
    default: return cudaErrorNotSupported;
  }
}

}  // namespace

namespace {
// fp32 copies q, k, log_a, b (d_k channels), w (max(d_k, d_v)), v (d_v), 2 norms per (token, head)
size_t prologue_floats(int64_t rows, int d_k, int d_v) {
  return (size_t)rows * (4 * (size_t)d_k + (size_t)(d_k > d_v ? d_k : d_v) + d_v + 2);
}
PrologueCopies carve_prologue(float *base, int64_t rows, int d_k, int d_v) {
  PrologueCopies c;
  const size_t dkn = (size_t)rows * d_k, dvn = (size_t)rows * d_v;
  const size_t wn = (size_t)rows * (d_k > d_v ? d_k : d_v);
  c.q = base;
  c.k = c.q + dkn;
  c.log_a = c.k + dkn;
  c.b = c.log_a + dkn;
  c.w = c.b + dkn;
  c.v = c.w + wn;
  c.inv_norm = c.v + dvn;
  return c;
}
}  // namespace

size_t bwd_workspace_bytes(int64_t n_seqs, int64_t t_total, int n_heads, int d_k, int d_v, uint32_t flags) {
  const int W = slice_width(d_v);
  const size_t slots = (size_t)(t_total / kBlock + n_seqs);
  const size_t ckpt = slots * n_heads * (size_t)d_k * d_v * sizeof(float);
  const size_t part = (size_t)(d_v / W) * t_total * n_heads * kRows * (size_t)d_k * sizeof(float);
  const size_t dz = (size_t)t_total * n_heads * d_v * sizeof(float);
  const size_t pro = (flags & GDN2_FUSED_PROLOGUE) ? prologue_floats(t_total * n_heads, d_k, d_v) * sizeof(float) : 0;
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  return up(ckpt) + up(part) + up(dz) + up(pro);
}

void bwd_carve(BwdProblem &p, void *workspace) {
  const int W = slice_width(p.d_v);
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  const size_t slots = (size_t)(p.t_total / kBlock + p.n_seqs);
  char *base = static_cast<char *>(workspace);
  p.ckpt = reinterpret_cast<float *>(base);
  base += up(slots * p.n_heads * (size_t)p.d_k * p.d_v * sizeof(float));
  p.part = reinterpret_cast<float *>(base);
  base += up((size_t)(p.d_v / W) * p.t_total * p.n_heads * kRows * (size_t)p.d_k * sizeof(float));
  p.dz = reinterpret_cast<float *>(base);
  base += up((size_t)p.t_total * p.n_heads * p.d_v * sizeof(float));
  p.prolog = (p.flags & GDN2_FUSED_PROLOGUE) ? reinterpret_cast<float *>(base) : nullptr;
  p.inv_norm = nullptr;
}

cudaError_t launch_bwd(const BwdProblem &p, cudaStream_t stream) {
  const bool in_bf = p.dtype_in == GDN2_BF16, out_bf = p.dtype_out == GDN2_BF16;
  if (p.prolog) {
    // activate into fp32 copies, then run the reverse pass on them; finish_kernel
    // applies the activations' chain rule (it sees inv_norm != NULL)
    const int64_t rows = p.t_total * p.n_heads;
    const PrologueCopies c = carve_prologue(p.prolog, rows, p.d_k, p.d_v);
    if (rows > 0) {
      if (in_bf) prologue_kernel<__nv_bfloat16><<<(unsigned)rows, kThreads, 0, stream>>>(p, c);
      else prologue_kernel<float><<<(unsigned)rows, kThreads, 0, stream>>>(p, c);
      const cudaError_t e = cudaGetLastError();
      if (e != cudaSuccess) return e;
    }
    BwdProblem a = p;
    a.q = c.q; a.k = c.k; a.v = c.v; a.log_a = c.log_a; a.b = c.b;
    a.w = (p.flags & GDN2_TIED_GATES) ? nullptr : c.w;
    a.inv_norm = c.inv_norm;
    a.prolog = nullptr;
    a.dtype_in = GDN2_F32;
    return out_bf ? launch_types<float, __nv_bfloat16>(a, stream) : launch_types<float, float>(a, stream);
  }
  if (in_bf && out_bf) return launch_types<__nv_bfloat16, __nv_bfloat16>(p, stream);
  if (in_bf) return launch_types<__nv_bfloat16, float>(p, stream);
  if (out_bf) return launch_types<float, __nv_bfloat16>(p, stream);
  return launch_types<float, float>(p, stream);
}

}  // namespace gdn2
