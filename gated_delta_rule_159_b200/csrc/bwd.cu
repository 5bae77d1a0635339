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
// Layout of the work: the columns of S evolve independently, so one CTA of four
// warps owns a slice of W columns of one (sequence, head) state; warp w owns W/4
// of those columns and lane l rows 4l .. 4l + 3 of them.  Every column sum of the
// recurrence (r, dz, dr) is then a sum over the 128 rows held by one warp (warp
// shuffles only), so the serial token loop has no block-wide barrier.  The row
// sums (dq, dp, dx, dy, dlog_a) are outputs only: each warp leaves its share in
// shared memory and they are added up once per block of tokens.
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

// 16-byte asynchronous global -> shared copy.
__device__ __forceinline__ void cp_async16(float *dst, const float *src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
               "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// Per-thread block of the state: 4 rows x CW columns, CW = W / 4 (the warp's columns).
// Shared buffers that hold one such block per thread are float4-interleaved by thread
// ([vec4][thread][4]): conflict-free, no padding.
template <int W>
struct BwdSmem {
  static constexpr int CW = W / 4, E = 4 * CW, NV = E / 4;
  static constexpr int NVS = NV > 5 ? NV : 5;  // a slot also holds the 20 row partials of a token
  float stash[kBlock][NVS][kThreads][4];  // state before each token of the block; then the row partials
  float ck[NV][kThreads][4];             // next block's checkpoint (cp.async)
  float rowv[kBlock][5][kThreads];       // a, y, x, p, q per token and row
  float z[kBlock][W], dout[kBlock][W], r[kBlock][W];
};

// Sums over the warp's 32 lanes of CW per-lane values; every lane receives all CW sums.
// Reduce-scatter inside groups of CW lanes, add across the groups, gather back.
template <int CW>
__device__ __forceinline__ void warp_colsum(float (&v)[CW], float (&out)[CW]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int off = CW / 2; off >= 1; off >>= 1) {
    const bool up = (lane & off) != 0;
#pragma unroll
    for (int j = 0; j < off; ++j) {
      const float send = up ? v[j] : v[j + off], keep = up ? v[j + off] : v[j];
      v[j] = keep + __shfl_xor_sync(0xffffffffu, send, off);
    }
  }
#pragma unroll
  for (int off = CW; off < 32; off <<= 1) v[0] += __shfl_xor_sync(0xffffffffu, v[0], off);
  // lane l now holds column l % CW
#pragma unroll
  for (int c = 0; c < CW; ++c) out[c] = __shfl_sync(0xffffffffu, v[0], c);
}

template <typename Tin>
struct TokenIo {
  const Tin *q, *k, *v, *g, *b, *w;
  bool scalar_decay, scalar_gates, p3;
  int H, dk, dv;
  // Raw inputs of token `tok` (global index) for row i of head h: k, log_a, b, w, q,
  // kept in the input type: converting them here would wait for the loads at once.
  __device__ __forceinline__ void fetch_row(int64_t tok, int h, int i, Tin (&r)[5]) const {
    const size_t ik = ((size_t)tok * H + h) * dk + i, is = (size_t)tok * H + h;
    r[0] = k[ik];
    r[1] = scalar_decay ? g[is] : g[ik];
    r[2] = scalar_gates ? b[is] : b[ik];
    r[3] = p3 ? r[0] : (scalar_gates ? w[is] : w[ik]);
    r[4] = q[ik];
  }
  // Row values a, y, x, p, q from the raw inputs.
  __device__ __forceinline__ void row_values(const Tin (&r)[5], float (&o)[5]) const {
    const float kk = to_f32(r[0]), bb = to_f32(r[2]);
    o[0] = exp_fast(to_f32(r[1]));
    o[1] = p3 ? bb * kk : kk;
    o[2] = p3 ? kk : bb * kk;
    o[3] = p3 ? kk : to_f32(r[3]) * kk;
    o[4] = to_f32(r[4]);
  }
  // Raw value (and, in the gist.science form, value gate) of column c of token `tok`.
  __device__ __forceinline__ void fetch_col(int64_t tok, int h, int c, Tin &vv, Tin &ww) const {
    const size_t iv = ((size_t)tok * H + h) * dv + c;
    vv = v[iv];
    ww = p3 ? (scalar_gates ? w[(size_t)tok * H + h] : w[iv]) : vv;
  }
};

template <int W, typename Tin, typename Tout>
__global__ void __launch_bounds__(kThreads) bwd_kernel(BwdProblem p) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  BwdSmem<W> &sm = *reinterpret_cast<BwdSmem<W> *>(smem_raw);
  constexpr int CW = BwdSmem<W>::CW, NV = BwdSmem<W>::NV;
  const int NS = p.d_v / W;
  const int unit = blockIdx.x / NS, slice = blockIdx.x % NS;
  const int H = p.n_heads, dk = p.d_k, dv = p.d_v;
  const int n = unit / H, h = unit % H;
  const int i = threadIdx.x, lane = i & 31, warp = i >> 5;
  const int c0 = slice * W;                     // first column of the CTA's slice
  const int cw0 = warp * CW;                    // the warp's columns inside the slice
  const int r0 = 4 * lane;                      // this thread's rows r0 .. r0 + 3
  const bool live = i < dk;                     // row i, for the per-row loads
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
  // element (row r0 + rr, column c0 + cw0 .. + CW) of a [dk][dv] matrix
  auto at = [&](const float *base, int rr) { return base + (size_t)(r0 + rr) * dv + c0 + cw0; };
  auto atw = [&](float *base, int rr) { return base + (size_t)(r0 + rr) * dv + c0 + cw0; };
  auto ckpt = [&](int64_t j) { return p.ckpt + ((size_t)(slot0 + j) * H + h) * D; };

  float S[4][CW], G[4][CW];
  auto load_state = [&](const float *base) {  // zero for rows past d_k or a NULL base
#pragma unroll
    for (int rr = 0; rr < 4; ++rr)
#pragma unroll
      for (int c = 0; c < CW; c += 4) {
        if (base && r0 + rr < dk) load4(&S[rr][c], at(base, rr) + c);
        else S[rr][c] = S[rr][c + 1] = S[rr][c + 2] = S[rr][c + 3] = 0.f;
      }
  };
  load_state(p.S0 ? p.S0 + (size_t)unit * D : nullptr);

  // One forward token on the registers S: Sbar = a S, r = Sbar^T y (warp column sums),
  // S = Sbar - x r^T + p z^T.  r is returned for the caller to keep.
  auto fwd_token = [&](int s, float (&rr_out)[CW]) {
    const float4 a = *reinterpret_cast<const float4 *>(&sm.rowv[s][0][r0]);
    const float4 y = *reinterpret_cast<const float4 *>(&sm.rowv[s][1][r0]);
    const float4 x = *reinterpret_cast<const float4 *>(&sm.rowv[s][2][r0]);
    const float4 pp = *reinterpret_cast<const float4 *>(&sm.rowv[s][3][r0]);
    const float av[4] = {a.x, a.y, a.z, a.w}, yv[4] = {y.x, y.y, y.z, y.w};
    const float xv[4] = {x.x, x.y, x.z, x.w}, pv[4] = {pp.x, pp.y, pp.z, pp.w};
    float part[CW], zc[CW];
#pragma unroll
    for (int c = 0; c < CW; ++c) {
      zc[c] = sm.z[s][cw0 + c];
      part[c] = 0.f;
    }
#pragma unroll
    for (int rr = 0; rr < 4; ++rr)
#pragma unroll
      for (int c = 0; c < CW; ++c) {
        S[rr][c] *= av[rr];
        part[c] += S[rr][c] * yv[rr];
      }
    warp_colsum<CW>(part, rr_out);
#pragma unroll
    for (int rr = 0; rr < 4; ++rr)
#pragma unroll
      for (int c = 0; c < CW; ++c) S[rr][c] += pv[rr] * zc[c] - xv[rr] * rr_out[c];
  };

  // The token values of one block (raw inputs of row i; v, the value gate and dO of
  // the slice's columns) are fetched into registers one block ahead and written to
  // shared memory when the block starts.
  Tin raw[kBlock][5], rvv[kBlock], rww[kBlock];
  Tout rdo[kBlock];
  auto blk_cnt = [&](int64_t blk) { return (int)((len - blk * kBlock) < kBlock ? (len - blk * kBlock) : kBlock); };
  auto fetch_block = [&](int64_t blk, bool with_dout) {
    const int cnt = blk_cnt(blk);
#pragma unroll
    for (int s = 0; s < kBlock; ++s) {
      raw[s][0] = raw[s][1] = raw[s][2] = raw[s][3] = raw[s][4] = from_f32<Tin>(0.f);
      rvv[s] = rww[s] = from_f32<Tin>(0.f);
      rdo[s] = from_f32<Tout>(0.f);
      if (s < cnt) {
        const int64_t tok = bos + blk * kBlock + s;
        if (live) io.fetch_row(tok, h, i, raw[s]);
        if (i < W) {
          io.fetch_col(tok, h, c0 + i, rvv[s], rww[s]);
          if (with_dout) rdo[s] = dO[((size_t)tok * H + h) * dv + c0 + i];
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
        sm.z[s][i] = io.p3 ? to_f32(rvv[s]) * to_f32(rww[s]) : to_f32(rvv[s]);
        sm.dout[s][i] = to_f32(rdo[s]);
      }
    }
  };

  // ---- forward sweep: checkpoints before tokens 0, K, 2K, ...
  if (nblk > 0) fetch_block(0, false);
  for (int64_t blk = 0; blk < nblk; ++blk) {
#pragma unroll
    for (int rr = 0; rr < 4; ++rr)
      if (r0 + rr < dk)
#pragma unroll
        for (int c = 0; c < CW; c += 4) store4(atw(ckpt(blk), rr) + c, &S[rr][c]);
    const int cnt = blk_cnt(blk);
    commit_block();
    __syncthreads();
    if (blk + 1 < nblk) fetch_block(blk + 1, false);
    for (int s = 0; s < cnt; ++s) {
      float rr_out[CW];
      fwd_token(s, rr_out);
    }
    __syncthreads();  // the next block rewrites the token values
  }

  // ---- backward, block by block in reverse
#pragma unroll
  for (int rr = 0; rr < 4; ++rr)
#pragma unroll
    for (int c = 0; c < CW; c += 4) {
      if (p.dS_T && r0 + rr < dk) load4(&G[rr][c], at(p.dS_T + (size_t)unit * D, rr) + c);
      else G[rr][c] = G[rr][c + 1] = G[rr][c + 2] = G[rr][c + 3] = 0.f;
    }
  // the checkpoint of the next block travels by cp.async into sm.ck (own elements only)
  auto fetch_ckpt = [&](int64_t blk) {
#pragma unroll
    for (int rr = 0; rr < 4; ++rr)
      if (r0 + rr < dk)
#pragma unroll
        for (int c = 0; c < CW; c += 4) cp_async16(sm.ck[(rr * CW + c) / 4][i], atw(ckpt(blk), rr) + c);
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
    for (int rr = 0; rr < 4; ++rr)
#pragma unroll
      for (int c = 0; c < CW; c += 4) {
        if (r0 + rr < dk) load4(&S[rr][c], sm.ck[(rr * CW + c) / 4][i]);
        else S[rr][c] = S[rr][c + 1] = S[rr][c + 2] = S[rr][c + 3] = 0.f;
      }
    commit_block();
    __syncthreads();
    if (blk > 0) {
      fetch_block(blk - 1, true);
      fetch_ckpt(blk - 1);
    }
    // recompute the block, stashing the state before each token (own elements only);
    // the warp keeps each token's r for its columns
    for (int s = 0; s < cnt; ++s) {
#pragma unroll
      for (int v4 = 0; v4 < NV; ++v4) store4(sm.stash[s][v4][i], &S[(4 * v4) / CW][(4 * v4) % CW]);
      float rr_out[CW];
      fwd_token(s, rr_out);
      if (lane == 0)
#pragma unroll
        for (int c = 0; c < CW; ++c) sm.r[s][cw0 + c] = rr_out[c];
    }
    __syncwarp();
    // walk it backward
    for (int s = cnt - 1; s >= 0; --s) {
      const float4 a4 = *reinterpret_cast<const float4 *>(&sm.rowv[s][0][r0]);
      const float4 y4 = *reinterpret_cast<const float4 *>(&sm.rowv[s][1][r0]);
      const float4 x4 = *reinterpret_cast<const float4 *>(&sm.rowv[s][2][r0]);
      const float4 p4 = *reinterpret_cast<const float4 *>(&sm.rowv[s][3][r0]);
      const float4 q4 = *reinterpret_cast<const float4 *>(&sm.rowv[s][4][r0]);
      const float av[4] = {a4.x, a4.y, a4.z, a4.w}, yv[4] = {y4.x, y4.y, y4.z, y4.w};
      const float xv[4] = {x4.x, x4.y, x4.z, x4.w}, pv[4] = {p4.x, p4.y, p4.z, p4.w};
      const float qv[4] = {q4.x, q4.y, q4.z, q4.w};
      float zc[CW], rc[CW], dc[CW];
#pragma unroll
      for (int c = 0; c < CW; ++c) {
        zc[c] = sm.z[s][cw0 + c];
        rc[c] = sm.r[s][cw0 + c];
        dc[c] = sm.dout[s][cw0 + c];
      }
      float sb[4][CW];
#pragma unroll
      for (int v4 = 0; v4 < NV; ++v4) load4(&sb[(4 * v4) / CW][(4 * v4) % CW], sm.stash[s][v4][i]);
      float dq[4], dp[4], dx[4], colA[CW], colB[CW];
#pragma unroll
      for (int c = 0; c < CW; ++c) colA[c] = colB[c] = 0.f;
#pragma unroll
      for (int rr = 0; rr < 4; ++rr) {
        dq[rr] = dp[rr] = dx[rr] = 0.f;
#pragma unroll
        for (int c = 0; c < CW; ++c) {
          sb[rr][c] *= av[rr];
          const float st = sb[rr][c] - xv[rr] * rc[c] + pv[rr] * zc[c];  // S after the token
          dq[rr] += st * dc[c];
          G[rr][c] += qv[rr] * dc[c];
          dp[rr] += G[rr][c] * zc[c];
          dx[rr] -= G[rr][c] * rc[c];
          colA[c] += G[rr][c] * pv[rr];  // -> dz
          colB[c] -= G[rr][c] * xv[rr];  // -> dr
        }
      }
      float dz[CW], dr[CW];
      warp_colsum<CW>(colA, dz);
      warp_colsum<CW>(colB, dr);
      float dy[4], dg[4];
#pragma unroll
      for (int rr = 0; rr < 4; ++rr) {
        dy[rr] = dg[rr] = 0.f;
#pragma unroll
        for (int c = 0; c < CW; ++c) {
          const float gb = G[rr][c] + yv[rr] * dr[c];
          dy[rr] += sb[rr][c] * dr[c];
          dg[rr] += gb * sb[rr][c];
          G[rr][c] = av[rr] * gb;
        }
      }
      // this warp's share of the row sums, into the thread's own (now free) stash slot:
      // element 5 rr + m of rows r0 + rr, m = dq, dp, dx, dy, dlog_a
      float rowp[20];
#pragma unroll
      for (int rr = 0; rr < 4; ++rr) {
        rowp[5 * rr + 0] = dq[rr];
        rowp[5 * rr + 1] = dp[rr];
        rowp[5 * rr + 2] = dx[rr];
        rowp[5 * rr + 3] = dy[rr];
        rowp[5 * rr + 4] = dg[rr];
      }
#pragma unroll
      for (int v4 = 0; v4 < 5; ++v4) store4(sm.stash[s][v4][i], &rowp[4 * v4]);
      if (lane == 0) {
        const int64_t tok = bos + blk * kBlock + s;
        float *dzp = p.dz + ((size_t)tok * H + h) * dv + c0 + cw0;
#pragma unroll
        for (int c = 0; c < CW; c += 4) store4(dzp + c, &dz[c]);
      }
    }
    __syncthreads();
    // add the four warps' row sums of each token (thread i: row i)
    if (live) {
      const int tr = i >> 2, e0 = 5 * (i & 3);  // lane holding row i in every warp, element base
      for (int s = 0; s < cnt; ++s) {
        const int64_t tok = bos + blk * kBlock + s;
        float *pr = p.part + (((size_t)slice * p.t_total + tok) * H + h) * kRows * dk + i;
#pragma unroll
        for (int m = 0; m < kRows; ++m) {
          const int e = e0 + m;
          float acc = 0.f;
#pragma unroll
          for (int w = 0; w < kThreads / 32; ++w) acc += sm.stash[s][e / 4][w * 32 + tr][e % 4];
          pr[m * dk] = acc;
        }
      }
    }
    __syncthreads();  // the next block rewrites the stash and the token values
  }
#pragma unroll
  for (int rr = 0; rr < 4; ++rr)
    if (p.dS0 && r0 + rr < dk)
#pragma unroll
      for (int c = 0; c < CW; c += 4) store4(atw(p.dS0 + (size_t)unit * D, rr) + c, &G[rr][c]);
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
#pragma unroll 4
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
  // (the block-wide flag test keeps the barrier inside uniform; without those flags nothing
  // reads the sums)
  float sums[5] = {vdg, gb, p3 ? gwv : gw, qq * vdq, kk * gdk};
  if (sd || sg || prolog) block_sums<5>(sums, red);

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
