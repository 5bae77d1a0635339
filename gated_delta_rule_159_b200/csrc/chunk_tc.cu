// chunk_tc.cu -- chunked Gated DeltaNet-2 forward on the sm_100a tensor cores
// (d_k = d_v = 128, chunk C = 64, bf16 inputs, fp32 state).
//
// The chunkwise WY form (alanhou.org "Core Mechanism": decay absorbed into
// asymmetric erase factors; gist.science Methodologie 3: a lower-triangular
// (I + T)^-1 solve yields erase-side and write-side auxiliaries) for one chunk
// of rows i, j in [0, 64) starting from state S (d_k x d_v):
//
//   x = b.k (erase outer), y = k (erase read), p = w.k (write outer), z = v,
//   L_i = sum_{j<=i} log_a_j (per channel), L_ref = L_31, L_C = L_63.
//   Scaled operands (every factor's exponent is bounded by half a chunk):
//     k_r = k e^{L - L_ref},  q_r = q e^{L - L_ref},
//     x_r = x e^{L_ref - L},  p_r = p e^{L_ref - L},  S_r = Diag(e^{L_ref}) S.
//   G1  [A B ; QX QP] = [k_r ; q_r] [x_r ; p_r]^T         (M=128 N=128 K=128)
//       A, B strictly lower; QX, QP lower incl. diagonal.
//   solve T = (I + A)^-1 (16x16 diagonal blocks by forward substitution, then
//       the off-diagonal blocks level by level: T_IJ = -T_II sum_K A_IK T_KJ).
//   G2  W_r^T = k_r^T T^T ,  (B V)^T = V^T B^T              (M=128 N=64 K=64)
//   G3  M^T = (B V)^T T^T + S_r^T W_r^T                     (M=128 N=64 K=64+128)
//       row i of M is the erase read r_i = Sbar_i^T k_i of every token.
//   G4  O^T = S_r^T q_r^T + V^T QP^T - M^T QX^T             (M=128 N=64 K=128+64+64)
//   G5  dS  = p_r^T V - x_r^T M                             (M=128 N=128 K=64+64)
//   S  <- Diag(e^{L_C}) S + Diag(e^{L_C - L_ref}) dS.
// All GEMMs are tcgen05.mma kind::f16 (bf16 operands from shared memory, fp32
// accumulators in TMEM); the state S is kept in TMEM in fp32 for the whole
// sequence and only its bf16 image S_r is an MMA operand.  Operand tiles arrive
// by TMA (128-byte swizzle); transposed operands use MN-major descriptors, so no
// tile is ever transposed in memory.
//
// One CTA (256 threads) per SM, persistent over (sequence, head) units taken
// longest-first from an atomic counter in the caller's workspace.  Every
// mbarrier wait is bounded; a timeout sets the workspace status word and the
// CTA winds down instead of hanging.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstring>
#include <mutex>

#include "common.cuh"
#include "internal.h"
#include "sm100_ptx.cuh"

namespace gdn2 {
namespace {

constexpr int C = 64;
constexpr int D = 128;
constexpr int kThreads = 256;
constexpr uint32_t kTmemCols = 512;
constexpr uint64_t kWaitTimeoutNs = 1000000000ull;  // 1 s

// Shared-memory map, byte offsets from a 1024-byte-aligned base.  Every operand
// tile is a stack of 8-row x 128-byte swizzle atoms.
constexpr uint32_t OFF_KQ = 0;         // 2 K-blocks x [k_r rows 0-63 | q_r rows 0-63], 16 KB each
constexpr uint32_t OFF_XP = 32768;     // 2 K-blocks x [x_r rows | p_r rows]
constexpr uint32_t OFF_V = 65536;      // 2 column blocks x [64 rows], 8 KB each
constexpr uint32_t OFF_G = 81920;      // raw log_a tile; fp32 A during the solve
constexpr uint32_t OFF_SR = 98304;     // S_r bf16: 2 dv-blocks x [128 dk rows], 16 KB each
constexpr uint32_t OFF_T = 131072;     // T bf16 [64 x 64]
constexpr uint32_t OFF_BM = 139264;    // B bf16 [64 x 64]
constexpr uint32_t OFF_QX = 147456;    // QX bf16 [64 x 64]
constexpr uint32_t OFF_QP = 155648;    // QP bf16 [64 x 64]
constexpr uint32_t OFF_WT = 163840;    // W_r^T bf16 [128 x 64]; fp32 T during the solve
constexpr uint32_t OFF_BZ = 180224;    // (B V)^T bf16 [128 x 64]; o staging (with OFF_MT)
constexpr uint32_t OFF_MT = 196608;    // -M^T bf16 [128 x 64]; solve scratch
constexpr uint32_t OFF_MISC = 212992;
constexpr uint32_t MISC_GC = 0;        // float[128]  e^{L_C}
constexpr uint32_t MISC_DL = 512;      // float[128]  e^{L_C - L_ref}
constexpr uint32_t MISC_SM = 1024;     // float[128]  e^{L_ref}
constexpr uint32_t MISC_PART = 1536;   // float[4][128] quarter sums of log_a
constexpr uint32_t MISC_BAR_TMA = 3584;
constexpr uint32_t MISC_BAR_MMA = 3592;
constexpr uint32_t MISC_TMEM = 3600;
constexpr uint32_t MISC_ABORT = 3604;
constexpr uint32_t MISC_UNIT = 3608;
constexpr uint32_t MISC_BYTES = 3616;
constexpr uint32_t kSmemBytes = OFF_MISC + MISC_BYTES + 1024;  // + base alignment slack

struct TcParams {
  CUtensorMap tm_q, tm_k, tm_v, tm_g, tm_b, tm_w;
  ChunkProblem p;
  int32_t *counter;
  int n_units;
};

__device__ __forceinline__ uint32_t lds_u32(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ void sts_u32(uint32_t a, uint32_t v) {
  asm volatile("st.shared.u32 [%0], %1;" ::"r"(a), "r"(v) : "memory");
}
__device__ __forceinline__ void sts_u16(uint32_t a, uint16_t v) {
  asm volatile("st.shared.u16 [%0], %1;" ::"r"(a), "h"(v) : "memory");
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

// fp32 64x64 scratch with a 16-byte-chunk XOR swizzle (conflict-free row writes).
__device__ __forceinline__ int fidx(int i, int j) { return i * 64 + ((((j >> 2) ^ (i & 7))) << 2) + (j & 3); }

// Byte offset of element pair (row r, 16-byte chunk `chunk`) in a 128B-swizzled tile.
__device__ __forceinline__ uint32_t swz(int r, uint32_t chunk) {
  return (uint32_t)r * 128u + (((chunk ^ (uint32_t)(r & 7))) << 4);
}

__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                         int32_t *status) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  if (*abort_flag) return false;
  const uint64_t t0 = global_timer_ns();
  uint32_t it = 0;
  while (!ptx::mbar_try_wait(bar, parity)) {
    if ((++it & 255u) == 0) {
      if (*abort_flag) return false;
      if (global_timer_ns() - t0 > kWaitTimeoutNs) {
        *abort_flag = 1;
        if (status) atomicExch(status, kStatusTimeout);
        return false;
      }
    }
  }
  return true;
}

__device__ __forceinline__ uint4 pack8(const float *f, float s) {
  uint4 v;
  v.x = pack_bf16x2(f[0] * s, f[1] * s);
  v.y = pack_bf16x2(f[2] * s, f[3] * s);
  v.z = pack_bf16x2(f[4] * s, f[5] * s);
  v.w = pack_bf16x2(f[6] * s, f[7] * s);
  return v;
}

template <bool kScalarDecay, bool kScalarGates, typename Tout>
__global__ void __launch_bounds__(kThreads, 1) chunk_tc_kernel(const __grid_constant__ TcParams P) {
  extern __shared__ uint8_t smem_raw[];
  const ChunkProblem &p = P.p;
  const uint32_t raw = ptx::smem_u32(smem_raw);
  const uint32_t sb = (raw + 1023u) & ~1023u;
  uint8_t *gb = smem_raw + (sb - raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int qd = warp & 3, hf = warp >> 2;
  const int H = p.n_heads;
  const bool tied = (p.flags & GDN2_TIED_GATES) != 0;

  float *sGC = reinterpret_cast<float *>(gb + OFF_MISC + MISC_GC);
  float *sDL = reinterpret_cast<float *>(gb + OFF_MISC + MISC_DL);
  float *sSM = reinterpret_cast<float *>(gb + OFF_MISC + MISC_SM);
  float *part = reinterpret_cast<float *>(gb + OFF_MISC + MISC_PART);
  volatile int *sAbort = reinterpret_cast<volatile int *>(gb + OFF_MISC + MISC_ABORT);
  volatile int *sUnit = reinterpret_cast<volatile int *>(gb + OFF_MISC + MISC_UNIT);
  const uint32_t barTma = sb + OFF_MISC + MISC_BAR_TMA;
  const uint32_t barMma = sb + OFF_MISC + MISC_BAR_MMA;

  if (tid == 0) {
    ptx::mbar_init(barTma, 1);
    ptx::mbar_init(barMma, 1);
    ptx::fence_mbar_init();
    *sAbort = 0;
    ptx::tma_prefetch_desc(&P.tm_q);
    ptx::tma_prefetch_desc(&P.tm_k);
    ptx::tma_prefetch_desc(&P.tm_v);
  }
  if (warp == 0) {
    ptx::tmem_alloc(sb + OFF_MISC + MISC_TMEM, kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(gb + OFF_MISC + MISC_TMEM);
  const uint32_t tmD1 = tmem;        // G1 result, then dS (128 cols)
  const uint32_t tmS = tmem + 128;   // fp32 state (128 cols)
  const uint32_t tmW = tmem + 256;   // W_r^T, then M^T (64 cols)
  const uint32_t tmBZ = tmem + 320;  // (B V)^T, then O^T (64 cols)
  const uint32_t lane_base = (uint32_t)(qd * 32) << 16;
  const int row = qd * 32 + lane;    // the TMEM lane this thread reads
  uint32_t tma_phase = 0, mma_phase = 0;

  const __nv_bfloat16 *g_la = static_cast<const __nv_bfloat16 *>(p.log_a);
  const __nv_bfloat16 *g_b = static_cast<const __nv_bfloat16 *>(p.b);
  const __nv_bfloat16 *g_w = static_cast<const __nv_bfloat16 *>(tied ? p.b : p.w);

  for (;;) {
    if (tid == 0) *sUnit = atomicAdd(P.counter, 1);
    __syncthreads();
    const int u = *sUnit;
    if (u >= P.n_units || *sAbort) break;
    const int unit = p.schedule ? p.schedule[u] : u;
    const int n = unit / H, h = unit % H;
    int64_t bos, len;
    if (p.cu_seqlens) {
      bos = p.cu_seqlens[n];
      len = (int64_t)p.cu_seqlens[n + 1] - bos;
    } else {
      bos = (int64_t)n * p.seq_len;
      len = p.seq_len;
    }

    // ---- initial state into TMEM (thread: dk row `row`, dv columns [64 hf, 64 hf + 64))
    for (int h32 = 0; h32 < 2; ++h32) {
      uint32_t r[32];
      if (p.S0) {
        const float4 *src = reinterpret_cast<const float4 *>(p.S0 + ((size_t)unit * D + row) * D + hf * 64 + h32 * 32);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float4 f = src[j];
          r[4 * j] = __float_as_uint(f.x);
          r[4 * j + 1] = __float_as_uint(f.y);
          r[4 * j + 2] = __float_as_uint(f.z);
          r[4 * j + 3] = __float_as_uint(f.w);
        }
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) r[j] = 0u;
      }
      ptx::tmem_st32(tmS + lane_base + hf * 64 + h32 * 32, r);
    }
    ptx::tmem_wait_st();

    for (int64_t c0 = 0; c0 < len; c0 += C) {
      const int nvalid = (int)((len - c0) < C ? (len - c0) : C);
      const int t0 = (int)(bos + c0);

      // ---- a1: TMA loads of the chunk tiles
      if (tid == 0 && !*sAbort) {
        uint32_t bytes = 3u * 2u * 8192u;
        if (!kScalarDecay) bytes += 2u * 8192u;
        if (!kScalarGates) bytes += 2u * 2u * 8192u;
        ptx::mbar_arrive_expect_tx(barTma, bytes);
#pragma unroll
        for (int kb = 0; kb < 2; ++kb) {
          ptx::tma_load_3d(sb + OFF_KQ + kb * 16384, &P.tm_k, kb * 64, h, t0, barTma);
          ptx::tma_load_3d(sb + OFF_KQ + kb * 16384 + 8192, &P.tm_q, kb * 64, h, t0, barTma);
          ptx::tma_load_3d(sb + OFF_V + kb * 8192, &P.tm_v, kb * 64, h, t0, barTma);
          if (!kScalarGates) {
            ptx::tma_load_3d(sb + OFF_XP + kb * 16384, &P.tm_b, kb * 64, h, t0, barTma);
            ptx::tma_load_3d(sb + OFF_XP + kb * 16384 + 8192, &P.tm_w, kb * 64, h, t0, barTma);
          }
          if (!kScalarDecay) ptx::tma_load_3d(sb + OFF_G + kb * 8192, &P.tm_g, kb * 64, h, t0, barTma);
        }
      }
      wait_bar(barTma, tma_phase, sAbort, p.status);
      tma_phase ^= 1u;

      // ---- a2/a3: cumulative log-decay and scaled operands, in place
      {
        const int cp = tid & 63, rq = tid >> 6, kb = cp >> 5;
        const uint32_t ch16 = (uint32_t)((cp & 31) >> 2), cofs = (uint32_t)(cp & 3) * 4u;
        float L0[16], L1[16];
        float a0 = 0.f, a1 = 0.f;
#pragma unroll
        for (int rr = 0; rr < 16; ++rr) {
          const int r = rq * 16 + rr;
          float g0 = 0.f, g1 = 0.f;
          if (r < nvalid) {
            if (kScalarDecay) {
              g0 = g1 = __bfloat162float(g_la[(size_t)(t0 + r) * H + h]);
            } else {
              const float2 f = unpack_bf16x2(lds_u32(sb + OFF_G + kb * 8192 + swz(r, ch16) + cofs));
              g0 = f.x;
              g1 = f.y;
            }
          }
          a0 += g0;
          a1 += g1;
          L0[rr] = a0;
          L1[rr] = a1;
        }
        part[rq * 128 + 2 * cp] = a0;
        part[rq * 128 + 2 * cp + 1] = a1;
        __syncthreads();
        float off0 = 0.f, off1 = 0.f;
        for (int j = 0; j < rq; ++j) {
          off0 += part[j * 128 + 2 * cp];
          off1 += part[j * 128 + 2 * cp + 1];
        }
        const float ref0 = part[2 * cp] + part[128 + 2 * cp];
        const float ref1 = part[2 * cp + 1] + part[128 + 2 * cp + 1];
        const float end0 = ref0 + part[256 + 2 * cp] + part[384 + 2 * cp];
        const float end1 = ref1 + part[256 + 2 * cp + 1] + part[384 + 2 * cp + 1];
        if (rq == 0) {
          sGC[2 * cp] = exp_fast(end0);
          sGC[2 * cp + 1] = exp_fast(end1);
          sDL[2 * cp] = exp_fast(end0 - ref0);
          sDL[2 * cp + 1] = exp_fast(end1 - ref1);
          sSM[2 * cp] = exp_fast(ref0);
          sSM[2 * cp + 1] = exp_fast(ref1);
        }
#pragma unroll
        for (int rr = 0; rr < 16; ++rr) {
          const int r = rq * 16 + rr;
          const uint32_t o = kb * 16384 + swz(r, ch16) + cofs;
          const float l0 = off0 + L0[rr] - ref0, l1 = off1 + L1[rr] - ref1;
          const float e10 = exp_fast(l0), e11 = exp_fast(l1);
          const float e20 = exp_fast(-l0), e21 = exp_fast(-l1);
          float2 kk = unpack_bf16x2(lds_u32(sb + OFF_KQ + o));
          float2 qq = unpack_bf16x2(lds_u32(sb + OFF_KQ + o + 8192));
          float2 bb, ww;
          if (kScalarGates) {
            bb.x = bb.y = 0.f;
            ww = bb;
            if (r < nvalid) {
              bb.x = bb.y = __bfloat162float(g_b[(size_t)(t0 + r) * H + h]);
              ww.x = ww.y = __bfloat162float(g_w[(size_t)(t0 + r) * H + h]);
            }
          } else {
            bb = unpack_bf16x2(lds_u32(sb + OFF_XP + o));
            ww = unpack_bf16x2(lds_u32(sb + OFF_XP + o + 8192));
          }
          if (r >= nvalid) {
            kk = make_float2(0.f, 0.f);
            qq = kk;
            bb = kk;
            ww = kk;
            sts_u32(sb + OFF_V + kb * 8192 + swz(r, ch16) + cofs, 0u);
          }
          sts_u32(sb + OFF_KQ + o, pack_bf16x2(kk.x * e10, kk.y * e11));
          sts_u32(sb + OFF_KQ + o + 8192, pack_bf16x2(qq.x * e10, qq.y * e11));
          sts_u32(sb + OFF_XP + o, pack_bf16x2(bb.x * kk.x * e20, bb.y * kk.y * e21));
          sts_u32(sb + OFF_XP + o + 8192, pack_bf16x2(ww.x * kk.x * e20, ww.y * kk.y * e21));
        }
      }
      __syncthreads();

      // ---- S_r = Diag(e^{L_ref}) S as a bf16 MN-major operand
      {
        const float sm = sSM[row];
#pragma unroll
        for (int h32 = 0; h32 < 2; ++h32) {
          uint32_t r[32];
          ptx::tmem_ld32(tmS + lane_base + hf * 64 + h32 * 32, r);
          ptx::tmem_wait_ld();
          float f[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) f[j] = __uint_as_float(r[j]);
#pragma unroll
          for (int q8 = 0; q8 < 4; ++q8)
            sts_v4(sb + OFF_SR + hf * 16384 + swz(row, (uint32_t)(h32 * 4 + q8)), pack8(f + 8 * q8, sm));
        }
      }
      ptx::fence_proxy_async_smem();
      ptx::tc_fence_before();
      __syncthreads();

      // ---- a4: G1  [A B; QX QP] = [k_r; q_r] [x_r; p_r]^T
      if (tid == 0) {
        ptx::tc_fence_after();
        constexpr uint32_t id = ptx::idesc_bf16(128, 128, false, false);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t ko = (uint32_t)(kk >> 2) * 16384u + (uint32_t)(kk & 3) * 32u;
          ptx::umma_bf16(tmD1, ptx::sdesc_sw128(sb + OFF_KQ + ko, 16, 1024),
                         ptx::sdesc_sw128(sb + OFF_XP + ko, 16, 1024), id, kk > 0);
        }
        ptx::umma_commit(barMma);
      }
      wait_bar(barMma, mma_phase, sAbort, p.status);
      mma_phase ^= 1u;
      ptx::tc_fence_after();

      // masks: A, B strictly lower (fp32 A for the solve, bf16 B); QX, QP lower incl. diagonal
      {
        float *Af = reinterpret_cast<float *>(gb + OFF_G);
#pragma unroll
        for (int h32 = 0; h32 < 2; ++h32) {
          uint32_t r[32];
          ptx::tmem_ld32(tmD1 + lane_base + hf * 64 + h32 * 32, r);
          ptx::tmem_wait_ld();
          float f[32];
          if (qd < 2) {
            const int i = row;
#pragma unroll
            for (int j = 0; j < 32; ++j) f[j] = (h32 * 32 + j < i) ? __uint_as_float(r[j]) : 0.f;
            if (hf == 0) {
#pragma unroll
              for (int j4 = 0; j4 < 8; ++j4)
                *reinterpret_cast<float4 *>(Af + fidx(i, h32 * 32 + 4 * j4)) =
                    make_float4(f[4 * j4], f[4 * j4 + 1], f[4 * j4 + 2], f[4 * j4 + 3]);
            } else {
#pragma unroll
              for (int q8 = 0; q8 < 4; ++q8)
                sts_v4(sb + OFF_BM + swz(i, (uint32_t)(h32 * 4 + q8)), pack8(f + 8 * q8, 1.f));
            }
          } else {
            const int i = row - 64;
#pragma unroll
            for (int j = 0; j < 32; ++j) f[j] = (h32 * 32 + j <= i) ? __uint_as_float(r[j]) : 0.f;
            const uint32_t dst = hf == 0 ? OFF_QX : OFF_QP;
#pragma unroll
            for (int q8 = 0; q8 < 4; ++q8) sts_v4(sb + dst + swz(i, (uint32_t)(h32 * 4 + q8)), pack8(f + 8 * q8, 1.f));
          }
        }
      }
      __syncthreads();

      // ---- a5: T = (I + A)^-1 by blocked forward substitution (fp32)
      {
        const float *Af = reinterpret_cast<const float *>(gb + OFF_G);
        float *Tf = reinterpret_cast<float *>(gb + OFF_WT);
        float *Xs = reinterpret_cast<float *>(gb + OFF_MT);
        if (tid < 64) {
          const int I = tid >> 4, m = tid & 15;
          float t[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            float acc = (i == m) ? 1.f : 0.f;
#pragma unroll
            for (int j = 0; j < i; ++j) acc -= Af[fidx(16 * I + i, 16 * I + j)] * t[j];
            t[i] = acc;
          }
#pragma unroll
          for (int i = 0; i < 16; ++i) Tf[fidx(16 * I + i, 16 * I + m)] = t[i];
        } else {
          for (int e = tid - 64; e < 6 * 256; e += kThreads - 64) {
            const int blk = e >> 8, i = (e >> 4) & 15, m = e & 15;
            const int I = blk < 3 ? 0 : (blk < 5 ? 1 : 2);
            const int J = blk < 3 ? blk + 1 : (blk < 5 ? blk - 1 : 3);
            Tf[fidx(16 * I + i, 16 * J + m)] = 0.f;
          }
        }
        __syncthreads();
        for (int d = 1; d < 4; ++d) {
          const int nb = 4 - d;
          for (int e = tid; e < nb * 256; e += kThreads) {
            const int J = e >> 8, I = J + d, i = (e >> 4) & 15, m = e & 15;
            float acc = 0.f;
            for (int K = J; K < I; ++K) {
#pragma unroll
              for (int s = 0; s < 16; ++s) acc += Af[fidx(16 * I + i, 16 * K + s)] * Tf[fidx(16 * K + s, 16 * J + m)];
            }
            Xs[e] = acc;
          }
          __syncthreads();
          for (int e = tid; e < nb * 256; e += kThreads) {
            const int J = e >> 8, I = J + d, i = (e >> 4) & 15, m = e & 15;
            float acc = 0.f;
            for (int r2 = 0; r2 <= i; ++r2) acc -= Tf[fidx(16 * I + i, 16 * I + r2)] * Xs[(J << 8) + (r2 << 4) + m];
            Tf[fidx(16 * I + i, 16 * J + m)] = acc;
          }
          __syncthreads();
        }
        {
          const int i = tid >> 2, seg = tid & 3;
#pragma unroll
          for (int u2 = 0; u2 < 2; ++u2) {
            const int j0 = seg * 16 + u2 * 8;
            float f[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) f[j] = Tf[fidx(i, j0 + j)];
            sts_v4(sb + OFF_T + swz(i, (uint32_t)(j0 >> 3)), pack8(f, 1.f));
          }
        }
      }
      ptx::fence_proxy_async_smem();
      ptx::tc_fence_before();
      __syncthreads();

      // ---- a6: G2  W_r^T = k_r^T T^T,  (B V)^T = V^T B^T
      if (tid == 0) {
        ptx::tc_fence_after();
        constexpr uint32_t id = ptx::idesc_bf16(128, 64, true, false);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          ptx::umma_bf16(tmW, ptx::sdesc_sw128(sb + OFF_KQ + kk * 2048, 16384, 1024),
                         ptx::sdesc_sw128(sb + OFF_T + kk * 32, 16, 1024), id, kk > 0);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          ptx::umma_bf16(tmBZ, ptx::sdesc_sw128(sb + OFF_V + kk * 2048, 8192, 1024),
                         ptx::sdesc_sw128(sb + OFF_BM + kk * 32, 16, 1024), id, kk > 0);
        ptx::umma_commit(barMma);
      }
      wait_bar(barMma, mma_phase, sAbort, p.status);
      mma_phase ^= 1u;
      ptx::tc_fence_after();
      {
        const uint32_t src = hf == 0 ? tmW : tmBZ;
        const uint32_t dst = hf == 0 ? OFF_WT : OFF_BZ;
#pragma unroll
        for (int h32 = 0; h32 < 2; ++h32) {
          uint32_t r[32];
          ptx::tmem_ld32(src + lane_base + h32 * 32, r);
          ptx::tmem_wait_ld();
          float f[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) f[j] = __uint_as_float(r[j]);
#pragma unroll
          for (int q8 = 0; q8 < 4; ++q8) sts_v4(sb + dst + swz(row, (uint32_t)(h32 * 4 + q8)), pack8(f + 8 * q8, 1.f));
        }
      }
      ptx::fence_proxy_async_smem();
      ptx::tc_fence_before();
      __syncthreads();

      // ---- a7 (erase reads): G3  M^T = (B V)^T T^T + S_r^T W_r^T
      if (tid == 0) {
        ptx::tc_fence_after();
        constexpr uint32_t idA = ptx::idesc_bf16(128, 64, false, false);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          ptx::umma_bf16(tmW, ptx::sdesc_sw128(sb + OFF_BZ + kk * 32, 16, 1024),
                         ptx::sdesc_sw128(sb + OFF_T + kk * 32, 16, 1024), idA, kk > 0);
        constexpr uint32_t idB = ptx::idesc_bf16(128, 64, true, true);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          ptx::umma_bf16(tmW, ptx::sdesc_sw128(sb + OFF_SR + kk * 2048, 16384, 1024),
                         ptx::sdesc_sw128(sb + OFF_WT + kk * 2048, 16384, 1024), idB, 1);
        ptx::umma_commit(barMma);
      }
      wait_bar(barMma, mma_phase, sAbort, p.status);
      mma_phase ^= 1u;
      ptx::tc_fence_after();
      {
        uint32_t r[32];
        ptx::tmem_ld32(tmW + lane_base + hf * 32, r);
        ptx::tmem_wait_ld();
        float f[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) f[j] = __uint_as_float(r[j]);
#pragma unroll
        for (int q8 = 0; q8 < 4; ++q8) sts_v4(sb + OFF_MT + swz(row, (uint32_t)(hf * 4 + q8)), pack8(f + 8 * q8, -1.f));
      }
      ptx::fence_proxy_async_smem();
      ptx::tc_fence_before();
      __syncthreads();

      // ---- a7/a8: G4 outputs and G5 state increment
      if (tid == 0) {
        ptx::tc_fence_after();
        constexpr uint32_t idO1 = ptx::idesc_bf16(128, 64, true, false);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          ptx::umma_bf16(tmBZ, ptx::sdesc_sw128(sb + OFF_SR + kk * 2048, 16384, 1024),
                         ptx::sdesc_sw128(sb + OFF_KQ + (kk >> 2) * 16384 + 8192 + (kk & 3) * 32, 16, 1024), idO1,
                         kk > 0);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          ptx::umma_bf16(tmBZ, ptx::sdesc_sw128(sb + OFF_V + kk * 2048, 8192, 1024),
                         ptx::sdesc_sw128(sb + OFF_QP + kk * 32, 16, 1024), idO1, 1);
        constexpr uint32_t idO2 = ptx::idesc_bf16(128, 64, false, false);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          ptx::umma_bf16(tmBZ, ptx::sdesc_sw128(sb + OFF_MT + kk * 32, 16, 1024),
                         ptx::sdesc_sw128(sb + OFF_QX + kk * 32, 16, 1024), idO2, 1);
        constexpr uint32_t idS1 = ptx::idesc_bf16(128, 128, true, true);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          ptx::umma_bf16(tmD1, ptx::sdesc_sw128(sb + OFF_XP + 8192 + kk * 2048, 16384, 1024),
                         ptx::sdesc_sw128(sb + OFF_V + kk * 2048, 8192, 1024), idS1, kk > 0);
        constexpr uint32_t idS2 = ptx::idesc_bf16(128, 128, true, false);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          ptx::umma_bf16(tmD1, ptx::sdesc_sw128(sb + OFF_XP + kk * 2048, 16384, 1024),
                         ptx::sdesc_sw128(sb + OFF_MT + kk * 32, 16, 1024), idS2, 1);
        ptx::umma_commit(barMma);
      }
      wait_bar(barMma, mma_phase, sAbort, p.status);
      mma_phase ^= 1u;
      ptx::tc_fence_after();
      {
        // o^T lane = dv channel `row`, columns = tokens [32 hf, 32 hf + 32)
        uint32_t r[32];
        ptx::tmem_ld32(tmBZ + lane_base + hf * 32, r);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int i = hf * 32 + j;
          const float f = __uint_as_float(r[j]);
          if (sizeof(Tout) == 2) {
            const __nv_bfloat16 hv = __float2bfloat16_rn(f);
            sts_u16(sb + OFF_BZ + (uint32_t)i * 256u + (uint32_t)row * 2u, *reinterpret_cast<const uint16_t *>(&hv));
          } else {
            sts_f32(sb + OFF_BZ + (uint32_t)i * 512u + (uint32_t)row * 4u, f);
          }
        }
        // S <- e^{L_C} S + e^{L_C - L_ref} dS   (thread: dk row `row`)
        const float gc = sGC[row], dl = sDL[row];
#pragma unroll
        for (int h32 = 0; h32 < 2; ++h32) {
          uint32_t s[32], ds[32];
          ptx::tmem_ld32(tmS + lane_base + hf * 64 + h32 * 32, s);
          ptx::tmem_ld32(tmD1 + lane_base + hf * 64 + h32 * 32, ds);
          ptx::tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 32; ++j)
            s[j] = __float_as_uint(fmaf(gc, __uint_as_float(s[j]), dl * __uint_as_float(ds[j])));
          ptx::tmem_st32(tmS + lane_base + hf * 64 + h32 * 32, s);
        }
        ptx::tmem_wait_st();
      }
      __syncthreads();
      {
        constexpr int kRowBytes = D * (int)sizeof(Tout);
        constexpr int kU4 = kRowBytes / 16;
        uint8_t *go = static_cast<uint8_t *>(p.o);
        for (int e = tid; e < nvalid * kU4; e += kThreads) {
          const int i = e / kU4, uu = e % kU4;
          const uint4 val = lds_v4(sb + OFF_BZ + (uint32_t)(i * kRowBytes + uu * 16));
          *reinterpret_cast<uint4 *>(go + ((size_t)(t0 + i) * H + h) * kRowBytes + uu * 16) = val;
        }
      }
      ptx::tc_fence_before();
      __syncthreads();
      if (*sAbort) break;
    }

    // ---- a8: final state
    if (p.S_T && !*sAbort) {
      float *dst = p.S_T + ((size_t)unit * D + row) * D + hf * 64;
#pragma unroll
      for (int h32 = 0; h32 < 2; ++h32) {
        uint32_t r[32];
        ptx::tmem_ld32(tmS + lane_base + hf * 64 + h32 * 32, r);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 8; ++j)
          reinterpret_cast<float4 *>(dst + h32 * 32)[j] =
              make_float4(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1]), __uint_as_float(r[4 * j + 2]),
                          __uint_as_float(r[4 * j + 3]));
      }
    }
    ptx::tc_fence_before();
    __syncthreads();
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------- host side
PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// [T_tot][H][128] bf16 viewed as (channel, head, token); box 64 channels x 1 head x 64 tokens.
bool make_map(CUtensorMap *m, const void *base, int64_t t_total, int H) {
  auto enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)t_total};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2};
  cuuint32_t box[3] = {64, 1, 64};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <bool SD, bool SG, typename Tout>
cudaError_t launch_t(const TcParams &P, int grid, cudaStream_t stream) {
  auto kern = chunk_tc_kernel<SD, SG, Tout>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  kern<<<grid, kThreads, kSmemBytes, stream>>>(P);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_chunk_tc(const ChunkProblem &p, cudaStream_t stream, const char **why) {
  if (p.d_k != D || p.d_v != D || p.chunk != C || p.dtype_in != GDN2_BF16) {
    *why = "tensor-core path needs d_k = d_v = 128, chunk 64 and bf16 inputs";
    return cudaErrorNotSupported;
  }
  if (p.t_total >= (int64_t)1 << 31) {
    *why = "tensor-core path needs T_tot < 2^31";
    return cudaErrorNotSupported;
  }
  const bool sd = (p.flags & GDN2_SCALAR_DECAY) != 0;
  const bool sg = (p.flags & GDN2_SCALAR_GATES) != 0;
  const bool tied = (p.flags & GDN2_TIED_GATES) != 0;
  TcParams P;
  memset(&P, 0, sizeof(P));
  P.p = p;
  P.n_units = p.n_seqs * p.n_heads;
  P.counter = p.status + 1;
  if (P.n_units == 0) return cudaSuccess;
  const int64_t T = p.t_total > 0 ? p.t_total : 1;
  bool ok = make_map(&P.tm_q, p.q, T, p.n_heads) && make_map(&P.tm_k, p.k, T, p.n_heads) &&
            make_map(&P.tm_v, p.v, T, p.n_heads);
  if (ok && !sd) ok = make_map(&P.tm_g, p.log_a, T, p.n_heads);
  if (ok && !sg) ok = make_map(&P.tm_b, p.b, T, p.n_heads) && make_map(&P.tm_w, tied ? p.b : p.w, T, p.n_heads);
  if (!ok) {
    *why = "cuTensorMapEncodeTiled failed (driver entry point missing or bad tensor geometry)";
    return cudaErrorInvalidValue;
  }
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = P.n_units < sms ? P.n_units : sms;
  const bool obf = p.dtype_out == GDN2_BF16;
  if (sd && sg) return obf ? launch_t<true, true, __nv_bfloat16>(P, grid, stream) : launch_t<true, true, float>(P, grid, stream);
  if (sd) return obf ? launch_t<true, false, __nv_bfloat16>(P, grid, stream) : launch_t<true, false, float>(P, grid, stream);
  if (sg) return obf ? launch_t<false, true, __nv_bfloat16>(P, grid, stream) : launch_t<false, true, float>(P, grid, stream);
  return obf ? launch_t<false, false, __nv_bfloat16>(P, grid, stream) : launch_t<false, false, float>(P, grid, stream);
}

}  // namespace gdn2
