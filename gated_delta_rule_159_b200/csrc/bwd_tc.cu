// bwd_tc.cu -- gradients of the chunked Gated DeltaNet-2 forward on the sm_100a tensor cores
// (d_k = d_v = 128, chunk C = 64, bf16 inputs, fp32 accumulation), chunk by chunk in reverse.
//
// The method trains through its chunked form with a gate-aware backward (gist.science
// Methodologie 3, "Poortbewuste terugwaartse pass"; alanhou.org "Core Mechanism"); the pages
// give no formula for it.  This file differentiates the chunk algebra of chunk_tc.cu.  For one
// chunk (rows t, s in [0, 64); the operands scaled to the per-channel reference
// rho = (L_0 + L_63) / 2 exactly as the forward scales them):
//
//   k_r = k e^{L - rho}, q_r = q e^{L - rho}, x_r = b.k e^{rho - L}, p_r = w.k e^{rho - L},
//   S_r = Diag(e^{rho}) S_c (S_c: the state before the chunk), gamma = e^{L_63 - rho},
//   A = (k_r x_r^T)|strict, B = (k_r p_r^T)|strict, QX = (q_r x_r^T)|lower, QP = (q_r p_r^T)|lower,
//   R = B V + k_r S_r,  M = T R with T = (I + A)^-1  (row t of M: the erase read of token t),
//   O = q_r S_r + QP V - QX M,    S_{c+1} = Diag(gamma) (S_r + p_r^T V - x_r^T M).
//
// With Lam = dLoss/dS_{c+1} and Lam_g = Diag(gamma) Lam, reverse mode gives
//
//   dM = -(QX^T dO + x_r Lam_g),  dR = T^T dM,
//   [dA dB; dQX dQP] = ([dR; dO] [-M; V]^T) masked like [A B; QX QP],
//   dV   = QP^T dO + B^T dR + p_r Lam_g,
//   dk_r = dA x_r + dB p_r + dR S_r^T,    dq_r = dQX x_r + dQP p_r + dO S_r^T,
//   dx_r = dA^T k_r + dQX^T q_r - M Lam_g^T,   dp_r = dB^T k_r + dQP^T q_r + V Lam_g^T,
//   dLoss/dS_c = Diag(e^{rho}) (Lam_g + q_r^T dO + k_r^T dR),
//   dL_t = dq_r.q_r + dk_r.k_r - dx_r.x_r - dp_r.p_r (per channel), plus at t = 63 the decay
//   term sum_j Lam_ij (S_{c+1})_ij; d log_a_s = sum_{t >= s} dL_t (inside the chunk).
//
// rho only moves factors between operands (the chunk's function does not depend on it), so
// it takes no gradient.  Every product runs as a tcgen05.mma (kind::f16, bf16 operands, fp32
// TMEM accumulators) with M = 128 rows: the 64-row matrices are stacked in pairs
// ([k_r; q_r], [x_r; p_r], [dR; dO], [-M; V]) so that one instruction covers two of them, and
// the transposed operand forms are MN-major shared-memory descriptors of the same tiles.  The
// carried adjoint lives in TMEM (lane = d_k channel) for the whole sequence, so the thread of a
// d_k channel scales and stores its row with one factor and 16-byte vectors.
//
// The S_r and T tiles come from a forward pass of chunk_tc_kernel that writes each chunk's bf16
// S_r (the operand it builds anyway, with the same rho) and bf16 T = (I + A)^-1 as swizzled tile
// images to the workspace; bulk copies bring them to shared memory, so this pass neither
// recomputes the state nor solves.  One CTA (512 threads) per SM takes (sequence, head) units
// from an atomic counter and walks their chunks last to first; per chunk its phases are:
//   1  (the raw k, q, v, log_a, b, w, dO tiles (TMA) and the S_r, T images (bulk copies) were
//      requested right after the previous chunk's last products) cumulative decay, the scaled
//      operands in place, Lam_g from the TMEM adjoint;
//   2  G1 [A B; QX QP] = [k_r; q_r][x_r; p_r]^T, then dM^T = Lam_g^T x_r^T and R^T = S_r^T k_r^T
//      while the masks write B, QX, QP;
//   3  R^T += V^T B^T, dM^T += dO^T QX;
//   4  R^T, -dM^T to bf16 TMEM operands; M^T = R^T T^T, dR^T = dM^T T;
//   5  -M and dR to their shared-memory tiles;
//   6  the adjoint update, the S_r terms of [dk_r^T | dq_r^T], [dA dB; dQX dQP] (one commit),
//      then dV^T;
//   7  the decay term of the next chunk (row sums of adjoint x S_r), the masks of the gradient
//      tile (over S_r's space);
//   8  [dx_r^T | dp_r^T] and the rest of [dk_r^T | dq_r^T]; dV out while they run;
//   9  the chain rule through the scaling and the gates, the suffix sums of dL, the stores.
// Chunks whose decay range exceeds kFastSpan nats on some channel are outside the factored
// form: the kernel records kStatusRange and leaves the rest of that unit (gdn2_bwd, the
// token-serial reverse mode, covers any range).  Every mbarrier wait is bounded.
#include <cstring>

#include "common.cuh"
#include "internal.h"
#include "sm100_ptx.cuh"
#include "tc_util.cuh"

namespace gdn2 {
namespace {

using namespace tc;

constexpr int C = 64;
constexpr int D = 128;
constexpr int kThreads = 512;
constexpr uint32_t kTmemCols = 512;
constexpr uint64_t kWaitTimeoutNs = 1000000000ull;  // 1 s
constexpr float kLog2eF = 1.4426950408889634f;
constexpr float kFastSpan = 128.f;  // as in the forward: factors stay within e^{+-64}
constexpr size_t kSlotBytes = kBwdCkptSlotBytes;  // per chunk: bf16 S_r tile image, then bf16 T

// Shared-memory map (byte offsets from a 1024-byte-aligned base).  The 128-row operand tiles
// are two column blocks of 64 (16 KB apart), each a stack of 8-row x 128-byte swizzle atoms.
constexpr uint32_t OFF_KQ = 0;          // [k_r rows 0-63 | q_r rows 64-127] per block
constexpr uint32_t OFF_XP = 32768;      // [x_r | p_r]
constexpr uint32_t OFF_MV = 65536;      // [-M | V]
constexpr uint32_t OFF_RO = 98304;      // [dR | dO]
constexpr uint32_t OFF_SR = 131072;     // S_r [d_k rows][d_v]; from phase 7 the gradient tile dG
constexpr uint32_t OFF_LG = 163840;     // Lam_g [d_k rows][d_v]
constexpr uint32_t OFF_BQP = 196608;    // [B rows 0-63 | QP rows 64-127], one 64-column block
constexpr uint32_t OFF_MISC = 212992;
// Tiles that live in the rows of another tile until that tile is written:
constexpr uint32_t OFF_T = OFF_MV;             // T bf16 [64 x 64] (the -M rows of block 0)
constexpr uint32_t OFF_QX = OFF_MV + 16384;    // QX bf16 [64 x 64] (the -M rows of block 1)
constexpr uint32_t OFF_DG = OFF_SR;            // [dA dB; dQX dQP] as [column block][128 rows][64]
constexpr uint32_t OFF_GRAW = OFF_LG;          // raw log_a tile [2 blocks][64 rows] until Lam_g is built
constexpr uint32_t MISC_BAR = 0;       // mbarriers
constexpr uint32_t MISC_TMEM = 80;
constexpr uint32_t MISC_ABORT = 84;
constexpr uint32_t MISC_UNIT = 88;
constexpr uint32_t MISC_WIDE = 92;
constexpr uint32_t MISC_ISS = 96;      // uint32: load phases armed on BAR_LD (for the wind-down)
constexpr uint32_t MISC_RHO = 128;     // float[128]     rho of the current chunk
constexpr uint32_t MISC_ESR = 640;     // float[2][128]  e^{rho} per chunk parity
constexpr uint32_t MISC_DLC = 1664;    // float[2][128]  decay term of L_63 per chunk parity
constexpr uint32_t MISC_L0 = 2688;     // float[128]     L_0
constexpr uint32_t MISC_PART = 3200;   // float[4][128]  per-row-group sums of dL
constexpr uint32_t MISC_LPRE = 5248;   // float[4][128]  exclusive row-group prefixes of L
constexpr uint32_t MISC_RS = 7296;     // float[4][128]  row sums per lane quadrant
constexpr uint32_t MISC_GAM = 9344;    // float[128]     gamma = e^{L_63 - rho} of the current chunk
constexpr uint32_t MISC_SCAL = 9856;   // float[3][64]   scalar log_a, b, w per token of the current chunk
constexpr uint32_t MISC_RED = 10624;   // float[4][3][64] channel sums per lane quadrant (scalar gradients)
constexpr uint32_t MISC_BYTES = 13696;
constexpr uint32_t kSmemBytes = OFF_MISC + MISC_BYTES + 1024;  // + base alignment slack
static_assert(kSmemBytes <= 232448, "shared memory over the sm_100 limit per CTA");
enum { BAR_LD = 0, BAR_G1, BAR_GA, BAR_GB, BAR_G5, BAR_GL, BAR_GZ, BAR_G7, BAR_DRAIN, kNumBars };
static_assert(MISC_BAR + 8 * kNumBars <= MISC_TMEM, "mbarriers overlap the TMEM address slot");

struct BwdTcParams {
  // raw tiles of a chunk by TMA, (channel, head, token) boxes of 64 x 1 x 64, 128-byte swizzle:
  // k, q over the k_r, q_r rows, v over the V rows, b, w over the x_r, p_r rows, log_a into
  // the Lam_g tile's space
  CUtensorMap tm_q, tm_k, tm_v, tm_g, tm_b, tm_w, tm_do;  // tm_do: bf16 dO only
  const __nv_bfloat16 *q, *k, *v, *log_a, *b, *w;  // forward inputs [T_tot][H][128]
  const void *dO;                                  // [T_tot][H][128] Tout
  const float *dS_T;                               // [N][H][128][128] or NULL
  void *dq, *dk, *dv, *dlog_a, *db, *dw;           // Tout, like the inputs (dw NULL when tied)
  float *dS0;                                      // [N][H][128][128] or NULL
  const uint8_t *ckpt;                             // per chunk the bf16 S_r tile image (32 KB)
  const float *S_fin;                              // [N][H][128][128] final states (fp32)
  const int64_t *ckpt_off;                         // NULL for equal lengths
  const int32_t *cu_seqlens;                       // NULL for equal lengths
  const int32_t *schedule;                         // unit order (longest first) or NULL
  int32_t *status, *counter;
  int n_units, n_heads, seq_len;
  uint64_t wait_ns;  // limit of every mbarrier wait (kWaitTimeoutNs unless the timeout test hook is armed)
  int dbg_skip;      // timeout test hook: CTA 0 arms its first load group but issues none of its copies
};

// Sums v[c] over the 32 lanes of the warp for every column c; lane l returns the sum of
// column l.  Each step halves the columns a lane keeps and adds its partner's half.
__device__ __forceinline__ float warp_colsum32(float (&v)[32]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) {
    const bool up = (lane & off) != 0;
#pragma unroll
    for (int j = 0; j < off; ++j) {
      const float send = up ? v[j] : v[j + off];
      const float keep = up ? v[j + off] : v[j];
      v[j] = keep + __shfl_xor_sync(0xffffffffu, send, off);
    }
  }
  return v[0];
}

__device__ __forceinline__ float bf(const __nv_bfloat16 x) { return __bfloat162float(x); }

// 8 x 8 transpose of bf16 values inside each 8-lane group of a warp.  On entry lane m of a
// group holds row m as four packed pairs (w[q] = elements 2q, 2q + 1); on exit it holds
// column m packed the same way (w[q] = rows 2q, 2q + 1).  Exchanges at lane distances 4, 2
// and 1: at each, a lane keeps the half of its elements whose index bit matches its own
// lane bit and trades the other half with its partner.  Every lane of the warp takes part.
__device__ __forceinline__ void transpose8x8_bf16(uint32_t (&w)[4], int lane) {
  const unsigned full = 0xffffffffu;
  {  // distance 4: elements 0-3 (words 0, 1) against 4-7 (words 2, 3)
    const bool up = (lane & 4) != 0;
    const uint32_t r0 = __shfl_xor_sync(full, up ? w[0] : w[2], 4);
    const uint32_t r1 = __shfl_xor_sync(full, up ? w[1] : w[3], 4);
    if (up) {
      w[0] = r0;
      w[1] = r1;
    } else {
      w[2] = r0;
      w[3] = r1;
    }
  }
  {  // distance 2: words 0, 2 against words 1, 3
    const bool up = (lane & 2) != 0;
    const uint32_t r0 = __shfl_xor_sync(full, up ? w[0] : w[1], 2);
    const uint32_t r1 = __shfl_xor_sync(full, up ? w[2] : w[3], 2);
    if (up) {
      w[0] = r0;
      w[2] = r1;
    } else {
      w[1] = r0;
      w[3] = r1;
    }
  }
  {  // distance 1: low halves against high halves, two words' halves per exchange
    const bool up = (lane & 1) != 0;
    const uint32_t r0 = __shfl_xor_sync(full, __byte_perm(w[0], w[1], up ? 0x5410 : 0x7632), 1);
    const uint32_t r1 = __shfl_xor_sync(full, __byte_perm(w[2], w[3], up ? 0x5410 : 0x7632), 1);
    if (up) {  // keeps the high halves; the partner's high halves become the low halves
      w[0] = __byte_perm(r0, w[0], 0x7610);
      w[1] = __byte_perm(r0, w[1], 0x7632);
      w[2] = __byte_perm(r1, w[2], 0x7610);
      w[3] = __byte_perm(r1, w[3], 0x7632);
    } else {   // keeps the low halves; the partner's low halves become the high halves
      w[0] = __byte_perm(w[0], r0, 0x5410);
      w[1] = __byte_perm(w[1], r0, 0x7610);
      w[2] = __byte_perm(w[2], r1, 0x5410);
      w[3] = __byte_perm(w[3], r1, 0x7610);
    }
  }
}

// Descriptors of the 128-column operand tiles (two 64-column blocks 16 KB apart), K step kk
// of 16: K-major walks the columns (32 bytes per step), MN-major walks the rows (16 rows,
// 2 KB per step).
__device__ __forceinline__ uint64_t kmaj(uint32_t base, int kk) {
  return ptx::sdesc_sw128(base + (uint32_t)(kk >> 2) * 16384u + (uint32_t)(kk & 3) * 32u, 16, 1024);
}
__device__ __forceinline__ uint64_t mnmaj(uint32_t base, int kk) {
  return ptx::sdesc_sw128(base + (uint32_t)kk * 2048u, 16384, 1024);
}

// kP3: the gist.science gate placement (erase read y = b.k, erase and write outer factors
// x = p = k, values z = w.v); kSD: log_a is [T_tot, H], kSG: b and w are [T_tot, H] (one value
// per token and head, broadcast over the channels; their gradients are channel sums).
template <typename Tout, bool kTied, bool kP3, bool kSD, bool kSG>
__global__ void __launch_bounds__(kThreads, 1) bwd_tc_kernel(const __grid_constant__ BwdTcParams P) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = ptx::smem_u32(smem_raw);
  const uint32_t sb = (raw + 1023u) & ~1023u;
  uint8_t *gb = smem_raw + (sb - raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int qd = warp & 3, cg = warp >> 2;  // TMEM lane quadrant, column group (row group)
  const int row = qd * 32 + lane;           // TMEM lane; the channel of the elementwise phases
  const int H = P.n_heads;
  constexpr int kIssuer = 480;              // warp 15 lane 0 issues every MMA, in order

  float *sRho = reinterpret_cast<float *>(gb + OFF_MISC + MISC_RHO);
  float *sEsr = reinterpret_cast<float *>(gb + OFF_MISC + MISC_ESR);
  float *sDlc = reinterpret_cast<float *>(gb + OFF_MISC + MISC_DLC);
  float *sL0 = reinterpret_cast<float *>(gb + OFF_MISC + MISC_L0);
  float *part = reinterpret_cast<float *>(gb + OFF_MISC + MISC_PART);
  float *lpre = reinterpret_cast<float *>(gb + OFF_MISC + MISC_LPRE);
  float *rs = reinterpret_cast<float *>(gb + OFF_MISC + MISC_RS);
  float *sGam = reinterpret_cast<float *>(gb + OFF_MISC + MISC_GAM);
  float *sScal = reinterpret_cast<float *>(gb + OFF_MISC + MISC_SCAL);
  float *red = reinterpret_cast<float *>(gb + OFF_MISC + MISC_RED);
  volatile int *sAbort = reinterpret_cast<volatile int *>(gb + OFF_MISC + MISC_ABORT);
  volatile int *sUnit = reinterpret_cast<volatile int *>(gb + OFF_MISC + MISC_UNIT);
  volatile int *sWide = reinterpret_cast<volatile int *>(gb + OFF_MISC + MISC_WIDE);
  volatile uint32_t *sIss = reinterpret_cast<volatile uint32_t *>(gb + OFF_MISC + MISC_ISS);
  auto bar = [&](int i) { return sb + OFF_MISC + MISC_BAR + 8u * (uint32_t)i; };
  auto waitb = [&](uint32_t b, uint32_t parity) { return wait_bar(b, parity, sAbort, P.status, P.wait_ns); };
  if (tid == 0) {
    for (int i = 0; i < kNumBars; ++i) ptx::mbar_init(bar(i), 1);
    ptx::fence_mbar_init();
    *sAbort = 0;
    *sIss = 0u;
    ptx::tma_prefetch_desc(&P.tm_q);
    ptx::tma_prefetch_desc(&P.tm_k);
    ptx::tma_prefetch_desc(&P.tm_v);
    ptx::tma_prefetch_desc(&P.tm_g);
    ptx::tma_prefetch_desc(&P.tm_b);
    if (!kTied) ptx::tma_prefetch_desc(&P.tm_w);
  }
  if (warp == 0) {
    ptx::tmem_alloc(sb + OFF_MISC + MISC_TMEM, kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(gb + OFF_MISC + MISC_TMEM);
  // TMEM columns: the adjoint Acc (lane = d_k channel i, column = d_v channel j), and three
  // 128-column work areas:
  //   X: G1 -> bf16 R^T (cols 0-31) and -dM^T (32-63) -> [dA dB; dQX dQP] -> [dx_r^T | dp_r^T]
  //   Y: R^T (0-63), M^T (64-127) -> dV^T (0-63)
  //   Z: dM^T (0-63), dR^T (64-127) -> [dk_r^T | dq_r^T]
  const uint32_t tmAcc = tmem, tmX = tmem + 128, tmY = tmem + 256, tmZ = tmem + 384;
  const uint32_t lane_base = (uint32_t)(qd * 32) << 16;
  uint32_t it = 0;     // chunks processed by this CTA: the parity of the MMA barriers
  uint32_t ld_it = 0;  // load phases consumed (a chunk outside the range consumes one, no MMA phase)

  const Tout *g_do = static_cast<const Tout *>(P.dO);
  const __nv_bfloat16 *g_w = kTied ? P.b : P.w;
  Tout *g_dq = static_cast<Tout *>(P.dq), *g_dk = static_cast<Tout *>(P.dk), *g_dv = static_cast<Tout *>(P.dv);
  Tout *g_dla = static_cast<Tout *>(P.dlog_a), *g_db = static_cast<Tout *>(P.db), *g_dw = static_cast<Tout *>(P.dw);

  // the raw k, q, v, log_a, b (, w, dO) tiles of the chunk at token t0 of head h, and its S_r
  // tile image (thread kIssuer)
  constexpr bool kDoTma = sizeof(Tout) == 2;  // bf16 dO lands in its tile as it is
  bool dbg_armed = P.dbg_skip != 0 && blockIdx.x == 0;  // the timeout test hook (thread kIssuer)
  auto issue_loads = [&](int h, int t0, const uint8_t *sr_img) {
    constexpr uint32_t kTiles = 3u + (kDoTma ? 1u : 0u) + (kSD ? 0u : 1u) + (kSG ? 0u : (kTied ? 1u : 2u));
    ptx::mbar_arrive_expect_tx(bar(BAR_LD), kTiles * 16384u + (uint32_t)kSlotBytes);
    *sIss = *sIss + 1u;
    if (dbg_armed) {  // bytes announced, no copy issued: the wait for this group runs out
      dbg_armed = false;
      return;
    }
    ptx::bulk_load(sb + OFF_SR, sr_img, 32768u, bar(BAR_LD));
    ptx::bulk_load(sb + OFF_T, sr_img + 32768, 8192u, bar(BAR_LD));
#pragma unroll
    for (int kb = 0; kb < 2; ++kb) {
      const uint32_t o = (uint32_t)kb * 16384u;
      ptx::tma_load_3d(sb + OFF_KQ + o, &P.tm_k, kb * 64, h, t0, bar(BAR_LD));
      ptx::tma_load_3d(sb + OFF_KQ + o + 8192u, &P.tm_q, kb * 64, h, t0, bar(BAR_LD));
      ptx::tma_load_3d(sb + OFF_MV + o + 8192u, &P.tm_v, kb * 64, h, t0, bar(BAR_LD));
      if (!kSD) ptx::tma_load_3d(sb + OFF_GRAW + (uint32_t)kb * 8192u, &P.tm_g, kb * 64, h, t0, bar(BAR_LD));
      if (!kSG) {
        ptx::tma_load_3d(sb + OFF_XP + o, &P.tm_b, kb * 64, h, t0, bar(BAR_LD));
        if (!kTied) ptx::tma_load_3d(sb + OFF_XP + o + 8192u, &P.tm_w, kb * 64, h, t0, bar(BAR_LD));
      }
      if (kDoTma) ptx::tma_load_3d(sb + OFF_RO + o + 8192u, &P.tm_do, kb * 64, h, t0, bar(BAR_LD));
    }
  };

  for (;;) {
    if (tid == 0) *sUnit = atomicAdd(P.counter, 1);
    __syncthreads();
    const int u = *sUnit;
    if (u >= P.n_units || *sAbort) break;
    const int unit = P.schedule ? P.schedule[u] : u;
    const int n = unit / H, h = unit % H;
    int64_t bos, len;
    if (P.cu_seqlens) {
      bos = P.cu_seqlens[n];
      len = (int64_t)P.cu_seqlens[n + 1] - bos;
    } else {
      bos = (int64_t)n * P.seq_len;
      len = P.seq_len;
    }
    const int nchunks = (int)((len + C - 1) / C);
    const uint8_t *ck_unit = P.ckpt + ckpt_first_slot(P.ckpt_off, n, h, H, nchunks) * kSlotBytes;

    // ---- the final state's adjoint dS_T into TMEM (thread: d_k channel `row`, d_v channels
    //      [32 cg, 32 cg + 32)), and the decay term of the last chunk, sum_j dS_T S_T per d_k
    //      channel (S_T: the forward's final state)
    {
      uint32_t r[32];
      float acc = 0.f;
      const size_t o = ((size_t)unit * D + row) * D + cg * 32;
#pragma unroll
      for (int j4 = 0; j4 < 8; ++j4) {
        const float4 a = P.dS_T ? *reinterpret_cast<const float4 *>(P.dS_T + o + 4 * j4) : make_float4(0.f, 0.f, 0.f, 0.f);
        const float4 st = *reinterpret_cast<const float4 *>(P.S_fin + o + 4 * j4);
        r[4 * j4] = __float_as_uint(a.x);
        r[4 * j4 + 1] = __float_as_uint(a.y);
        r[4 * j4 + 2] = __float_as_uint(a.z);
        r[4 * j4 + 3] = __float_as_uint(a.w);
        acc += a.x * st.x + a.y * st.y + a.z * st.z + a.w * st.w;
      }
      ptx::tmem_st32(tmAcc + lane_base + cg * 32, r);
      ptx::tmem_wait_st();
      rs[cg * 128 + row] = acc;
      if (tid < 128) sEsr[((it & 1u) ^ 1u) * 128 + tid] = 1.f;  // the last chunk reads dS_T unscaled
      // the last chunk's tiles (every tile is free: the previous unit's MMAs are done)
      if (tid == kIssuer && nchunks > 0 && !*sAbort)
        issue_loads(h, (int)(bos + (int64_t)(nchunks - 1) * C), ck_unit + (size_t)(nchunks - 1) * kSlotBytes);
    }
    __syncthreads();
    if (tid < 128)
      sDlc[(it & 1u) * 128 + tid] = ((rs[tid] + rs[128 + tid]) + rs[256 + tid]) + rs[384 + tid];

    bool unit_ok = true;
    int lastpar = -1;  // parity of the last chunk processed (chunk 0): its e^{rho} gives dS0
    float scal_pre = 0.f;  // scalar flags: this thread's value of the chunk processed next
    for (int ci = nchunks - 1; ci >= 0; --ci) {
      const uint32_t par = it & 1u;
      const int t0 = (int)(bos + (int64_t)ci * C);
      const int nvalid = (int)((len - (int64_t)ci * C) < C ? (len - (int64_t)ci * C) : C);

      // ================= phase 1: loads, cumulative decay, operand tiles
      if (kSD || kSG) {  // the chunk's scalar log_a and / or b, w (zero past the chunk end)
        const int which = tid >> 6, r = tid & 63;
        const bool mine = tid < 192 && (which == 0 ? kSD : kSG);
        const __nv_bfloat16 *src = which == 0 ? P.log_a : (which == 1 || kTied) ? P.b : g_w;
        if (mine) {  // the unit's first chunk fetches its own; later ones were requested a chunk ago
          sScal[tid] = ci == nchunks - 1 ? (r < nvalid ? bf(src[(size_t)(t0 + r) * H + h]) : 0.f) : scal_pre;
        }
        __syncthreads();
        // the next chunk to process (ci - 1, a full chunk): requested now, stored at its start
        if (mine && ci > 0) scal_pre = bf(src[(size_t)(t0 - C + r) * H + h]);
      }
      // fp32 dO: the rows of channel `row` into the bf16 tile (rows past the chunk end re-read
      // its last row and are zeroed); the dO rows of the tile are free since the previous
      // chunk's products.  bf16 dO arrives with the other tiles.
      if (!kDoTma) {
        Tout dov[16];
#pragma unroll
        for (int t = 0; t < 16; ++t) {
          const int r = 16 * cg + t, rc = r < nvalid ? r : nvalid - 1;
          dov[t] = g_do[((size_t)(t0 + rc) * H + h) * D + row];
        }
#pragma unroll
        for (int t = 0; t < 16; ++t) {
          const int r = 16 * cg + t;
          sts_u16(sb + OFF_RO + 8192u + swz_elem(r, row, 16384u), bf16_bits(r < nvalid ? to_f32<Tout>(dov[t]) : 0.f));
        }
      }
      waitb(bar(BAR_LD), ld_it & 1u);
      ++ld_it;
      // cumulative log-decay, thread: channels 4 lane .. 4 lane + 3, rows 4 warp .. 4 warp + 3
      // (8-byte accesses); rows past the chunk end decay by nothing and their V and dO rows
      // are zeroed.  Row-group sums go to a [16][128] scratch in the [B; QP] tile (free until
      // the masks).
      float *part16 = reinterpret_cast<float *>(gb + OFF_BQP);
      const int e_kb = lane >> 4;
      const uint32_t e_ch16 = (uint32_t)((lane & 15) >> 1), e_cofs = (uint32_t)(lane & 1) * 8u;
      float4 L4[4];
      {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int rr = 0; rr < 4; ++rr) {
          const int r = warp * 4 + rr;
          float4 g4 = make_float4(0.f, 0.f, 0.f, 0.f);
          if (r < nvalid) {
            if (kSD) {
              const float sv = sScal[r];
              g4 = make_float4(sv, sv, sv, sv);
            } else {
              g4 = unpack4(lds_v2(sb + OFF_GRAW + (uint32_t)e_kb * 8192u + swz(r, e_ch16) + e_cofs));
            }
          } else {
            const uint32_t o = (uint32_t)e_kb * 16384u + 8192u + swz(r, e_ch16) + e_cofs;
            sts_v2(sb + OFF_MV + o, make_uint2(0u, 0u));
            if (kDoTma) sts_v2(sb + OFF_RO + o, make_uint2(0u, 0u));
          }
          acc.x += g4.x; acc.y += g4.y; acc.z += g4.z; acc.w += g4.w;
          L4[rr] = acc;
        }
        *reinterpret_cast<float4 *>(part16 + warp * 128 + 4 * lane) = acc;
        if (warp == 0) *reinterpret_cast<float4 *>(sL0 + 4 * lane) = L4[0];
      }
      if (tid == 0) *sWide = 0;
      __syncthreads();
      {
        // per channel c: exclusive prefixes over the 16 row groups, L_ref, the range check.
        // Channel-wise decay: four adjacent lanes per channel take 4 groups each and scan their
        // totals with shuffles; scalar decay: one thread per channel walks the 16 groups (each
        // form measured the faster one for its case).
        if (kSD) {
          if (tid < D) {
            const int c = tid;
            float run = 0.f;
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const float pj = part16[j * 128 + c];
              part16[j * 128 + c] = run;
              if ((j & 3) == 0) lpre[(j >> 2) * 128 + c] = run;
              run += pj;
            }
            const float l0 = sL0[c];
            const float rho = 0.5f * (l0 + run);
            if (!(l0 - run <= kFastSpan)) *sWide = 1;
            sRho[c] = rho;
            sGam[c] = ptx::ex2((run - rho) * kLog2eF);
            sEsr[par * 128 + c] = ptx::ex2(rho * kLog2eF);
          }
        } else {
          const int c = tid >> 2, g4 = tid & 3;
          float v[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) v[j] = part16[(4 * g4 + j) * 128 + c];
          const float tl = ((v[0] + v[1]) + v[2]) + v[3];
          float incl = tl;
          const float u1 = __shfl_up_sync(0xffffffffu, incl, 1, 4);
          if (g4 >= 1) incl += u1;
          const float u2 = __shfl_up_sync(0xffffffffu, incl, 2, 4);
          if (g4 >= 2) incl += u2;
          const float run = __shfl_sync(0xffffffffu, incl, 3, 4);  // the channel's total L_63
          float pre4 = incl - tl;
          lpre[g4 * 128 + c] = pre4;  // the epilogue's 16-row groups
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            part16[(4 * g4 + j) * 128 + c] = pre4;
            pre4 += v[j];
          }
          if (g4 == 3) {
            const float l0 = sL0[c];
            const float rho = 0.5f * (l0 + run);
            if (!(l0 - run <= kFastSpan)) *sWide = 1;
            sRho[c] = rho;
            sGam[c] = ptx::ex2((run - rho) * kLog2eF);
            sEsr[par * 128 + c] = ptx::ex2(rho * kLog2eF);
          }
        }
      }
      __syncthreads();
      // k_r, q_r, x_r, p_r over the raw k, q, b, w rows (zero past the chunk end)
      {
        const float4 off = *reinterpret_cast<const float4 *>(part16 + warp * 128 + 4 * lane);
        const float4 ref = *reinterpret_cast<const float4 *>(sRho + 4 * lane);
        const float4 base = make_float4((off.x - ref.x) * kLog2eF, (off.y - ref.y) * kLog2eF,
                                        (off.z - ref.z) * kLog2eF, (off.w - ref.w) * kLog2eF);
#pragma unroll
        for (int rr = 0; rr < 4; ++rr) {
          const int r = warp * 4 + rr;
          const uint32_t o0 = (uint32_t)e_kb * 16384u + swz(r, e_ch16) + e_cofs, o1 = o0 + 8192u;
          const float l0 = fmaf(L4[rr].x, kLog2eF, base.x), l1 = fmaf(L4[rr].y, kLog2eF, base.y);
          const float l2 = fmaf(L4[rr].z, kLog2eF, base.z), l3 = fmaf(L4[rr].w, kLog2eF, base.w);
          const float4 e = make_float4(ptx::ex2(l0), ptx::ex2(l1), ptx::ex2(l2), ptx::ex2(l3));
          const float4 f = make_float4(ptx::ex2(-l0), ptx::ex2(-l1), ptx::ex2(-l2), ptx::ex2(-l3));
          float4 kk = make_float4(0.f, 0.f, 0.f, 0.f), qq = kk, bb = kk, ww = kk;
          if (r < nvalid) {
            kk = unpack4(lds_v2(sb + OFF_KQ + o0));
            qq = unpack4(lds_v2(sb + OFF_KQ + o1));
            if (kSG) {
              const float sbv = sScal[64 + r], swv = sScal[128 + r];
              bb = make_float4(sbv, sbv, sbv, sbv);
              ww = make_float4(swv, swv, swv, swv);
            } else {
              bb = unpack4(lds_v2(sb + OFF_XP + o0));
              ww = kTied ? bb : unpack4(lds_v2(sb + OFF_XP + o1));
            }
          }
          const float4 kf = make_float4(kk.x * f.x, kk.y * f.y, kk.z * f.z, kk.w * f.w);
          sts_v2(sb + OFF_KQ + o1, pack4(qq.x * e.x, qq.y * e.y, qq.z * e.z, qq.w * e.w));
          if (kP3) {  // k_r = (b.k) e, x_r = p_r = k f, V = w.v (d_v channels, the same 4 columns)
            sts_v2(sb + OFF_KQ + o0, pack4(bb.x * kk.x * e.x, bb.y * kk.y * e.y, bb.z * kk.z * e.z, bb.w * kk.w * e.w));
            const uint2 kfp = pack4(kf.x, kf.y, kf.z, kf.w);
            sts_v2(sb + OFF_XP + o0, kfp);
            sts_v2(sb + OFF_XP + o1, kfp);
            const float4 vv = unpack4(lds_v2(sb + OFF_MV + o0 + 8192u));
            sts_v2(sb + OFF_MV + o0 + 8192u, pack4(vv.x * ww.x, vv.y * ww.y, vv.z * ww.z, vv.w * ww.w));
          } else {
            sts_v2(sb + OFF_KQ + o0, pack4(kk.x * e.x, kk.y * e.y, kk.z * e.z, kk.w * e.w));
            sts_v2(sb + OFF_XP + o0, pack4(bb.x * kf.x, bb.y * kf.y, bb.z * kf.z, bb.w * kf.w));
            sts_v2(sb + OFF_XP + o1, pack4(ww.x * kf.x, ww.y * kf.y, ww.z * kf.z, ww.w * kf.w));
          }
        }
      }
      // Lam_g = Diag(gamma e^{rho_next}) Acc, the bf16 tile [d_k rows][d_v] and the fp32 base of
      // this chunk's adjoint update (thread: d_k channel `row`, d_v channels [32 cg, 32 cg + 32))
      {
        const float gam = sGam[row];
        const float efac = sEsr[(par ^ 1u) * 128 + row];
        uint32_t r[32];
        float lg[32];
        ptx::tmem_ld32(tmAcc + lane_base + cg * 32, r);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          lg[j] = (__uint_as_float(r[j]) * efac) * gam;  // e^{rho_next} first: the adjoint, O(1)
          r[j] = __float_as_uint(lg[j]);
        }
        ptx::tmem_st32(tmAcc + lane_base + cg * 32, r);
#pragma unroll
        for (int q8 = 0; q8 < 4; ++q8)
          sts_v4(sb + OFF_LG + (uint32_t)(cg >> 1) * 16384u + swz(row, (uint32_t)((cg & 1) * 4 + q8)), pack8(lg + 8 * q8, 1.f));
        ptx::tmem_wait_st();
      }
      ptx::fence_proxy_async_smem();
      ptx::tc_fence_before();
      __syncthreads();
      if (*sWide || *sAbort) {
        // outside the factored form (recorded unless an earlier error was), or a timed-out
        // wait: the rest of the unit is left
        if (tid == 0 && !*sAbort) atomicCAS(P.status, 0, kStatusRange);
        unit_ok = false;
        break;
      }

      // ================= phase 2: G1, and the products that need no mask: dM^T = Lam_g^T x_r^T
      //      and the S_r part of R^T = S_r^T k_r^T; the masks of G1
      if (tid == kIssuer && !*sAbort) {
        ptx::tc_fence_after();
        constexpr uint32_t idG1 = ptx::idesc_bf16(128, 128, false, false);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) ptx::umma_bf16(tmX, kmaj(sb + OFF_KQ, kk), kmaj(sb + OFF_XP, kk), idG1, kk > 0);
        ptx::umma_commit(bar(BAR_G1));
        constexpr uint32_t idM = ptx::idesc_bf16(128, 64, true, false);  // A MN-major (Lam_g^T, S_r^T)
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) ptx::umma_bf16(tmZ, mnmaj(sb + OFF_LG, kk), kmaj(sb + OFF_XP, kk), idM, kk > 0);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) ptx::umma_bf16(tmY, mnmaj(sb + OFF_SR, kk), kmaj(sb + OFF_KQ, kk), idM, kk > 0);
      }
      waitb(bar(BAR_G1), par);
      ptx::tc_fence_after();
      if (!(row < 64 && cg < 2)) {
        // warp (qd, cg) reads G1 row `row`, columns [32 cg, 32 cg + 32): B for rows 0-63 (strictly
        // lower), QX | QP for rows 64-127 (lower with the diagonal); A is not needed (T came
        // from the forward)
        uint32_t r[32];
        ptx::tmem_ld32(tmX + lane_base + cg * 32, r);
        ptx::tmem_wait_ld();
        const int i = row & 63, jb = (cg & 1) * 32;
        const bool strict = row < 64;
        float f[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) f[j] = (strict ? jb + j < i : jb + j <= i) ? __uint_as_float(r[j]) : 0.f;
        // B into rows 0-63 of [B; QP]; QX into its own tile; QP into rows 64-127 of [B; QP]
        const uint32_t dst = strict ? sb + OFF_BQP : (cg < 2 ? sb + OFF_QX : sb + OFF_BQP + 8192u);
#pragma unroll
        for (int q8 = 0; q8 < 4; ++q8) sts_v4(dst + swz(i, (uint32_t)((cg & 1) * 4 + q8)), pack8(f + 8 * q8, 1.f));
        ptx::fence_proxy_async_smem();
      }
      ptx::tc_fence_before();
      __syncthreads();

      // ================= phase 3: the masked products: R^T += V^T B^T, dM^T += dO^T QX
      if (tid == kIssuer && !*sAbort) {
        ptx::tc_fence_after();
        constexpr uint32_t idV = ptx::idesc_bf16(128, 64, true, false);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          ptx::umma_bf16(tmY, ptx::sdesc_sw128(sb + OFF_MV + 8192u + (uint32_t)kk * 2048u, 16384, 1024),
                         ptx::sdesc_sw128(sb + OFF_BQP + (uint32_t)kk * 32u, 16, 1024), idV, 1);
        // QX as [s][t]: MN-major B
        constexpr uint32_t idQ = ptx::idesc_bf16(128, 64, true, true);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          ptx::umma_bf16(tmZ, ptx::sdesc_sw128(sb + OFF_RO + 8192u + (uint32_t)kk * 2048u, 16384, 1024),
                         ptx::sdesc_sw128(sb + OFF_QX + (uint32_t)kk * 2048u, 8192, 1024), idQ, 1);
        ptx::umma_commit(bar(BAR_GA));
      }

      // ================= phase 4: R^T and -dM^T as bf16 TMEM operands; M^T, dR^T
      waitb(bar(BAR_GA), par);
      ptx::tc_fence_after();
      {
        uint32_t r[16], hb[8];
        ptx::tmem_ld16(tmY + lane_base + cg * 16, r);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 8; ++j) hb[j] = pack_bf16x2(__uint_as_float(r[2 * j]), __uint_as_float(r[2 * j + 1]));
        ptx::tmem_st8(tmX + lane_base + cg * 8, hb);
        ptx::tmem_ld16(tmZ + lane_base + cg * 16, r);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 8; ++j) hb[j] = pack_bf16x2(-__uint_as_float(r[2 * j]), -__uint_as_float(r[2 * j + 1]));
        ptx::tmem_st8(tmX + 32 + lane_base + cg * 8, hb);
        ptx::tmem_wait_st();
      }
      ptx::tc_fence_before();
      __syncthreads();
      if (tid == kIssuer && !*sAbort) {
        ptx::tc_fence_after();
        // M^T = R^T T^T (B = T as [t][s], K-major); dR^T = dM^T T (B = T as [s][t], MN-major)
        constexpr uint32_t idK = ptx::idesc_bf16(128, 64, false, false);
        constexpr uint32_t idN = ptx::idesc_bf16(128, 64, false, true);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          ptx::umma_bf16_ts(tmY + 64, tmX + (uint32_t)kk * 8u, ptx::sdesc_sw128(sb + OFF_T + (uint32_t)kk * 32u, 16, 1024),
                            idK, kk > 0);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          ptx::umma_bf16_ts(tmZ + 64, tmX + 32u + (uint32_t)kk * 8u,
                            ptx::sdesc_sw128(sb + OFF_T + (uint32_t)kk * 2048u, 8192, 1024), idN, kk > 0);
        ptx::umma_commit(bar(BAR_GB));
      }

      // ================= phase 5: -M and dR to their tiles ([t][j], over T, QX and the solve array)
      waitb(bar(BAR_GB), par);
      ptx::tc_fence_after();
      {
        uint32_t r[16];
        ptx::tmem_ld16(tmY + 64 + lane_base + cg * 16, r);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 16; ++j)
          sts_u16(sb + OFF_MV + swz_elem(cg * 16 + j, row, 16384u), bf16_bits(-__uint_as_float(r[j])));
        ptx::tmem_ld16(tmZ + 64 + lane_base + cg * 16, r);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 16; ++j)
          sts_u16(sb + OFF_RO + swz_elem(cg * 16 + j, row, 16384u), bf16_bits(__uint_as_float(r[j])));
      }
      // this thread's S_r values (d_k channel `row`, d_v channels [32 cg, 32 cg + 32)) for the
      // decay term, taken before the barrier after which the gradient tile may overwrite them
      uint4 srv[4];
#pragma unroll
      for (int q8 = 0; q8 < 4; ++q8)
        srv[q8] = lds_v4(sb + OFF_SR + (uint32_t)(cg >> 1) * 16384u + swz(row, (uint32_t)((cg & 1) * 4 + q8)));
      ptx::fence_proxy_async_smem();
      ptx::tc_fence_before();
      __syncthreads();

      // ================= phase 6: the S_r terms [dk_r^T | dq_r^T] = S_r [dR; dO]^T and
      //      [dA dB; dQX dQP] = [dR; dO][-M; V]^T (commit G5: the masks need these, and then S_r's
      //      space is free); the adjoint update Acc += [k_r; q_r]^T [dR; dO] (commit GL: the decay
      //      term and the next chunk need it); dV^T = [dR; dO]^T [B; QP] + Lam_g^T p_r^T (commit
      //      GZ).  The last two run under the masks.
      if (tid == kIssuer && !*sAbort) {
        ptx::tc_fence_after();
        constexpr uint32_t idKK = ptx::idesc_bf16(128, 128, false, false);
        constexpr uint32_t idNN = ptx::idesc_bf16(128, 128, true, true);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) ptx::umma_bf16(tmZ, kmaj(sb + OFF_SR, kk), kmaj(sb + OFF_RO, kk), idKK, kk > 0);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) ptx::umma_bf16(tmX, kmaj(sb + OFF_RO, kk), kmaj(sb + OFF_MV, kk), idKK, kk > 0);
        ptx::umma_commit(bar(BAR_G5));
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) ptx::umma_bf16(tmAcc, mnmaj(sb + OFF_KQ, kk), mnmaj(sb + OFF_RO, kk), idNN, 1);
        ptx::umma_commit(bar(BAR_GL));
        constexpr uint32_t idV1 = ptx::idesc_bf16(128, 64, true, true);
        constexpr uint32_t idV2 = ptx::idesc_bf16(128, 64, true, false);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          ptx::umma_bf16(tmY, mnmaj(sb + OFF_RO, kk), ptx::sdesc_sw128(sb + OFF_BQP + (uint32_t)kk * 2048u, 8192, 1024),
                         idV1, kk > 0);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) ptx::umma_bf16(tmY, mnmaj(sb + OFF_LG, kk), kmaj(sb + OFF_XP + 8192u, kk), idV2, 1);
        ptx::umma_commit(bar(BAR_GZ));
      }

      // ================= phase 7: the gradient-tile masks (over S_r's space: every thread took
      //      its S_r values for the decay term before the barrier that ended phase 5)
      waitb(bar(BAR_G5), par);
      ptx::tc_fence_after();
      {
        // row `row` of [dA dB; dQX dQP], columns [32 cg, 32 cg + 32): strictly lower for the dR
        // rows, lower with the diagonal for the dO rows; stored as [column block][row][64]
        uint32_t r[32];
        ptx::tmem_ld32(tmX + lane_base + cg * 32, r);
        ptx::tmem_wait_ld();
        const int i = row & 63, jb = (cg & 1) * 32;
        const bool strict = row < 64;
        float f[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) f[j] = (strict ? jb + j < i : jb + j <= i) ? __uint_as_float(r[j]) : 0.f;
#pragma unroll
        for (int q8 = 0; q8 < 4; ++q8)
          sts_v4(sb + OFF_DG + (uint32_t)(cg >> 1) * 16384u + swz(row, (uint32_t)((cg & 1) * 4 + q8)), pack8(f + 8 * q8, 1.f));
      }
      ptx::fence_proxy_async_smem();
      ptx::tc_fence_before();
      __syncthreads();

      // ================= phase 8: [dx_r^T | dp_r^T] = [k_r; q_r]^T dG + Lam_g [-M; V]^T,
      //      [dk_r^T | dq_r^T] += [x_r; p_r]^T dG^T
      if (tid == kIssuer && !*sAbort) {
        ptx::tc_fence_after();
        constexpr uint32_t idNN = ptx::idesc_bf16(128, 128, true, true);
        constexpr uint32_t idKK = ptx::idesc_bf16(128, 128, false, false);
        constexpr uint32_t idNK = ptx::idesc_bf16(128, 128, true, false);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) ptx::umma_bf16(tmX, mnmaj(sb + OFF_KQ, kk), mnmaj(sb + OFF_DG, kk), idNN, kk > 0);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) ptx::umma_bf16(tmX, kmaj(sb + OFF_LG, kk), kmaj(sb + OFF_MV, kk), idKK, 1);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) ptx::umma_bf16(tmZ, mnmaj(sb + OFF_XP, kk), kmaj(sb + OFF_DG, kk), idNK, 1);
        ptx::umma_commit(bar(BAR_G7));
      }
      // the raw inputs of the epilogue's rows [c0, c0 + 8) (channel `row`): the first half's are
      // requested while the last products run, the second half's once the first half's chain
      // rule is done; rows past the chunk end re-read its last row and are ignored.  Scalar
      // log_a, b, w come from shared memory; the gist.science placement needs no w here.
      // (2-byte loads: 16-byte loads of 8 channels with a transpose after them were slower.)
      __nv_bfloat16 rla[8], rk[8], rq[8], rb[8], rw[8];
      auto load_raw = [&](int c0) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int t = c0 + j, tc = t < nvalid ? t : nvalid - 1;
          const size_t gi = ((size_t)(t0 + tc) * H + h) * D + row;
          rk[j] = P.k[gi];
          rq[j] = P.q[gi];
          if (!kSD) rla[j] = P.log_a[gi];
          if (!kSG) {
            rb[j] = P.b[gi];
            if (!kP3) rw[j] = kTied ? rb[j] : g_w[gi];
          }
        }
      };
      // Gradient rows out: the thread holds one channel (`row`) of 8 consecutive tokens
      // [c0, c0 + 8).  bf16: after an 8 x 8 transpose inside each 8-lane group, lane m writes
      // token c0 + m for the group's 8 channels with one 16-byte store; fp32: one store per
      // element.  Tokens past the chunk end are not written.
      auto store8 = [&](Tout *g, const float (&v)[8], int c0) {
        if constexpr (sizeof(Tout) == 2) {
          uint32_t w[4] = {pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                           pack_bf16x2(v[6], v[7])};
          transpose8x8_bf16(w, lane);
          const int t = c0 + (lane & 7);
          if (t < nvalid)
            *reinterpret_cast<uint4 *>(g + ((size_t)(t0 + t) * H + h) * D + (row - (lane & 7))) =
                make_uint4(w[0], w[1], w[2], w[3]);
        } else {
#pragma unroll
          for (int j = 0; j < 8; ++j)
            if (c0 + j < nvalid) g[((size_t)(t0 + c0 + j) * H + h) * D + row] = from_f32<Tout>(v[j]);
        }
      };
      load_raw(cg * 16);
      waitb(bar(BAR_GL), par);  // the adjoint is final for this chunk
      ptx::tc_fence_after();
      if (ci > 0) {
        // the decay term of chunk ci - 1 (processed next): sum_j Lam_{c-1}[i][j] S_c[i][j] =
        // sum_j Acc[i][j] S_r[i][j] (Lam_{c-1} = e^{rho} Acc); thread (d_k channel `row`, d_v
        // channels [32 cg, 32 cg + 32)), summed over the four column groups after the next barrier
        uint32_t r[32];
        ptx::tmem_ld32(tmAcc + lane_base + cg * 32, r);
        ptx::tmem_wait_ld();
        float acc = 0.f;
#pragma unroll
        for (int q8 = 0; q8 < 4; ++q8) {
          const uint32_t w4[4] = {srv[q8].x, srv[q8].y, srv[q8].z, srv[q8].w};
#pragma unroll
          for (int e2 = 0; e2 < 4; ++e2) {
            const float2 f = unpack_bf16x2(w4[e2]);
            acc = fmaf(__uint_as_float(r[8 * q8 + 2 * e2]), f.x, acc);
            acc = fmaf(__uint_as_float(r[8 * q8 + 2 * e2 + 1]), f.y, acc);
          }
        }
        rs[cg * 128 + row] = acc;
      }
      waitb(bar(BAR_GZ), par);  // dV^T is done: it goes out while the last products run
      ptx::tc_fence_after();
      // dV: thread d_v channel `row`, tokens [16 cg, 16 cg + 16).  dZ is the gradient of the
      // values as they enter (v, or w.v in the gist.science placement: dv = w dZ, and v dZ goes
      // to the value gate: out as dw, or kept for db (tied) or the channel sums (scalar))
      float vdz[16];
      {
        uint32_t r[16];
        ptx::tmem_ld16(tmY + lane_base + cg * 16, r);
        float vr[16], wr[16];
        if (kP3) {
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int t = cg * 16 + j, tc = t < nvalid ? t : nvalid - 1;
            const size_t gi = ((size_t)(t0 + tc) * H + h) * D + row;
            vr[j] = bf(P.v[gi]);
            wr[j] = kSG ? sScal[128 + t] : bf((kTied ? P.b : g_w)[gi]);
          }
        }
        ptx::tmem_wait_ld();
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          float dv8[8], dw8[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const int jj = hf * 8 + j;
            const bool valid = cg * 16 + jj < nvalid;
            const float dz = __uint_as_float(r[jj]);
            vdz[jj] = (kP3 && valid) ? vr[jj] * dz : 0.f;
            dv8[j] = kP3 ? wr[jj] * dz : dz;
            dw8[j] = vdz[jj];
          }
          store8(g_dv, dv8, cg * 16 + hf * 8);
          if (kP3 && !kTied && !kSG) store8(g_dw, dw8, cg * 16 + hf * 8);
        }
      }
      waitb(bar(BAR_G7), par);
      ptx::tc_fence_after();
      // every tile is free (the epilogue reads TMEM and global memory only): the next chunk's
      // raw tiles land while this chunk's gradients are formed and stored
      if (tid == kIssuer && ci > 0 && !*sAbort) issue_loads(h, t0 - C, ck_unit + (size_t)(ci - 1) * kSlotBytes);

      // ================= phase 9: chain rule and stores.  Thread: d_k channel i = `row`, tokens
      //      [16 cg, 16 cg + 16).  The cumulative decay is recomputed as phase 1 computed it.
      //      Per channel: dx = dx_r e^{L_ref - L}, dp = dp_r e^{L_ref - L}, and
      //        default placement:     dk = dk_r e^{L - L_ref} + b dx + w dp,  db = k dx,  dw = k dp;
      //        gist.science placement: dy = dk_r e^{L - L_ref} (y = b.k), dk = b dy + dx + dp,
      //                                db = k dy (+ v dZ of the same channel when tied);
      //      scalar gates and decay take the channel sums of db, dw, d log_a.
      {
        const int i = row;
        const float pre = lpre[cg * 128 + i], rho = sRho[i], dlc = sDlc[par * 128 + i];
        float dL[16], gbv[16], gwv[16];
        float loc = 0.f;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          const int c0 = cg * 16 + half * 8;
          uint32_t vx[8], vp[8], vk[8], vq[8];
          ptx::tmem_ld8(tmX + lane_base + (uint32_t)c0, vx);
          ptx::tmem_ld8(tmX + lane_base + 64u + (uint32_t)c0, vp);
          ptx::tmem_ld8(tmZ + lane_base + (uint32_t)c0, vk);
          ptx::tmem_ld8(tmZ + lane_base + 64u + (uint32_t)c0, vq);
          ptx::tmem_wait_ld();
          float dq8[8], dk8[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const int t = c0 + j, jj = half * 8 + j;
            const bool valid = t < nvalid;
            const float kk = valid ? bf(rk[j]) : 0.f, qq = valid ? bf(rq[j]) : 0.f;
            const float la = kSD ? sScal[t] : (valid ? bf(rla[j]) : 0.f);
            const float bb = kSG ? sScal[64 + t] : (valid ? bf(rb[j]) : 0.f);
            const float ww = kP3 ? 0.f : kSG ? sScal[128 + t] : (valid ? bf(rw[j]) : 0.f);
            loc += la;
            const float L = pre + loc;
            const float e = ptx::ex2((L - rho) * kLog2eF), f = ptx::ex2((rho - L) * kLog2eF);
            const float dxr = __uint_as_float(vx[j]), dpr = __uint_as_float(vp[j]);
            const float dkr = __uint_as_float(vk[j]), dqr = __uint_as_float(vq[j]);
            const float dx = dxr * f, dp = dpr * f;
            float dLt, dkv;
            if (kP3) {
              const float dy = dkr * e;
              dLt = e * (dqr * qq + dkr * bb * kk) - f * kk * (dxr + dpr);
              dkv = bb * dy + dx + dp;
              gbv[jj] = kk * dy + (kTied ? vdz[jj] : 0.f);
              gwv[jj] = vdz[jj];
            } else {
              dLt = e * (dqr * qq + dkr * kk) - f * kk * (dxr * bb + dpr * ww);
              dkv = dkr * e + bb * dx + ww * dp;
              gbv[jj] = kTied ? kk * (dx + dp) : kk * dx;
              gwv[jj] = kk * dp;
            }
            if (t == C - 1) dLt += dlc;
            dL[jj] = dLt;
            dq8[j] = dqr * e;
            dk8[j] = dkv;
          }
          // the second half's raw rows, requested while this half's gradients go out (the
          // first half's were requested before the adjoint wait)
          if (half == 0) load_raw(c0 + 8);
          store8(g_dq, dq8, c0);
          store8(g_dk, dk8, c0);
          if (!kSG) {
            float b8[8], w8[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              b8[j] = gbv[half * 8 + j];
              w8[j] = gwv[half * 8 + j];
            }
            store8(g_db, b8, c0);
            if (!kTied && !kP3) store8(g_dw, w8, c0);
          }
        }
        if (kSG) {  // db, dw channel sums: over the warp's 32 channels, then the lane quadrants
          float v[32];
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            v[j] = gbv[j];
            v[16 + j] = gwv[j];
          }
          red[(qd * 3 + (lane >> 4)) * 64 + cg * 16 + (lane & 15)] = warp_colsum32(v);
        }
        // d log_a_s = sum_{t >= s} dL_t: suffix sums inside the thread's 16 rows, then the
        // totals of the later row groups
        float suf = 0.f;
#pragma unroll
        for (int j = 15; j >= 0; --j) {
          suf += dL[j];
          dL[j] = suf;
        }
        part[cg * 128 + i] = suf;
        __syncthreads();
        if (ci > 0 && tid < 128)  // the decay term of chunk ci - 1 (rs is complete)
          sDlc[(par ^ 1u) * 128 + tid] = ((rs[tid] + rs[128 + tid]) + rs[256 + tid]) + rs[384 + tid];
        float above = 0.f;
        for (int g = 3; g > cg; --g) above += part[g * 128 + i];
        if (kSD) {  // d log_a: channel sums as for db, dw
          float v[32];
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            v[j] = dL[j] + above;
            v[16 + j] = 0.f;
          }
          const float sum = warp_colsum32(v);
          if (lane < 16) red[(qd * 3 + 2) * 64 + cg * 16 + lane] = sum;
        } else {
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
            float l8[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) l8[j] = dL[hf * 8 + j] + above;
            store8(g_dla, l8, cg * 16 + hf * 8);
          }
        }
        if (kSD || kSG) {
          __syncthreads();
          if (tid < 192) {  // one thread per (quantity, token): db, dw (scalar gates), d log_a (scalar decay)
            const int q = tid >> 6, t = tid & 63;
            const bool want = q == 2 ? kSD : (kSG && !(q == 1 && kTied));
            if (want && t < nvalid) {
              const float tot = ((red[q * 64 + t] + red[(3 + q) * 64 + t]) + red[(6 + q) * 64 + t]) + red[(9 + q) * 64 + t];
              Tout *dst = q == 0 ? g_db : q == 1 ? g_dw : g_dla;
              dst[(size_t)(t0 + t) * H + h] = from_f32<Tout>(tot);
            }
          }
        }
      }
      ptx::tc_fence_before();
      __syncthreads();  // part and the TMEM work areas are reused by the next chunk
      lastpar = (int)par;
      ++it;
      if (*sAbort) break;
    }

    // ---- dS0 = Diag(e^{rho_0}) Acc (the first chunk's adjoint update has landed)
    if (unit_ok && !*sAbort && P.dS0) {
      uint32_t r[32];
      ptx::tmem_ld32(tmAcc + lane_base + cg * 32, r);
      ptx::tmem_wait_ld();
      float4 *dst = reinterpret_cast<float4 *>(P.dS0 + ((size_t)unit * D + row) * D + cg * 32);
      const float es = lastpar >= 0 ? sEsr[lastpar * 128 + row] : 1.f;
#pragma unroll
      for (int j4 = 0; j4 < 8; ++j4)
        dst[j4] = make_float4(__uint_as_float(r[4 * j4]) * es, __uint_as_float(r[4 * j4 + 1]) * es,
                              __uint_as_float(r[4 * j4 + 2]) * es, __uint_as_float(r[4 * j4 + 3]) * es);
    }
    ptx::tc_fence_before();
    __syncthreads();
  }

  if (*sAbort) {
    // wind-down after a timed-out wait: let the MMAs the issuing thread queued finish (bounded)
    // before the tensor memory is freed
    if (tid == kIssuer) {
      ptx::umma_commit(bar(BAR_DRAIN));
      drain_bar(bar(BAR_DRAIN), 0u, P.wait_ns);
      if (*sIss > 0u) drain_bar(bar(BAR_LD), (*sIss - 1u) & 1u, P.wait_ns);  // the last armed load phase
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (warp == 0) ptx::tmem_dealloc(tmem, kTmemCols);
}

// off[n] = sum over m < n of ceil(len_m / 64), off[N] the total: the first checkpoint
// slot of each sequence divided by the head count.  One block; each thread owns a contiguous
// range of sequences.
__global__ void ckpt_offsets_kernel(const int32_t *cu, int N, int64_t *off) {
  __shared__ int64_t sums[1024];
  const int per = (N + (int)blockDim.x - 1) / (int)blockDim.x;
  const int a = (int)threadIdx.x * per, e = a + per < N ? a + per : N;
  int64_t s = 0;
  for (int n = a; n < e; ++n) s += (cu[n + 1] - cu[n] + C - 1) / C;
  sums[threadIdx.x] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    int64_t run = 0;
    for (int i = 0; i < (int)blockDim.x; ++i) {
      const int64_t v = sums[i];
      sums[i] = run;
      run += v;
    }
    off[N] = run;
  }
  __syncthreads();
  int64_t run = sums[threadIdx.x];
  for (int n = a; n < e; ++n) {
    off[n] = run;
    run += (cu[n + 1] - cu[n] + C - 1) / C;
  }
}

template <typename Tout, bool kTied, bool kP3, bool kSD, bool kSG>
cudaError_t launch_t(const BwdTcParams &P, int grid, cudaStream_t stream) {
  auto kern = bwd_tc_kernel<Tout, kTied, kP3, kSD, kSG>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  kern<<<grid, kThreads, kSmemBytes, stream>>>(P);
  return cudaGetLastError();
}

template <typename Tout, bool kP3, bool kSD, bool kSG>
cudaError_t launch_tied(const BwdTcParams &P, int grid, cudaStream_t stream, bool tied) {
  return tied ? launch_t<Tout, true, kP3, kSD, kSG>(P, grid, stream) : launch_t<Tout, false, kP3, kSD, kSG>(P, grid, stream);
}
template <typename Tout, bool kP3>
cudaError_t launch_scalars(const BwdTcParams &P, int grid, cudaStream_t stream, bool tied, bool sd, bool sg) {
  if (sd) return sg ? launch_tied<Tout, kP3, true, true>(P, grid, stream, tied) : launch_tied<Tout, kP3, true, false>(P, grid, stream, tied);
  return sg ? launch_tied<Tout, kP3, false, true>(P, grid, stream, tied) : launch_tied<Tout, kP3, false, false>(P, grid, stream, tied);
}
template <typename Tout>
cudaError_t launch_flags(const BwdTcParams &P, int grid, cudaStream_t stream, bool tied, bool p3, bool sd, bool sg) {
  return p3 ? launch_scalars<Tout, true>(P, grid, stream, tied, sd, sg) : launch_scalars<Tout, false>(P, grid, stream, tied, sd, sg);
}

}  // namespace

size_t bwd_tc_ckpt_slots(int64_t n_seqs, int64_t t_total, int n_heads, bool packed, int seq_len) {
  if (packed) return (size_t)n_heads * (size_t)(t_total / C + n_seqs);  // sum of ceil(len / 64) <= T/64 + N
  return (size_t)n_heads * (size_t)n_seqs * (size_t)((seq_len + C - 1) / C);
}

cudaError_t launch_ckpt_offsets(const int32_t *cu_seqlens, int n_seqs, int64_t *off, cudaStream_t stream) {
  ckpt_offsets_kernel<<<1, 1024, 0, stream>>>(cu_seqlens, n_seqs, off);
  return cudaGetLastError();
}

cudaError_t launch_bwd_tc(const BwdProblem &p, const void *ckpt, const float *S_fin, const int64_t *ckpt_off,
                          const int32_t *schedule, int32_t *status, int32_t *counter, cudaStream_t stream) {
  BwdTcParams P;
  memset(&P, 0, sizeof(P));
  P.q = static_cast<const __nv_bfloat16 *>(p.q);
  P.k = static_cast<const __nv_bfloat16 *>(p.k);
  P.v = static_cast<const __nv_bfloat16 *>(p.v);
  P.log_a = static_cast<const __nv_bfloat16 *>(p.log_a);
  P.b = static_cast<const __nv_bfloat16 *>(p.b);
  P.w = static_cast<const __nv_bfloat16 *>(p.w);
  P.dO = p.dO;
  P.dS_T = p.dS_T;
  P.dq = p.dq; P.dk = p.dk; P.dv = p.dv; P.dlog_a = p.dlog_a; P.db = p.db; P.dw = p.dw;
  P.dS0 = p.dS0;
  P.ckpt = static_cast<const uint8_t *>(ckpt);
  P.S_fin = S_fin;
  P.ckpt_off = ckpt_off;
  P.cu_seqlens = p.cu_seqlens;
  P.schedule = schedule;
  P.status = status;
  P.counter = counter;
  P.n_units = p.n_seqs * p.n_heads;
  P.n_heads = p.n_heads;
  P.seq_len = p.seq_len;
  P.wait_ns = kWaitTimeoutNs;
  if (P.n_units == 0) return cudaSuccess;
  uint64_t hook_ns = 0;
  if (take_debug_timeout(GDN2_DEBUG_BWD, &hook_ns)) {  // the timeout test hook, armed for this launch
    P.dbg_skip = 1;
    P.wait_ns = hook_ns;
  }
  const bool tied = (p.flags & GDN2_TIED_GATES) != 0;
  const int64_t T = p.t_total > 0 ? p.t_total : 1;
  const bool sd_m = (p.flags & GDN2_SCALAR_DECAY) != 0, sg_m = (p.flags & GDN2_SCALAR_GATES) != 0;
  bool ok = make_row_tile_map(&P.tm_q, p.q, T, p.n_heads) && make_row_tile_map(&P.tm_k, p.k, T, p.n_heads) &&
            make_row_tile_map(&P.tm_v, p.v, T, p.n_heads);
  if (ok && !sd_m) ok = make_row_tile_map(&P.tm_g, p.log_a, T, p.n_heads);
  if (ok && !sg_m) ok = make_row_tile_map(&P.tm_b, p.b, T, p.n_heads);
  if (ok && !sg_m && !tied) ok = make_row_tile_map(&P.tm_w, p.w, T, p.n_heads);
  if (ok && p.dtype_out == GDN2_BF16) ok = make_row_tile_map(&P.tm_do, p.dO, T, p.n_heads);
  if (!ok) return cudaErrorInvalidValue;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = P.n_units < sms ? P.n_units : sms;
  const bool p3 = (p.flags & GDN2_GATE_FORM_P3) != 0;
  const bool sd = (p.flags & GDN2_SCALAR_DECAY) != 0, sg = (p.flags & GDN2_SCALAR_GATES) != 0;
  if (p.dtype_out == GDN2_BF16) return launch_flags<__nv_bfloat16>(P, grid, stream, tied, p3, sd, sg);
  return launch_flags<float>(P, grid, stream, tied, p3, sd, sg);
}

// ---------------------------------------------------------------- fused prologue (GDN2_FUSED_PROLOGUE)
// gdn2_chunk_bwd with the prologue flag runs the chunked backward on activated copies of the
// inputs and applies the activations' chain rule to its gradients afterwards; both passes are
// elementwise over (token, head) rows, one warp per row, lane l holding channels 4 l .. 4 l + 3.
namespace {

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int sh = 16; sh >= 1; sh >>= 1) v += __shfl_xor_sync(0xffffffffu, v, sh);
  return v;
}
__device__ __forceinline__ float4 ld4(const __nv_bfloat16 *p) {
  return tc::unpack4(*reinterpret_cast<const uint2 *>(p));
}
__device__ __forceinline__ void st4(__nv_bfloat16 *p, float4 v) {
  *reinterpret_cast<uint2 *>(p) = tc::pack4(v.x, v.y, v.z, v.w);
}
template <typename T>
__device__ __forceinline__ float4 ld4t(const T *p);
template <>
__device__ __forceinline__ float4 ld4t<float>(const float *p) { return *reinterpret_cast<const float4 *>(p); }
template <>
__device__ __forceinline__ float4 ld4t<__nv_bfloat16>(const __nv_bfloat16 *p) { return ld4(p); }
template <typename T>
__device__ __forceinline__ void st4t(T *p, float4 v);
template <>
__device__ __forceinline__ void st4t<float>(float *p, float4 v) { *reinterpret_cast<float4 *>(p) = v; }
template <>
__device__ __forceinline__ void st4t<__nv_bfloat16>(__nv_bfloat16 *p, float4 v) { st4(p, v); }

// Activated bf16 copies: q / |q|, k / |k| (|x| = sqrt(sum x^2 + kNormEps)), log sigmoid(log_a),
// sigmoid(b), sigmoid(w); inv[2 row] = 1/|q|, inv[2 row + 1] = 1/|k|.
__global__ void prolog_act_kernel(const __nv_bfloat16 *q, const __nv_bfloat16 *k, const __nv_bfloat16 *la,
                                  const __nv_bfloat16 *b, const __nv_bfloat16 *w, int64_t rows, bool sd, bool sg,
                                  __nv_bfloat16 *qa, __nv_bfloat16 *ka, __nv_bfloat16 *laa, __nv_bfloat16 *ba,
                                  __nv_bfloat16 *wa, float *inv) {
  const int64_t row = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const size_t o = (size_t)row * 128 + 4 * lane;
  const float4 qq = ld4(q + o), kk = ld4(k + o);
  const float iq = rsqrtf(warp_sum(qq.x * qq.x + qq.y * qq.y + qq.z * qq.z + qq.w * qq.w) + kNormEps);
  const float ik = rsqrtf(warp_sum(kk.x * kk.x + kk.y * kk.y + kk.z * kk.z + kk.w * kk.w) + kNormEps);
  st4(qa + o, make_float4(qq.x * iq, qq.y * iq, qq.z * iq, qq.w * iq));
  st4(ka + o, make_float4(kk.x * ik, kk.y * ik, kk.z * ik, kk.w * ik));
  if (lane == 0) {
    inv[2 * row] = iq;
    inv[2 * row + 1] = ik;
  }
  if (sd) {
    if (lane == 0) laa[row] = __float2bfloat16_rn(log_sigmoid_f(__bfloat162float(la[row])));
  } else {
    const float4 g = ld4(la + o);
    st4(laa + o, make_float4(log_sigmoid_f(g.x), log_sigmoid_f(g.y), log_sigmoid_f(g.z), log_sigmoid_f(g.w)));
  }
  if (sg) {
    if (lane == 0) {
      ba[row] = __float2bfloat16_rn(sigmoid_f(__bfloat162float(b[row])));
      if (w) wa[row] = __float2bfloat16_rn(sigmoid_f(__bfloat162float(w[row])));
    }
  } else {
    const float4 bb = ld4(b + o);
    st4(ba + o, make_float4(sigmoid_f(bb.x), sigmoid_f(bb.y), sigmoid_f(bb.z), sigmoid_f(bb.w)));
    if (w) {
      const float4 ww = ld4(w + o);
      st4(wa + o, make_float4(sigmoid_f(ww.x), sigmoid_f(ww.y), sigmoid_f(ww.z), sigmoid_f(ww.w)));
    }
  }
}

// The activations' chain rule, in place on the gradients with respect to the activated inputs:
// dq = (dq^ - q^ (q^ . dq^)) / |q| (k alike), d log_a *= 1 - sigmoid(log_a), db *= s (1 - s) with
// s = sigmoid(b) (w alike; dw absent with tied gates).
template <typename Tout>
__global__ void prolog_chain_kernel(const __nv_bfloat16 *q, const __nv_bfloat16 *k, const __nv_bfloat16 *la,
                                    const __nv_bfloat16 *b, const __nv_bfloat16 *w, const float *inv, int64_t rows,
                                    bool sd, bool sg, Tout *dq, Tout *dk, Tout *dla, Tout *db, Tout *dw) {
  const int64_t row = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const size_t o = (size_t)row * 128 + 4 * lane;
  const float iq = inv[2 * row], ik = inv[2 * row + 1];
  {
    const float4 qq = ld4(q + o), g = ld4t<Tout>(dq + o);
    const float4 qh = make_float4(qq.x * iq, qq.y * iq, qq.z * iq, qq.w * iq);
    const float s = warp_sum(qh.x * g.x + qh.y * g.y + qh.z * g.z + qh.w * g.w);
    st4t<Tout>(dq + o, make_float4((g.x - qh.x * s) * iq, (g.y - qh.y * s) * iq, (g.z - qh.z * s) * iq,
                                   (g.w - qh.w * s) * iq));
  }
  {
    const float4 kk = ld4(k + o), g = ld4t<Tout>(dk + o);
    const float4 kh = make_float4(kk.x * ik, kk.y * ik, kk.z * ik, kk.w * ik);
    const float s = warp_sum(kh.x * g.x + kh.y * g.y + kh.z * g.z + kh.w * g.w);
    st4t<Tout>(dk + o, make_float4((g.x - kh.x * s) * ik, (g.y - kh.y * s) * ik, (g.z - kh.z * s) * ik,
                                   (g.w - kh.w * s) * ik));
  }
  auto dsig = [](float x) {
    const float s = sigmoid_f(x);
    return s * (1.f - s);
  };
  if (sd) {
    if (lane == 0) dla[row] = from_f32<Tout>(to_f32<Tout>(dla[row]) * (1.f - sigmoid_f(__bfloat162float(la[row]))));
  } else {
    const float4 g = ld4(la + o), gd = ld4t<Tout>(dla + o);
    st4t<Tout>(dla + o, make_float4(gd.x * (1.f - sigmoid_f(g.x)), gd.y * (1.f - sigmoid_f(g.y)),
                                    gd.z * (1.f - sigmoid_f(g.z)), gd.w * (1.f - sigmoid_f(g.w))));
  }
  if (sg) {
    if (lane == 0) {
      db[row] = from_f32<Tout>(to_f32<Tout>(db[row]) * dsig(__bfloat162float(b[row])));
      if (dw) dw[row] = from_f32<Tout>(to_f32<Tout>(dw[row]) * dsig(__bfloat162float(w[row])));
    }
  } else {
    const float4 bb = ld4(b + o), gb = ld4t<Tout>(db + o);
    st4t<Tout>(db + o, make_float4(gb.x * dsig(bb.x), gb.y * dsig(bb.y), gb.z * dsig(bb.z), gb.w * dsig(bb.w)));
    if (dw) {
      const float4 ww = ld4(w + o), gw = ld4t<Tout>(dw + o);
      st4t<Tout>(dw + o, make_float4(gw.x * dsig(ww.x), gw.y * dsig(ww.y), gw.z * dsig(ww.z), gw.w * dsig(ww.w)));
    }
  }
}

}  // namespace

cudaError_t launch_prolog_act(const BwdProblem &p, const PrologueCopiesBf16 &c, cudaStream_t stream) {
  const int64_t rows = p.t_total * p.n_heads;
  if (rows == 0) return cudaSuccess;
  const bool sd = (p.flags & GDN2_SCALAR_DECAY) != 0, sg = (p.flags & GDN2_SCALAR_GATES) != 0;
  const bool tied = (p.flags & GDN2_TIED_GATES) != 0;
  prolog_act_kernel<<<(unsigned)((rows + 7) / 8), 256, 0, stream>>>(
      static_cast<const __nv_bfloat16 *>(p.q), static_cast<const __nv_bfloat16 *>(p.k),
      static_cast<const __nv_bfloat16 *>(p.log_a), static_cast<const __nv_bfloat16 *>(p.b),
      tied ? nullptr : static_cast<const __nv_bfloat16 *>(p.w), rows, sd, sg, c.q, c.k, c.log_a, c.b,
      tied ? nullptr : c.w, c.inv_norm);
  return cudaGetLastError();
}

cudaError_t launch_prolog_chain(const BwdProblem &p, const float *inv_norm, cudaStream_t stream) {
  const int64_t rows = p.t_total * p.n_heads;
  if (rows == 0) return cudaSuccess;
  const bool sd = (p.flags & GDN2_SCALAR_DECAY) != 0, sg = (p.flags & GDN2_SCALAR_GATES) != 0;
  const bool tied = (p.flags & GDN2_TIED_GATES) != 0;
  const auto *q = static_cast<const __nv_bfloat16 *>(p.q), *k = static_cast<const __nv_bfloat16 *>(p.k);
  const auto *la = static_cast<const __nv_bfloat16 *>(p.log_a), *b = static_cast<const __nv_bfloat16 *>(p.b);
  const auto *w = tied ? nullptr : static_cast<const __nv_bfloat16 *>(p.w);
  const unsigned grid = (unsigned)((rows + 7) / 8);
  if (p.dtype_out == GDN2_BF16) {
    using T = __nv_bfloat16;
    prolog_chain_kernel<T><<<grid, 256, 0, stream>>>(q, k, la, b, w, inv_norm, rows, sd, sg, static_cast<T *>(p.dq),
                                                     static_cast<T *>(p.dk), static_cast<T *>(p.dlog_a),
                                                     static_cast<T *>(p.db), tied ? nullptr : static_cast<T *>(p.dw));
  } else {
    prolog_chain_kernel<float><<<grid, 256, 0, stream>>>(q, k, la, b, w, inv_norm, rows, sd, sg,
                                                         static_cast<float *>(p.dq), static_cast<float *>(p.dk),
                                                         static_cast<float *>(p.dlog_a), static_cast<float *>(p.db),
                                                         tied ? nullptr : static_cast<float *>(p.dw));
  }
  return cudaGetLastError();
}

}  // namespace gdn2
