// chunk_tc.cu -- chunked Gated DeltaNet-2 forward on the sm_100a tensor cores
// (d_k = d_v = 128, chunk C = 64, bf16 inputs, fp32 state).
//
// The chunkwise WY form (alanhou.org "Core Mechanism": decay absorbed into
// asymmetric erase factors; gist.science Methodologie 3: a lower-triangular
// (I + T)^-1 solve yields erase-side and write-side auxiliaries) for one chunk
// of rows i, j in [0, 64) starting from state S (d_k x d_v):
//
//   x = b.k (erase outer), y = k (erase read), p = w.k (write outer), z = v,
//   L_i = sum_{j<=i} log_a_j (per channel), L_C = L_63,
//   L_ref = (L_0 + L_63) / 2 per channel, the midpoint of the chunk's decay range.
//   Scaled operands (every factor's exponent is at most half the chunk's decay range):
//     k_r = k e^{L - L_ref},  q_r = q e^{L - L_ref},
//     x_r = x e^{L_ref - L},  p_r = p e^{L_ref - L},  S_r = Diag(e^{L_ref}) S.
//   A chunk in which some channel decays by more than kFastSpan (128 nats) between its
//   first and last row would need factors beyond e^{64}; such a chunk runs the
//   recurrence token by token instead (CUDA cores, the state kept in registers), which
//   is exact for any finite log_a <= 0.
//   G1  [A B ; QX QP] = [k_r ; q_r] [x_r ; p_r]^T         (M=128 N=128 K=128)
//       A, B strictly lower; QX, QP lower incl. diagonal.
//   solve T = (I + A)^-1: 8x8 diagonal blocks by forward substitution, then the
//       off-diagonal blocks level by level, T_LU = -T_LL (A_LU T_UU).
//   R^T = V^T B^T + S_r^T k_r^T    (the right-hand side of M = T R)
//   M^T = R^T T^T                   row i of M is the erase read r_i = Sbar_i^T k_i
//   O^T = S_r^T q_r^T + V^T QP^T - M^T QX^T
//   S'  = Diag(e^{L_C - L_ref}) (S_r' + p_r^T V - x_r^T M),  S_r' = Diag(e^{L_ref}) S in fp32.
// All GEMMs are tcgen05.mma kind::f16 with fp32 accumulators in TMEM, computed in
// their transposed forms (M = d_v = 128 rows): O^T, R^T, M^T and S^T.  The state lives
// in TMEM in fp32 for the whole sequence, transposed, as S = Diag(tau) Sacc: each chunk
// rewrites Sacc as e^{L_ref} S, the increment GEMMs accumulate onto it, and tau becomes
// e^{L_C - L_ref}.  The A operands S_r^T, R^T and -M^T are written by the threads into
// TMEM as bf16 and read from there by the tensor core; the B operands and V^T come
// from shared memory, where the tiles arrive by TMA (128-byte swizzle) and transposed
// operands use MN-major descriptors, so no tile is ever transposed in memory.  The
// T-independent GEMMs run on the tensor core while warps 0-14 solve for T, and the next
// chunk's operands (cumulative decay, k_r, q_r, p_r, x_r) are built while this chunk's
// remaining GEMMs (M = T R, the last terms of O and of the state) run; a chunk's G1 is
// issued before its S_r build.  A tcgen05.mma holds its issuing thread for roughly
// its execution time, so products are merged into as few N = 128 instructions as the
// operand layouts allow.
//
// One CTA (512 threads) per SM, persistent over (sequence, head) units taken
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
#include "tc_util.cuh"

namespace gdn2 {
namespace {

constexpr int C = 64;
constexpr int D = 128;
constexpr int kThreads = 512;
constexpr uint32_t kTmemCols = 512;
constexpr uint64_t kWaitTimeoutNs = 1000000000ull;  // 1 s
constexpr float kLog2eF = 1.4426950408889634f;
// Largest in-chunk decay range L_0 - L_63 (nats, per channel) of the factored form: its
// operand factors then stay within e^{+-64}, far from the fp32/bf16 limit (e^{88.7}), and
// a state term that underflows in S_r = e^{L_ref} S can only have been worth e^{64 - 87.3}
// of the state's size in any output.
constexpr float kFastSpan = 128.f;
// One backward checkpoint slot per chunk: the bf16 S_r tile image (32 KB), then the bf16 T tile
// image (8 KB), both in the swizzled layout of this kernel's shared-memory tiles.
constexpr size_t kCkptT = (size_t)D * D * 2;
constexpr size_t kCkptBytes = kBwdCkptSlotBytes;
static_assert(kCkptBytes == kCkptT + (size_t)C * C * 2, "checkpoint slot layout");

// Shared-memory map, byte offsets from a 1024-byte-aligned base.  Every operand
// tile is a stack of 8-row x 128-byte swizzle atoms.
constexpr uint32_t OFF_KQ = 0;         // 2 K-blocks x [k_r rows 0-63 | q_r rows 0-63], 16 KB each
constexpr uint32_t OFF_XP = 32768;     // 2 K-blocks x [x_r rows | p_r rows]
constexpr uint32_t OFF_V = 65536;      // 2 column blocks x [64 rows], 8 KB each
constexpr uint32_t OFF_G = 81920;      // raw log_a tile; after the cumulative decay, the raw b tile
constexpr uint32_t OFF_OS = 98304;     // o staging: 2 (bf16) or 4 (fp32) sub-blocks of [64 tokens][128 B]
constexpr uint32_t OFF_T = 131072;     // T bf16 [64 x 64]
constexpr uint32_t OFF_BM = 139264;    // B bf16 [64 x 64]; with QP right after it, the 128-row B operand [B; QP]
constexpr uint32_t OFF_QP = 147456;    // QP bf16 [64 x 64] (QX when x_r == p_r)
constexpr uint32_t OFF_QX = 155648;    // QX bf16 [64 x 64]
constexpr uint32_t OFF_AF = 163840;    // fp32 A [64 x 68] (masks -> solve)
constexpr uint32_t OFF_TF = 181248;    // fp32 T [64 x 68] (solve)
constexpr uint32_t OFF_XS = 198656;    // fp32 solve scratch, <= 4 KB
constexpr uint32_t OFF_MISC = 212992;
constexpr uint32_t MISC_DL0 = 0;       // float[128]  e^{L_C - L_ref} of the chunks with even parity
constexpr uint32_t MISC_DL = 512;      // float[128]  e^{L_C - L_ref} of the chunks with odd parity
constexpr uint32_t MISC_SM = 1024;     // float[128]  e^{L_ref}
constexpr uint32_t MISC_PART = 1536;   // float[16][128] 4-row sums of log_a, then exclusive prefixes
constexpr uint32_t MISC_REF = 9728;    // float[128]  L_ref
constexpr uint32_t MISC_BAR = 10240;   // 12 mbarriers
constexpr uint32_t MISC_TMEM = 10336;
constexpr uint32_t MISC_ABORT = 10340;
constexpr uint32_t MISC_UNIT = 10344;
constexpr uint32_t MISC_WIDE = 10348;  // int: some channel of the chunk being prepared has a wide decay range
constexpr uint32_t MISC_ISS = 10352;   // uint32[4]   phases armed per TMA barrier (A, L, W, X)
constexpr uint32_t MISC_L0 = 10368;    // float[128]  L_0 (the chunk's first row)
constexpr uint32_t MISC_SCN = 10880;   // float[3][64] the next chunk's raw scalar log_a and gates
constexpr uint32_t MISC_BYTES = 11648;
// Token-serial chunks stage their per-token vectors in [OFF_OS, OFF_MISC) (fp32):
// a, q, y, x, p as [32 tokens][128], z as [32][128], q.x and q.p [32], and the
// cross-warp exchange of the column sums [2][4][128] float2.
constexpr uint32_t SER_A = 0, SER_Q = 4096, SER_Y = 8192, SER_X = 12288, SER_P = 16384, SER_Z = 20480;
constexpr uint32_t SER_QX = 24576, SER_QP = 24608, SER_XCH = 24640;  // float offsets from OFF_OS
static_assert(OFF_OS + 4 * SER_XCH + 2 * 4 * 128 * 8 <= OFF_MISC, "token-serial staging overflows");
constexpr uint32_t kSmemBytes = OFF_MISC + MISC_BYTES + 1024;  // + base alignment slack
// mbarrier slots
// (BAR_DRAIN0/1: used once, after a timed-out wait, to let the MMAs of the two issuing threads finish)
enum { BAR_TMA_A = 0, BAR_TMA_L, BAR_TMA_W, BAR_TMA_X, BAR_G1, BAR_E1, BAR_GA, BAR_GB, BAR_G4, BAR_G5,
       BAR_DRAIN0, BAR_DRAIN1, kNumBars };
static_assert(MISC_BAR + 8 * kNumBars <= MISC_TMEM, "mbarriers overlap the TMEM address slot");
static_assert(MISC_ISS + 16 <= MISC_L0, "issue counters overlap L_0");

struct TcParams {
  CUtensorMap tm_q, tm_k, tm_v, tm_g, tm_b, tm_w;
  CUtensorMap tm_o;  // o viewed as (channel, head, token), box 64 (bf16) or 32 (fp32) x 1 x 64, no swizzle
  ChunkProblem p;
  int32_t *counter;
  int n_units;
  uint64_t wait_ns;  // limit of every mbarrier wait (kWaitTimeoutNs unless the timeout test hook is armed)
  int dbg_skip;      // timeout test hook: CTA 0 arms its first k/q/v load group but issues none of its copies
};

using namespace tc;

// fp32 64x64 scratch, rows padded to 68 floats (272 B): conflict-free float4 row writes.
__device__ __forceinline__ int fidx(int i, int j) { return i * 68 + j; }

// A chunk whose decay range is beyond the factored form, token by token (CUDA cores, fp32):
// per token, Sbar = Diag(a) S; r = Sbar^T y; u = Sbar^T q; o = u - (q.x) r + (q.p) z;
// S = Sbar - x r^T + p z^T, with (y, x, p, z) = (k, b.k, w.k, v), or (b.k, k, k, w.v) in the
// gist.science form.  The 512 threads hold the state as the chunk kernel's TMEM layout gives it
// (thread: dv channel `row`, dk channels [32 cg, 32 cg + 32)); the four warps of a lane
// quadrant add their column sums through shared memory.  The per-token vectors of 32 tokens at
// a time are staged in fp32 in [OFF_OS, OFF_MISC).  tmem_s: this thread's 32 state columns;
// tau: the previous chunk's e^{L_C - L_ref} for them (NULL: 1); the state goes back to TMEM
// as it is (tau = 1).  Kept out of line so that its registers do not press on the factored path.
template <bool kScalarDecay, bool kScalarGates, bool kP3, bool kProlog, typename Tout>
__device__ __noinline__ void serial_chunk(const ChunkProblem &p, uint8_t *gb, uint32_t tmem_s, const float *tau,
                                          int t0, int nvalid, int h) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int qd = warp & 3, cg = warp >> 2, row = qd * 32 + lane;
  const int H = p.n_heads;
  const __nv_bfloat16 *g_la = static_cast<const __nv_bfloat16 *>(p.log_a);
  const __nv_bfloat16 *g_b = static_cast<const __nv_bfloat16 *>(p.b);
  const __nv_bfloat16 *g_w = static_cast<const __nv_bfloat16 *>((p.flags & GDN2_TIED_GATES) ? p.b : p.w);
  float *fs = reinterpret_cast<float *>(gb + OFF_OS);
  const __nv_bfloat16 *g_q = static_cast<const __nv_bfloat16 *>(p.q);
  const __nv_bfloat16 *g_k = static_cast<const __nv_bfloat16 *>(p.k);
  const __nv_bfloat16 *g_v = static_cast<const __nv_bfloat16 *>(p.v);
  for (int half = 0; half * 32 < nvalid; ++half) {
    const int nt = nvalid - half * 32 < 32 ? nvalid - half * 32 : 32;
    // stage the per-token vectors of tokens [32 half, 32 half + nt): one token row per warp
    // at a time, lane l holding channels 4 l .. 4 l + 3 (both d_k and d_v are 128)
    for (int tl = warp; tl < nt; tl += 16) {
      const size_t rt = (size_t)(t0 + half * 32 + tl) * H + h;
      float4 la, bb, ww;
      float4 kk = unpack4(*reinterpret_cast<const uint2 *>(g_k + rt * D + 4 * lane));
      float4 qq = unpack4(*reinterpret_cast<const uint2 *>(g_q + rt * D + 4 * lane));
      const float4 vv = unpack4(*reinterpret_cast<const uint2 *>(g_v + rt * D + 4 * lane));
      if (kScalarDecay) {
        const float x = __bfloat162float(g_la[rt]);
        la = make_float4(x, x, x, x);
      } else {
        la = unpack4(*reinterpret_cast<const uint2 *>(g_la + rt * D + 4 * lane));
      }
      if (kScalarGates) {
        const float xb = __bfloat162float(g_b[rt]), xw = __bfloat162float(g_w[rt]);
        bb = make_float4(xb, xb, xb, xb);
        ww = make_float4(xw, xw, xw, xw);
      } else {
        bb = unpack4(*reinterpret_cast<const uint2 *>(g_b + rt * D + 4 * lane));
        ww = unpack4(*reinterpret_cast<const uint2 *>(g_w + rt * D + 4 * lane));
      }
      if (kProlog) {
        la = make_float4(log_sigmoid_f(la.x), log_sigmoid_f(la.y), log_sigmoid_f(la.z), log_sigmoid_f(la.w));
        bb = make_float4(sigmoid_f(bb.x), sigmoid_f(bb.y), sigmoid_f(bb.z), sigmoid_f(bb.w));
        ww = make_float4(sigmoid_f(ww.x), sigmoid_f(ww.y), sigmoid_f(ww.z), sigmoid_f(ww.w));
        float k2 = kk.x * kk.x + kk.y * kk.y + kk.z * kk.z + kk.w * kk.w;
        float q2 = qq.x * qq.x + qq.y * qq.y + qq.z * qq.z + qq.w * qq.w;
#pragma unroll
        for (int sh = 16; sh >= 1; sh >>= 1) {
          k2 += __shfl_xor_sync(0xffffffffu, k2, sh);
          q2 += __shfl_xor_sync(0xffffffffu, q2, sh);
        }
        const float ik = rsqrtf(k2 + kNormEps), iq = rsqrtf(q2 + kNormEps);
        kk = make_float4(kk.x * ik, kk.y * ik, kk.z * ik, kk.w * ik);
        qq = make_float4(qq.x * iq, qq.y * iq, qq.z * iq, qq.w * iq);
      }
      const float4 bk = make_float4(bb.x * kk.x, bb.y * kk.y, bb.z * kk.z, bb.w * kk.w);
      // erase read y, erase outer x, write outer p and written value z (per d_v channel):
      // (k, b.k, w.k, v) by default, (b.k, k, k, w.v) in the gist.science form
      const float4 yy = kP3 ? bk : kk;
      const float4 xx = kP3 ? kk : bk;
      const float4 pp = kP3 ? kk : make_float4(ww.x * kk.x, ww.y * kk.y, ww.z * kk.z, ww.w * kk.w);
      const float4 zz = kP3 ? make_float4(ww.x * vv.x, ww.y * vv.y, ww.z * vv.z, ww.w * vv.w) : vv;
      const float4 aa = make_float4(ptx::ex2(la.x * kLog2eF), ptx::ex2(la.y * kLog2eF), ptx::ex2(la.z * kLog2eF),
                                    ptx::ex2(la.w * kLog2eF));
      float qx = qq.x * xx.x + qq.y * xx.y + qq.z * xx.z + qq.w * xx.w;
      float qp = qq.x * pp.x + qq.y * pp.y + qq.z * pp.z + qq.w * pp.w;
#pragma unroll
      for (int sh = 16; sh >= 1; sh >>= 1) {
        qx += __shfl_xor_sync(0xffffffffu, qx, sh);
        qp += __shfl_xor_sync(0xffffffffu, qp, sh);
      }
      const int e = tl * 128 + 4 * lane;
      *reinterpret_cast<float4 *>(fs + SER_A + e) = aa;
      *reinterpret_cast<float4 *>(fs + SER_Q + e) = qq;
      *reinterpret_cast<float4 *>(fs + SER_Y + e) = yy;
      *reinterpret_cast<float4 *>(fs + SER_X + e) = xx;
      *reinterpret_cast<float4 *>(fs + SER_P + e) = pp;
      *reinterpret_cast<float4 *>(fs + SER_Z + e) = zz;
      if (lane == 0) {
        fs[SER_QX + tl] = qx;
        fs[SER_QP + tl] = qp;
      }
    }
    __syncthreads();
    // the state into registers (dv channel `row`, dk channels [32 cg, 32 cg + 32)): the first
    // half takes S = Diag(tau) Sacc, the second the first half's result
    float sv[32];
    {
      uint32_t r[32];
      ptx::tmem_ld32(tmem_s, r);
      ptx::tmem_wait_ld();
      const bool scale = half == 0 && tau != nullptr;
#pragma unroll
      for (int j = 0; j < 32; ++j) sv[j] = __uint_as_float(r[j]) * (scale ? tau[j] : 1.f);
    }
    // per token: Sbar = Diag(a) S; r = Sbar^T y and u = Sbar^T q (column sums over d_k, the
    // four warps of a lane quadrant holding a quarter each); o = u - (q.x) r + (q.p) z;
    // S = Sbar - x r^T + p z^T
    float2 *xch = reinterpret_cast<float2 *>(fs + SER_XCH);
    for (int tl = 0; tl < nt; ++tl) {
      const float *A = fs + SER_A + tl * 128 + cg * 32;
      const float *Y = fs + SER_Y + tl * 128 + cg * 32;
      const float *Qv = fs + SER_Q + tl * 128 + cg * 32;
      float rp = 0.f, up = 0.f;
#pragma unroll
      for (int j4 = 0; j4 < 8; ++j4) {
        const float4 a4 = *reinterpret_cast<const float4 *>(A + 4 * j4);
        const float4 y4 = *reinterpret_cast<const float4 *>(Y + 4 * j4);
        const float4 q4 = *reinterpret_cast<const float4 *>(Qv + 4 * j4);
        sv[4 * j4] *= a4.x;
        sv[4 * j4 + 1] *= a4.y;
        sv[4 * j4 + 2] *= a4.z;
        sv[4 * j4 + 3] *= a4.w;
        rp = fmaf(sv[4 * j4], y4.x, rp);
        rp = fmaf(sv[4 * j4 + 1], y4.y, rp);
        rp = fmaf(sv[4 * j4 + 2], y4.z, rp);
        rp = fmaf(sv[4 * j4 + 3], y4.w, rp);
        up = fmaf(sv[4 * j4], q4.x, up);
        up = fmaf(sv[4 * j4 + 1], q4.y, up);
        up = fmaf(sv[4 * j4 + 2], q4.z, up);
        up = fmaf(sv[4 * j4 + 3], q4.w, up);
        asm volatile("" ::: "memory");  // keep the loads of one step at a time in registers
      }
      xch[((tl & 1) * 4 + cg) * 128 + row] = make_float2(rp, up);
      named_bar(2 + qd, 128);  // the four warps of this lane quadrant
      float r = 0.f, u = 0.f;
#pragma unroll
      for (int g = 0; g < 4; ++g) {  // the same order in all four warps: identical r and u
        const float2 pr = xch[((tl & 1) * 4 + g) * 128 + row];
        r += pr.x;
        u += pr.y;
      }
      const float zr = fs[SER_Z + tl * 128 + row];
      if (cg == 0 && p.o) {
        const float ov = u - fs[SER_QX + tl] * r + fs[SER_QP + tl] * zr;
        Tout *go = static_cast<Tout *>(p.o) + ((size_t)(t0 + half * 32 + tl) * H + h) * D + row;
        *go = from_f32<Tout>(ov);
      }
      const float *X = fs + SER_X + tl * 128 + cg * 32;
      const float *P = fs + SER_P + tl * 128 + cg * 32;
#pragma unroll
      for (int j4 = 0; j4 < 8; ++j4) {
        const float4 x4 = *reinterpret_cast<const float4 *>(X + 4 * j4);
        const float4 p4 = *reinterpret_cast<const float4 *>(P + 4 * j4);
        sv[4 * j4] = fmaf(p4.x, zr, fmaf(-x4.x, r, sv[4 * j4]));
        sv[4 * j4 + 1] = fmaf(p4.y, zr, fmaf(-x4.y, r, sv[4 * j4 + 1]));
        sv[4 * j4 + 2] = fmaf(p4.z, zr, fmaf(-x4.z, r, sv[4 * j4 + 2]));
        sv[4 * j4 + 3] = fmaf(p4.w, zr, fmaf(-x4.w, r, sv[4 * j4 + 3]));
        asm volatile("" ::: "memory");
      }
    }
    {  // the state back into TMEM (as Sacc with tau = 1)
      uint32_t r[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) r[j] = __float_as_uint(sv[j]);
      ptx::tmem_st32(tmem_s, r);
      ptx::tmem_wait_st();
    }
    __syncthreads();  // the staging of the next half overwrites what the token loop read
  }
}

// kP3: the gist.science gate placement.  The operands are then k_r = (b.k) e^{L - L_ref}
// (erase read), x_r = p_r = k e^{L_ref - L} (erase and write outer factors) and the
// values w.v; the host swaps the gate tensor maps so that the gate needed first (b)
// arrives with the TMA_W group and w with the TMA_X group.
// kProlog: the inputs are pre-activations (GDN2_FUSED_PROLOGUE): log_a <- log sigmoid,
// b, w <- sigmoid, and the q and k rows are L2-normalised here.
// kXP: x_r == p_r (the gist.science form always; the default form with tied gates),
// so B = A and QP = QX: G1 runs with N = 64 and the masks write B and read QP from the
// A and QX values.
// kCk: the checkpointing forward of gdn2_chunk_bwd (p.ckpt set, no o): each chunk's bf16 S_r
// and T tile images go to the chunk's checkpoint slot.  A separate instantiation keeps that
// work out of the plain forward's code.
template <bool kScalarDecay, bool kScalarGates, bool kP3, bool kProlog, bool kXP, typename Tout, bool kCk>
__global__ void __launch_bounds__(kThreads, 1) chunk_tc_kernel(const __grid_constant__ TcParams P) {
  extern __shared__ uint8_t smem_raw[];
  const ChunkProblem &p = P.p;
  const uint32_t raw = ptx::smem_u32(smem_raw);
  const uint32_t sb = (raw + 1023u) & ~1023u;
  uint8_t *gb = smem_raw + (sb - raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int qd = warp & 3, cg = warp >> 2;   // TMEM lane quadrant, column group
  const int row = qd * 32 + lane;            // the TMEM lane this thread reads
  const int H = p.n_heads;
  const bool tied = (p.flags & GDN2_TIED_GATES) != 0;

  // e^{L_C - L_ref} per d_k channel, one buffer per chunk parity: the S_r build of a chunk
  // reads the previous chunk's factors while the elementwise pass writes this chunk's
  static_assert(MISC_DL == MISC_DL0 + 512, "the two e^{L_C - L_ref} buffers are adjacent");
  auto sDLb = [&](uint32_t parity) { return reinterpret_cast<float *>(gb + OFF_MISC + MISC_DL0 + 512u * parity); };
  float *sSM = reinterpret_cast<float *>(gb + OFF_MISC + MISC_SM);
  // scalar flags: the raw per-token log_a [0, 64), the gate of pass 2 [64, 128) and the gate of
  // pass 3 [128, 192) of the chunk being prepared, fetched from global memory a chunk early
  float *sScN = reinterpret_cast<float *>(gb + OFF_MISC + MISC_SCN);
  float *part = reinterpret_cast<float *>(gb + OFF_MISC + MISC_PART);
  float *sRef = reinterpret_cast<float *>(gb + OFF_MISC + MISC_REF);
  float *sL0 = reinterpret_cast<float *>(gb + OFF_MISC + MISC_L0);
  volatile int *sWide = reinterpret_cast<volatile int *>(gb + OFF_MISC + MISC_WIDE);
  constexpr int kIssuer = 32;      // issues a unit's first TMA loads, the log_a and b loads and the o stores
  constexpr int kIssueWarp = 15;   // issues the T-independent MMAs during the solve
  constexpr int kSolveThreads = 480;  // warps 0-14
  enum { NB_SOLVE = 1 };
  volatile int *sAbort = reinterpret_cast<volatile int *>(gb + OFF_MISC + MISC_ABORT);
  volatile int *sUnit = reinterpret_cast<volatile int *>(gb + OFF_MISC + MISC_UNIT);
  auto bar = [&](int i) { return sb + OFF_MISC + MISC_BAR + 8u * (uint32_t)i; };
  auto waitb = [&](uint32_t b, uint32_t parity) { return wait_bar(b, parity, sAbort, p.status, P.wait_ns); };
  volatile uint32_t *sIss = reinterpret_cast<volatile uint32_t *>(gb + OFF_MISC + MISC_ISS);

  // the bf16 T tile's blocks above the diagonal are never written by the solve: zero once
  sts_v4(sb + OFF_T + 16u * (uint32_t)tid, make_uint4(0u, 0u, 0u, 0u));
  static_assert(kThreads * 16 == 8192, "one 16-byte store per thread zeroes the 8 KB T tile");
  if (tid == 0) {
    for (int i = 0; i < kNumBars; ++i) ptx::mbar_init(bar(i), 1);
    ptx::fence_mbar_init();
    *sAbort = 0;
    for (int i = 0; i < 4; ++i) sIss[i] = 0u;
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
  // The state is held transposed, S^T (lane = d_v channel, column = d_k channel), so that
  // S_r^T, R^T and -M^T -- the A operands of every state-side GEMM -- are read by the tensor
  // core straight from TMEM as bf16 (two channels per column) and never visit shared memory.
  const uint32_t tmD1 = tmem;        // G1 result; then [R^T | O^T] (cols 0-63 | 64-127), fp32
  const uint32_t tmS = tmem + 128;   // S^T fp32 (128 cols)
  const uint32_t tmO = tmem + 64;    // O^T fp32 (64 cols), beside R^T: both come from one N = 128 product
  const uint32_t tmM = tmem + 256;   // M^T fp32 (64 cols)
  const uint32_t tmSR = tmem + 320;  // S_r^T bf16 A operand (64 cols)
  const uint32_t tmRb = tmem + 384;  // R^T bf16 A operand (32 cols)
  const uint32_t tmMb = tmem + 416;  // -M^T bf16 A operand (32 cols)
  const uint32_t lane_base = (uint32_t)(qd * 32) << 16;
  uint32_t it = 0;                   // chunks processed by this CTA: parity of every mbarrier

  const __nv_bfloat16 *g_la = static_cast<const __nv_bfloat16 *>(p.log_a);
  const __nv_bfloat16 *g_b = static_cast<const __nv_bfloat16 *>(p.b);
  const __nv_bfloat16 *g_w = static_cast<const __nv_bfloat16 *>(tied ? p.b : p.w);

  // TMA issue (thread 0): group A = k, q, v (+ log_a), group B = b, w.
  // TMA issue: group A = k, q, v; group L = log_a (into the log_a slot, free from the start of
  // the previous chunk, so it is requested a whole chunk ahead); group W = w; group X = b.
  bool dbg_armed = P.dbg_skip != 0 && blockIdx.x == 0;  // the timeout test hook (thread kIssuer)
  auto issue_tma_a = [&](int h, int t0) {
    ptx::mbar_arrive_expect_tx(bar(BAR_TMA_A), 3u * 2u * 8192u);
    sIss[BAR_TMA_A] = sIss[BAR_TMA_A] + 1u;
    if (dbg_armed) {  // bytes announced, no copy issued: the wait for this group runs out
      dbg_armed = false;
      return;
    }
#pragma unroll
    for (int kb = 0; kb < 2; ++kb) {
      ptx::tma_load_3d(sb + OFF_KQ + kb * 16384, &P.tm_k, kb * 64, h, t0, bar(BAR_TMA_A));
      ptx::tma_load_3d(sb + OFF_KQ + kb * 16384 + 8192, &P.tm_q, kb * 64, h, t0, bar(BAR_TMA_A));
      ptx::tma_load_3d(sb + OFF_V + kb * 8192, &P.tm_v, kb * 64, h, t0, bar(BAR_TMA_A));
    }
  };
  auto issue_tma_l = [&](int h, int t0) {
    if (kScalarDecay) return;
    ptx::mbar_arrive_expect_tx(bar(BAR_TMA_L), 2u * 8192u);
    sIss[BAR_TMA_L] = sIss[BAR_TMA_L] + 1u;
#pragma unroll
    for (int kb = 0; kb < 2; ++kb) ptx::tma_load_3d(sb + OFF_G + kb * 8192, &P.tm_g, kb * 64, h, t0, bar(BAR_TMA_L));
  };
  // w lands in the p_r halves of XP (free once dS = p_r^T V is done), b in the log_a slot
  // (free once the cumulative decay of its chunk is done)
  auto issue_tma_w = [&](int h, int t0) {
    if (kScalarGates) return;
    ptx::mbar_arrive_expect_tx(bar(BAR_TMA_W), 2u * 8192u);
    sIss[BAR_TMA_W] = sIss[BAR_TMA_W] + 1u;
#pragma unroll
    for (int kb = 0; kb < 2; ++kb)
      ptx::tma_load_3d(sb + OFF_XP + kb * 16384 + 8192, &P.tm_w, kb * 64, h, t0, bar(BAR_TMA_W));
  };
  auto issue_tma_x = [&](int h, int t0) {
    if (kScalarGates) return;
    ptx::mbar_arrive_expect_tx(bar(BAR_TMA_X), 2u * 8192u);
    sIss[BAR_TMA_X] = sIss[BAR_TMA_X] + 1u;
#pragma unroll
    for (int kb = 0; kb < 2; ++kb)
      ptx::tma_load_3d(sb + OFF_G + kb * 8192, &P.tm_b, kb * 64, h, t0, bar(BAR_TMA_X));
  };

  // ---- a2/a3: cumulative log-decay and scaled operands of one chunk (rows t0n .. t0n + 63 of
  //      head h, the first nvn of them valid), in place, in three passes that the chunk loop
  //      runs between the previous chunk's GEMMs.  Thread: channels 4 lane .. 4 lane + 3,
  //      rows 4 warp .. 4 warp + 3.
  const int e_kb = lane >> 4;
  const uint32_t e_ch16 = (uint32_t)((lane & 15) >> 1), e_cofs = (uint32_t)(lane & 1) * 8u;
  // pass 1 (needs the log_a tile): inclusive cumsum L of this thread's rows, then per channel
  // the exclusive prefixes over the 16 row groups, L_ref = (L_0 + L_63) / 2, e^{L_C - L_ref}
  // into the parity-pn buffer and e^{L_ref}.  Ends with a CTA barrier, after which the log_a
  // slot is free; returns non-zero (in every thread) when some channel's decay range
  // L_0 - L_63 exceeds kFastSpan, i.e. the chunk must run token by token.
  // scalar flags: thread tid < 192 fetches value (tid & 63) of array (tid >> 6) for the chunk
  // starting at t0n (0 past its end); the caller stores it to sScN[tid] once it has landed
  auto scal_load = [&](int t0n, int nvn, int h) -> float {
    const int which = tid >> 6, r = tid & 63;
    if (tid >= 192 || r >= nvn) return 0.f;
    const __nv_bfloat16 *src = which == 0 ? (kScalarDecay ? g_la : nullptr)
                               : which == 1 ? (kScalarGates ? (kP3 ? g_b : g_w) : nullptr)
                                            : (kScalarGates ? (kP3 ? g_w : g_b) : nullptr);
    return src ? __bfloat162float(src[(size_t)(t0n + r) * H + h]) : 0.f;
  };
  auto elem_cumsum = [&](uint32_t pn, int t0n, int nvn, int h, float4 (&L)[4]) -> int {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int rr = 0; rr < 4; ++rr) {
      const int r = warp * 4 + rr;
      float4 g = make_float4(0.f, 0.f, 0.f, 0.f);
      if (r < nvn) {
        if (kScalarDecay) {
          float sv = sScN[r];
          if (kProlog) sv = log_sigmoid_f(sv);
          g = make_float4(sv, sv, sv, sv);
        } else {
          g = unpack4(lds_v2(sb + OFF_G + e_kb * 8192 + swz(r, e_ch16) + e_cofs));
          if (kProlog) g = make_float4(log_sigmoid_f(g.x), log_sigmoid_f(g.y), log_sigmoid_f(g.z), log_sigmoid_f(g.w));
        }
      }
      acc.x += g.x; acc.y += g.y; acc.z += g.z; acc.w += g.w;
      L[rr] = acc;
    }
    *reinterpret_cast<float4 *>(part + warp * 128 + 4 * lane) = acc;
    if (warp == 0) *reinterpret_cast<float4 *>(sL0 + 4 * lane) = L[0];  // L_0 = log_a of row 0
    if (tid == 0) *sWide = 0;
    __syncthreads();
    if (tid < D) {  // per channel: exclusive prefix over the 16 row groups, L_C = L_63, the reference
      float run = 0.f;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const float pj = part[j * 128 + tid];
        part[j * 128 + tid] = run;
        run += pj;
      }
      const float l0 = sL0[tid];
      const float refv = 0.5f * (l0 + run);
      if (!(l0 - run <= kFastSpan)) *sWide = 1;  // any writer sets it; nobody clears it before the barrier
      sRef[tid] = refv;
      sDLb(pn)[tid] = ptx::ex2((run - refv) * kLog2eF);
      sSM[tid] = ptx::ex2(refv * kLog2eF);
    }
    __syncthreads();
    return *sWide;
  };
  // pass 2 (needs the k, q, v tiles and the w tile): k_r, q_r and p_r in place; rows past the
  // chunk end are zeroed (v too).  ke2 keeps k e^{L_ref - L} for pass 3.
  auto elem_scale = [&](int t0n, int nvn, int h, const float4 (&L)[4], float4 (&ke2)[4]) {
    const float4 off = *reinterpret_cast<const float4 *>(part + warp * 128 + 4 * lane);
    const float4 ref = *reinterpret_cast<const float4 *>(sRef + 4 * lane);
    const float4 base = make_float4((off.x - ref.x) * kLog2eF, (off.y - ref.y) * kLog2eF,
                                    (off.z - ref.z) * kLog2eF, (off.w - ref.w) * kLog2eF);
#pragma unroll
    for (int rr = 0; rr < 4; ++rr) {
      const int r = warp * 4 + rr;
      const uint32_t o = (uint32_t)e_kb * 16384u + swz(r, e_ch16) + e_cofs;
      const float l0 = fmaf(L[rr].x, kLog2eF, base.x), l1 = fmaf(L[rr].y, kLog2eF, base.y);
      const float l2 = fmaf(L[rr].z, kLog2eF, base.z), l3 = fmaf(L[rr].w, kLog2eF, base.w);
      const float e10 = ptx::ex2(l0), e11 = ptx::ex2(l1), e12 = ptx::ex2(l2), e13 = ptx::ex2(l3);
      const float4 e2 = make_float4(ptx::ex2(-l0), ptx::ex2(-l1), ptx::ex2(-l2), ptx::ex2(-l3));
      float4 kk = unpack4(lds_v2(sb + OFF_KQ + o));
      float4 qq = kCk ? make_float4(0.f, 0.f, 0.f, 0.f) : unpack4(lds_v2(sb + OFF_KQ + o + 8192));
      float4 ww;  // the write gate w (the erase gate b in the gist.science form)
      if (kScalarGates) {
        ww = make_float4(0.f, 0.f, 0.f, 0.f);
        if (r < nvn) {
          float swv = sScN[64 + r];
          if (kProlog) swv = sigmoid_f(swv);
          ww = make_float4(swv, swv, swv, swv);
        }
      } else {
        ww = unpack4(lds_v2(sb + OFF_XP + o + 8192));
        if (kProlog) ww = make_float4(sigmoid_f(ww.x), sigmoid_f(ww.y), sigmoid_f(ww.z), sigmoid_f(ww.w));
      }
      if (r >= nvn) {
        kk = make_float4(0.f, 0.f, 0.f, 0.f);
        qq = kk;
        ww = kk;
        sts_v2(sb + OFF_V + e_kb * 8192 + swz(r, e_ch16) + e_cofs, make_uint2(0u, 0u));
      }
      if (kProlog) {  // the 32 lanes of this warp hold the row's 128 channels
        float k2 = kk.x * kk.x + kk.y * kk.y + kk.z * kk.z + kk.w * kk.w;
        float q2 = qq.x * qq.x + qq.y * qq.y + qq.z * qq.z + qq.w * qq.w;
#pragma unroll
        for (int sh = 16; sh >= 1; sh >>= 1) {
          k2 += __shfl_xor_sync(0xffffffffu, k2, sh);
          q2 += __shfl_xor_sync(0xffffffffu, q2, sh);
        }
        const float ik = rsqrtf(k2 + kNormEps), iq = rsqrtf(q2 + kNormEps);
        kk = make_float4(kk.x * ik, kk.y * ik, kk.z * ik, kk.w * ik);
        qq = make_float4(qq.x * iq, qq.y * iq, qq.z * iq, qq.w * iq);
      }
      ke2[rr] = make_float4(kk.x * e2.x, kk.y * e2.y, kk.z * e2.z, kk.w * e2.w);
      const float4 ke = ke2[rr];
      if (kP3) {
        sts_v2(sb + OFF_KQ + o, pack4(ww.x * kk.x * e10, ww.y * kk.y * e11, ww.z * kk.z * e12, ww.w * kk.w * e13));
        sts_v2(sb + OFF_XP + o + 8192, pack4(ke.x, ke.y, ke.z, ke.w));
      } else {
        sts_v2(sb + OFF_KQ + o, pack4(kk.x * e10, kk.y * e11, kk.z * e12, kk.w * e13));
        sts_v2(sb + OFF_XP + o + 8192, pack4(ww.x * ke.x, ww.y * ke.y, ww.z * ke.z, ww.w * ke.w));
      }
      if (!kCk) sts_v2(sb + OFF_KQ + o + 8192, pack4(qq.x * e10, qq.y * e11, qq.z * e12, qq.w * e13));
    }
  };
  // pass 3 (needs the b tile, which lands in the log_a slot, and a free x_r slot): x_r = b.k
  // e^{L_ref - L}; in the gist.science form x_r = k e^{L_ref - L} and the values are scaled by
  // the value gate.
  auto elem_x = [&](int t0n, int nvn, int h, const float4 (&ke2)[4]) {
#pragma unroll
    for (int rr = 0; rr < 4; ++rr) {
      const int r = warp * 4 + rr;
      const uint32_t o = (uint32_t)e_kb * 16384u + swz(r, e_ch16) + e_cofs;
      float4 bb;  // the erase gate b (the value gate w in the gist.science form)
      if (kScalarGates) {
        bb = make_float4(0.f, 0.f, 0.f, 0.f);
        if (r < nvn) {
          float sbv = sScN[128 + r];
          if (kProlog) sbv = sigmoid_f(sbv);
          bb = make_float4(sbv, sbv, sbv, sbv);
        }
      } else {
        bb = unpack4(lds_v2(sb + OFF_G + e_kb * 8192 + swz(r, e_ch16) + e_cofs));
        if (kProlog) bb = make_float4(sigmoid_f(bb.x), sigmoid_f(bb.y), sigmoid_f(bb.z), sigmoid_f(bb.w));
      }
      const float4 ke = ke2[rr];
      if (kP3) {
        sts_v2(sb + OFF_XP + o, pack4(ke.x, ke.y, ke.z, ke.w));
        if (r < nvn) {  // rows past the chunk end were zeroed in pass 2
          const uint32_t ov = sb + OFF_V + (uint32_t)e_kb * 8192u + swz(r, e_ch16) + e_cofs;
          const float4 vv = unpack4(lds_v2(ov));
          sts_v2(ov, pack4(vv.x * bb.x, vv.y * bb.y, vv.z * bb.z, vv.w * bb.w));
        }
      } else {
        sts_v2(sb + OFF_XP + o, pack4(bb.x * ke.x, bb.y * ke.y, bb.z * ke.z, bb.w * ke.w));
      }
    }
  };

  for (;;) {
    if (tid == 0) *sUnit = atomicAdd(P.counter, 1);
    __syncthreads();
    const int u = *sUnit;
    if (u >= P.n_units || *sAbort) break;
    const int unit = p.schedule ? p.schedule[u] : u;
    const int n = unit / H, h = unit % H;
    int64_t bos, len;
    if (p.seg_bounds) {
      bos = p.seg_bounds[2 * n];
      len = (int64_t)p.seg_bounds[2 * n + 1] - bos;
    } else if (p.cu_seqlens) {
      bos = p.cu_seqlens[n];
      len = (int64_t)p.cu_seqlens[n + 1] - bos;
    } else {
      bos = (int64_t)n * p.seq_len;
      len = p.seq_len;
    }
    const int nchunks = (int)((len + C - 1) / C);
    // checkpoints for the backward (gdn2_chunk_bwd): slot ci receives the bf16 S_r of chunk ci
    // as this chunk builds it (the swizzled [d_k rows][d_v] tile image the backward copies to
    // shared memory as it is) and the chunk's bf16 T tile; chunks of the token-serial form
    // write nothing
    uint8_t *ck_unit = kCk ? static_cast<uint8_t *>(p.ckpt) + ckpt_first_slot(p.ckpt_off, n, h, H, nchunks) * kCkptBytes
                           : nullptr;
    if (tid == kIssuer && nchunks > 0 && !*sAbort) {
      issue_tma_l(h, (int)bos);
      issue_tma_a(h, (int)bos);
      issue_tma_w(h, (int)bos);
    }

    // ---- initial state into TMEM as S^T (thread: dv channel `row`, dk columns [32 cg, 32 cg + 32));
    //      each load instruction of a warp reads 32 consecutive dv entries of one dk row
    {
      uint32_t r[32];
      if (p.S0) {
        const float *src = p.S0 + ((size_t)unit * D + cg * 32) * D + row;
#pragma unroll
        for (int j = 0; j < 32; ++j) r[j] = __float_as_uint(src[(size_t)j * D]);
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) r[j] = 0u;
      }
      ptx::tmem_st32(tmS + lane_base + cg * 32, r);
      ptx::tmem_wait_st();
    }
    // The state is kept as S = Diag(tau) Sacc (tau per dk channel): each chunk's S_r build
    // rewrites Sacc as e^{L_ref} S, the chunk's increment GEMMs accumulate onto it, and tau
    // becomes that chunk's e^{L_C - L_ref}: S' = e^{L_C - L_ref} (e^{L_ref} S + dS).  tau is
    // read from the previous chunk's sDLb buffer; it is 1 before the first chunk.

    // The operands of chunk c + 1 are built while chunk c's GEMMs run; a unit's first chunk
    // builds them here.
    float4 L[4], ke2[4];
    int wide_next = 0;  // the next chunk to run needs the token-serial form (set by elem_cumsum)
    if (nchunks > 0) {
      const int nv0 = (int)(len < C ? len : C);
      const uint32_t par0 = it & 1u;
      if (kScalarDecay || kScalarGates) {
        const float sv = scal_load((int)bos, nv0, h);
        if (tid < 192) sScN[tid] = sv;
        __syncthreads();
      }
      if (!kScalarDecay) waitb(bar(BAR_TMA_L), par0);
      wide_next = elem_cumsum(par0, (int)bos, nv0, h, L);
      if (tid == kIssuer && !*sAbort) issue_tma_x(h, (int)bos);
      waitb(bar(BAR_TMA_A), par0);
      if (!kScalarGates) waitb(bar(BAR_TMA_W), par0);
      elem_scale((int)bos, nv0, h, L, ke2);
      if (!kScalarGates) waitb(bar(BAR_TMA_X), par0);
      elem_x((int)bos, nv0, h, ke2);
      ptx::fence_proxy_async_smem();
      __syncthreads();
    }

    for (int ci = 0; ci < nchunks; ++ci, ++it) {
      const uint32_t par = it & 1u;
      const int64_t c0 = (int64_t)ci * C;
      const int nvalid = (int)((len - c0) < C ? (len - c0) : C);
      const int t0 = (int)(bos + c0);
      const bool has_next = ci + 1 < nchunks;
      const int nvalid_next = has_next ? (int)((len - c0 - C) < C ? (len - c0 - C) : C) : 0;

      // the log_a slot is free (the b tile it last held was consumed by this chunk's x_r):
      // the next chunk's log_a can land
      if (tid == kIssuer && has_next && !*sAbort) issue_tma_l(h, t0 + C);
      // scalar flags: the next chunk's values, requested now and stored before the barrier
      // that ends the masks (this chunk's were read while the previous chunk built its operands)
      float scal_next = 0.f;
      if ((kScalarDecay || kScalarGates) && has_next) scal_next = scal_load(t0 + C, nvalid_next, h);

      if (wide_next) {
        // ---- a decay range beyond the factored form: the recurrence token by token.  The
        //      chunk's operand tiles are not used; its raw inputs are re-read from global memory.
        if (ci > 0) {  // the previous chunk's GEMMs (the last of them updates the state) are done
          waitb(bar(BAR_G5), par ^ 1u);
          ptx::tc_fence_after();
        }
        if (tid == kIssuer) ptx::bulk_wait_group_read0();  // the previous o store has read the staging area
        if ((kScalarDecay || kScalarGates) && tid < 192) sScN[tid] = scal_next;
        __syncthreads();
        // One arrival per chunk on every MMA barrier keeps their phases in step with the chunk
        // count (plain arrivals: this chunk issues no MMA, and the previous chunk's are done).
        // They come after the barrier above: every thread has then seen the previous chunk's G5
        // phase complete, so no wait can find that barrier two phases ahead.
        if (tid == 0) {
          ptx::mbar_arrive(bar(BAR_G1));
          ptx::mbar_arrive(bar(BAR_E1));
          ptx::mbar_arrive(bar(BAR_GA));
          ptx::mbar_arrive(bar(BAR_GB));
          ptx::mbar_arrive(bar(BAR_G4));
          ptx::mbar_arrive(bar(BAR_G5));
        }
        // the tiles of this chunk are dead: the next chunk's w, k, q, v can land now
        if (tid == kIssuer && has_next && !*sAbort) {
          issue_tma_w(h, t0 + C);
          issue_tma_a(h, t0 + C);
        }
        serial_chunk<kScalarDecay, kScalarGates, kP3, kProlog, Tout>(p, gb, tmS + lane_base + cg * 32,
                                                                   ci > 0 ? sDLb(par ^ 1u) + cg * 32 : nullptr,
                                                                   t0, nvalid, h);
        if (tid < D) sDLb(par)[tid] = 1.f;  // the next chunk reads the state with tau = 1
        // the staging covered the bf16 T tile, whose blocks above the diagonal the solve never
        // writes: zero it again
        sts_v4(sb + OFF_T + 16u * (uint32_t)tid, make_uint4(0u, 0u, 0u, 0u));
        // the next chunk's operands, as the factored path builds them under its GEMMs
        if (has_next) {
          if (!kScalarDecay) waitb(bar(BAR_TMA_L), par ^ 1u);
          wide_next = elem_cumsum(par ^ 1u, t0 + C, nvalid_next, h, L);
          if (tid == kIssuer && !*sAbort) issue_tma_x(h, t0 + C);
          waitb(bar(BAR_TMA_A), par ^ 1u);
          if (!kScalarGates) waitb(bar(BAR_TMA_W), par ^ 1u);
          elem_scale(t0 + C, nvalid_next, h, L, ke2);
          if (!kScalarGates) waitb(bar(BAR_TMA_X), par ^ 1u);
          elem_x(t0 + C, nvalid_next, h, ke2);
        }
        ptx::fence_proxy_async_smem();
        ptx::tc_fence_before();
        __syncthreads();
        if (*sAbort) break;
        continue;
      }

      // ---- a4: G1 [A B; QX QP] = [k_r; q_r] [x_r; p_r]^T, issued first: it needs only this
      //      chunk's operands (built during the previous chunk) and runs under the S_r build
      if (tid == 0 && !*sAbort) {
        ptx::tc_fence_after();
        constexpr uint32_t id1 = ptx::idesc_bf16(128, kXP ? 64 : 128, false, false);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t ko = (uint32_t)(kk >> 2) * 16384u + (uint32_t)(kk & 3) * 32u;
          ptx::umma_bf16(tmD1, ptx::sdesc_sw128(sb + OFF_KQ + ko, 16, 1024),
                         ptx::sdesc_sw128(sb + OFF_XP + ko, 16, 1024), id1, kk > 0);
        }
        ptx::umma_commit(bar(BAR_G1));
      }

      // ---- S_r^T = S^T Diag(e^{L_ref}) as the bf16 TMEM A operand (thread: dv channel `row`,
      //      dk columns [32 cg, 32 cg + 32)); the fp32 accumulator becomes the same, and the
      //      chunk's increment GEMMs accumulate onto it
      {
        // two products, in this order: tau * Sacc is the state, O(1); e^{L_ref} tau alone can
        // underflow (both factors reach e^{-80} under the range precondition)
        const float *tp = sDLb(par ^ 1u) + cg * 32;
        const float *smv = sSM + cg * 32;
        uint32_t r[32], hb[16];
        if (ci > 0) {  // the previous chunk's increment GEMMs have landed in the state
          waitb(bar(BAR_G5), par ^ 1u);
          ptx::tc_fence_after();
        }
        ptx::tmem_ld32(tmS + lane_base + cg * 32, r);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int j4 = 0; j4 < 8; ++j4) {
          const float4 t4 = ci > 0 ? *reinterpret_cast<const float4 *>(tp + 4 * j4) : make_float4(1.f, 1.f, 1.f, 1.f);
          const float4 s4 = *reinterpret_cast<const float4 *>(smv + 4 * j4);
          const float f0 = (__uint_as_float(r[4 * j4]) * t4.x) * s4.x;
          const float f1 = (__uint_as_float(r[4 * j4 + 1]) * t4.y) * s4.y;
          const float f2 = (__uint_as_float(r[4 * j4 + 2]) * t4.z) * s4.z;
          const float f3 = (__uint_as_float(r[4 * j4 + 3]) * t4.w) * s4.w;
          r[4 * j4] = __float_as_uint(f0);
          r[4 * j4 + 1] = __float_as_uint(f1);
          r[4 * j4 + 2] = __float_as_uint(f2);
          r[4 * j4 + 3] = __float_as_uint(f3);
          hb[2 * j4] = pack_bf16x2(f0, f1);
          hb[2 * j4 + 1] = pack_bf16x2(f2, f3);
        }
        ptx::tmem_st32(tmS + lane_base + cg * 32, r);
        ptx::tmem_st16(tmSR + lane_base + cg * 16, hb);
        if (ck_unit) {
          // S_r[i][j] of this chunk (i = 32 cg + jj, j = `row`) into the o staging area, which a
          // checkpointing forward (no o) leaves free; one bulk copy takes the image to the slot.
          // The previous chunk's copies have read the area (bulk_wait_group_read0 after GB).
#pragma unroll
          for (int jj = 0; jj < 32; ++jj) {
            const uint32_t pair = hb[jj >> 1];
            sts_u16(sb + OFF_OS + swz_elem(cg * 32 + jj, row, 16384u), (uint16_t)((jj & 1) ? (pair >> 16) : (pair & 0xffffu)));
          }
          ptx::fence_proxy_async_smem();
        }
        ptx::tmem_wait_st();
      }
      ptx::tc_fence_before();
      __syncthreads();
      if (ck_unit && tid == kIssuer && !*sAbort) {
        ptx::bulk_store(ck_unit + (size_t)ci * kCkptBytes, sb + OFF_OS, 32768u);
        ptx::bulk_commit_group();
      }


      waitb(bar(BAR_G1), par);
      ptx::tc_fence_after();

      // masks: A, B strictly lower (fp32 A for the solve, bf16 B); QX, QP lower incl. diagonal.
      // warp (qd, cg) reads D1 columns [32 cg, 32 cg + 32); with kXP only columns 0-63 exist.
      // The checkpointing forward writes no o: QX and QP (rows 64-127) are not needed.
      if ((!kXP || cg < 2) && !(kCk && qd >= 2)) {
        float *Af = reinterpret_cast<float *>(gb + OFF_AF);
        uint32_t r[32];
        ptx::tmem_ld32(tmD1 + lane_base + cg * 32, r);
        ptx::tmem_wait_ld();
        const int jb = (cg & 1) * 32;  // column offset inside the 64-wide matrix
        float f[32];
        if (qd < 2) {
          const int i = row;
#pragma unroll
          for (int j = 0; j < 32; ++j) f[j] = (jb + j < i) ? __uint_as_float(r[j]) : 0.f;
          if (cg < 2) {
#pragma unroll
            for (int j4 = 0; j4 < 8; ++j4)
              *reinterpret_cast<float4 *>(Af + fidx(i, jb + 4 * j4)) =
                  make_float4(f[4 * j4], f[4 * j4 + 1], f[4 * j4 + 2], f[4 * j4 + 3]);
            if (kXP) {  // B = A
#pragma unroll
              for (int q8 = 0; q8 < 4; ++q8)
                sts_v4(sb + OFF_BM + swz(i, (uint32_t)((cg & 1) * 4 + q8)), pack8(f + 8 * q8, 1.f));
            }
          } else {
#pragma unroll
            for (int q8 = 0; q8 < 4; ++q8)
              sts_v4(sb + OFF_BM + swz(i, (uint32_t)((cg & 1) * 4 + q8)), pack8(f + 8 * q8, 1.f));
          }
        } else {
          const int i = row - 64;
#pragma unroll
          for (int j = 0; j < 32; ++j) f[j] = (jb + j <= i) ? __uint_as_float(r[j]) : 0.f;
          const uint32_t dst = (cg < 2 && !kXP) ? OFF_QX : OFF_QP;  // with x_r == p_r, QX = QP: one slot
#pragma unroll
          for (int q8 = 0; q8 < 4; ++q8)
            sts_v4(sb + dst + swz(i, (uint32_t)((cg & 1) * 4 + q8)), pack8(f + 8 * q8, 1.f));
        }
      }
      // a proxy fence costs each thread that runs it far more than a barrier: only the warps
      // whose stores an MMA reads (B, QX, QP) run it; the fp32 A is read by the solve's threads
      if (kXP ? (cg < 2) : !(qd < 2 && cg < 2)) ptx::fence_proxy_async_smem();
      if ((kScalarDecay || kScalarGates) && tid < 192) sScN[tid] = scal_next;
      ptx::tc_fence_before();
      __syncthreads();

      // ---- a6 (T-independent MMAs, issued by warp 15 while warps 0-14 solve; one issuing thread
      //      keeps them in order, and the issue stalls of the MMA queue delay nobody):
      //        dS = p_r^T V                                                        (commit E1)
      //        [R^T | O^T] = V^T [B; QP]^T + S_r^T [k_r; q_r]^T, one N = 128 product each:
      //          R = B V + k_r S_r is the right-hand side of M = T R,
      //          M = (I + A)^-1 (B V + Ytilde S) with Ytilde S = k_r S_r;
      //          O^T = S_r^T q_r^T + V^T QP^T before the erase term                (commit GA)
      if (warp == kIssueWarp) {
        if (lane == 0 && !*sAbort) {
          ptx::tc_fence_after();
          // dS^T = V^T p_r: A = V^T (MN-major), B = p_r as [tokens][dk] (MN-major, N = 128)
          constexpr uint32_t idS = ptx::idesc_bf16(128, 128, true, true);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            ptx::umma_bf16(tmS, ptx::sdesc_sw128(sb + OFF_V + kk * 2048, 8192, 1024),
                           ptx::sdesc_sw128(sb + OFF_XP + 8192 + kk * 2048, 16384, 1024), idS, 1);
          ptx::umma_commit(bar(BAR_E1));
          // the checkpointing forward writes no o: R^T alone (N = 64, the B and k_r rows)
          constexpr uint32_t idV = ptx::idesc_bf16(128, kCk ? 64 : 128, true, false);   // A = V^T (MN-major)
          constexpr uint32_t idT = ptx::idesc_bf16(128, kCk ? 64 : 128, false, false);  // A from TMEM
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            ptx::umma_bf16(tmD1, ptx::sdesc_sw128(sb + OFF_V + kk * 2048, 8192, 1024),
                           ptx::sdesc_sw128(sb + OFF_BM + kk * 32, 16, 1024), idV, kk > 0);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            ptx::umma_bf16_ts(tmD1, tmSR + kk * 8,
                              ptx::sdesc_sw128(sb + OFF_KQ + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024), idT, 1);
          ptx::umma_commit(bar(BAR_GA));
          if (has_next) {  // p_r is dead once dS = p_r^T V is done: the next chunk's w can land
            waitb(bar(BAR_E1), par);
            if (!*sAbort) issue_tma_w(h, t0 + C);
            // k_r, q_r and V are dead once GA is done: the next chunk's k, q, v tiles can land
            // (the solve runs meanwhile, so this wait delays nobody)
            waitb(bar(BAR_GA), par);
            if (!*sAbort) issue_tma_a(h, t0 + C);
          }
        }
        __syncwarp();
      } else {

      // ---- a5: T = (I + A)^-1 (fp32).  8x8 diagonal blocks by forward substitution, then three
      //      merge levels: for each pair of diagonal blocks of size s (upper U, lower L) of the
      //      merged 2s block, T_LU = -T_LL (A_LU T_UU).  Blocks above the diagonal are never
      //      read (loops stop at the triangle), so they are never written either.  Each block
      //      also goes to the bf16 T tile (the MMA operand) as soon as it is final; the tile's
      //      blocks above the diagonal hold the zeros written at the kernel's start.
      {
        const float *Af = reinterpret_cast<const float *>(gb + OFF_AF);
        float *Tf = reinterpret_cast<float *>(gb + OFF_TF);
        float *Xs = reinterpret_cast<float *>(gb + OFF_XS);
        if (tid < 64) {
          const int r0 = 8 * (tid >> 3), m = tid & 7;
          float a[28];
          {
            int n = 0;
#pragma unroll
            for (int i = 1; i < 8; ++i)
#pragma unroll
              for (int j = 0; j < i; ++j) a[n++] = Af[fidx(r0 + i, r0 + j)];
          }
          float t[8];
          int n = 0;
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            float acc = (i == m) ? 1.f : 0.f;
#pragma unroll
            for (int j = 0; j < i; ++j) acc -= a[n++] * t[j];
            t[i] = acc;
          }
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            Tf[fidx(r0 + i, r0 + m)] = t[i];
            sts_u16(sb + OFF_T + swz(r0 + i, (uint32_t)(r0 >> 3)) + (uint32_t)m * 2u, bf16_bits(t[i]));
          }
        }
        named_bar(NB_SOLVE, kSolveThreads);
        // s = 8: 4 pairs x 64 outputs on CUDA cores
        if (tid < 256) {
          const int pr = tid >> 6, r = (tid >> 3) & 7, c = tid & 7, u0 = 16 * pr, l0 = u0 + 8;
          float acc = 0.f;
#pragma unroll
          for (int k = 0; k < 8; ++k) acc += (k >= c ? Af[fidx(l0 + r, u0 + k)] * Tf[fidx(u0 + k, u0 + c)] : 0.f);
          Xs[tid] = acc;
        }
        named_bar(NB_SOLVE, kSolveThreads);
        if (tid < 256) {
          const int pr = tid >> 6, r = (tid >> 3) & 7, c = tid & 7, u0 = 16 * pr, l0 = u0 + 8;
          float acc = 0.f;
#pragma unroll
          for (int k = 0; k < 8; ++k) acc -= (k <= r ? Tf[fidx(l0 + r, l0 + k)] * Xs[pr * 64 + k * 8 + c] : 0.f);
          Tf[fidx(l0 + r, u0 + c)] = acc;
          sts_u16(sb + OFF_T + swz(l0 + r, (uint32_t)(u0 >> 3)) + (uint32_t)c * 2u, bf16_bits(acc));
        }
        named_bar(NB_SOLVE, kSolveThreads);
        // s = 16 (2 pairs) and s = 32 (1 pair) on tf32 mma.sync: one warp per 16x8 output tile.
        // Every fragment of a step is loaded before its chain of MMAs starts.
        const int g = lane >> 2, t4 = lane & 3;
#pragma unroll
        for (int lev = 1; lev < 3; ++lev) {
          const int sz = 8 << lev;                   // 16, 32
          const int nk = sz / 8;                     // 8-wide K steps: 2, 4
          const int tpp = (sz / 16) * (sz / 8);      // 16x8 tiles per pair: 2, 8
          const int ntiles = (64 / (2 * sz)) * tpp;  // 4, 8
          const int pr = warp / tpp, ti = warp % tpp, mt = ti / (sz / 8), nt = ti % (sz / 8);
          const int u0 = pr * 2 * sz, l0 = u0 + sz, rr = 16 * mt, cc = 8 * nt;
          // step a: X = A_LU T_UU (only K steps from the tile's first column on contribute;
          // the blocks of T_UU above its diagonal were never written)
          if (warp < ntiles) {
            uint32_t av[4][4], bv[4][2];
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              if (kk < nk && kk >= nt) {
                const int kc = u0 + 8 * kk + t4;
                av[kk][0] = ptx::to_tf32(Af[fidx(l0 + rr + g, kc)]);
                av[kk][1] = ptx::to_tf32(Af[fidx(l0 + rr + g + 8, kc)]);
                av[kk][2] = ptx::to_tf32(Af[fidx(l0 + rr + g, kc + 4)]);
                av[kk][3] = ptx::to_tf32(Af[fidx(l0 + rr + g + 8, kc + 4)]);
                bv[kk][0] = ptx::to_tf32(Tf[fidx(kc, u0 + cc + g)]);
                bv[kk][1] = ptx::to_tf32(Tf[fidx(kc + 4, u0 + cc + g)]);
              }
            }
            float x[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              if (kk < nk && kk >= nt) ptx::mma_tf32_16x8x8(x, av[kk], bv[kk]);
            float *xs = Xs + pr * sz * sz;
            xs[(rr + g) * sz + cc + 2 * t4] = x[0];
            xs[(rr + g) * sz + cc + 2 * t4 + 1] = x[1];
            xs[(rr + g + 8) * sz + cc + 2 * t4] = x[2];
            xs[(rr + g + 8) * sz + cc + 2 * t4 + 1] = x[3];
          }
          named_bar(NB_SOLVE, kSolveThreads);
          // step b: T_LU = -T_LL X (only K steps up to the tile's last row contribute)
          if (warp < ntiles) {
            const float *xs = Xs + pr * sz * sz;
            uint32_t av[4][4], bv[4][2];
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              if (kk < nk && kk <= (rr + 15) / 8) {
                // T_LL is lower triangular; its 8x8 blocks above the diagonal were never written
                const int kc = l0 + 8 * kk + t4, kr = 8 * kk + t4;
                av[kk][0] = ptx::to_tf32(kr <= rr + g ? Tf[fidx(l0 + rr + g, kc)] : 0.f);
                av[kk][1] = ptx::to_tf32(kr <= rr + g + 8 ? Tf[fidx(l0 + rr + g + 8, kc)] : 0.f);
                av[kk][2] = ptx::to_tf32(kr + 4 <= rr + g ? Tf[fidx(l0 + rr + g, kc + 4)] : 0.f);
                av[kk][3] = ptx::to_tf32(kr + 4 <= rr + g + 8 ? Tf[fidx(l0 + rr + g + 8, kc + 4)] : 0.f);
                bv[kk][0] = ptx::to_tf32(xs[(8 * kk + t4) * sz + cc + g]);
                bv[kk][1] = ptx::to_tf32(xs[(8 * kk + t4 + 4) * sz + cc + g]);
              }
            }
            float y[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              if (kk < nk && kk <= (rr + 15) / 8) ptx::mma_tf32_16x8x8(y, av[kk], bv[kk]);
            const int ri = l0 + rr + g, cj = u0 + cc + 2 * t4;
            if (lev == 1) {  // the last level's T_LU is read by no later level: bf16 only
              Tf[fidx(ri, cj)] = -y[0];
              Tf[fidx(ri, cj + 1)] = -y[1];
              Tf[fidx(ri + 8, cj)] = -y[2];
              Tf[fidx(ri + 8, cj + 1)] = -y[3];
            }
            sts_u32(sb + OFF_T + swz(ri, (uint32_t)(cj >> 3)) + (uint32_t)(cj & 7) * 2u, pack_bf16x2(-y[0], -y[1]));
            sts_u32(sb + OFF_T + swz(ri + 8, (uint32_t)(cj >> 3)) + (uint32_t)(cj & 7) * 2u, pack_bf16x2(-y[2], -y[3]));
          }
          if (lev == 1) named_bar(NB_SOLVE, kSolveThreads);
        }
        }  // solve scope
      }  // warps 0-14
      if (warp < 8) ptx::fence_proxy_async_smem();  // warps 0-7 wrote the bf16 T tile
      ptx::tc_fence_before();
      __syncthreads();
      // the backward's checkpoint also keeps this chunk's bf16 T (the tile image after S_r); the
      // issuing thread waits for this copy's reads before the next chunk's solve rewrites it
      // (bulk_wait_group_read0 before the epilogue below)
      if (ck_unit && tid == kIssuer && !*sAbort) {
        ptx::bulk_store(ck_unit + (size_t)ci * kCkptBytes + kCkptT, sb + OFF_T, 8192u);
        ptx::bulk_commit_group();
      }

      // ---- R^T (fp32, D1 cols 0-63) -> bf16 TMEM A operand
      waitb(bar(BAR_GA), par);
      ptx::tc_fence_after();
      {
        uint32_t r[16], hb[8];
        ptx::tmem_ld16(tmD1 + lane_base + cg * 16, r);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 8; ++j) hb[j] = pack_bf16x2(__uint_as_float(r[2 * j]), __uint_as_float(r[2 * j + 1]));
        ptx::tmem_st8(tmRb + lane_base + cg * 8, hb);
        ptx::tmem_wait_st();
      }
      ptx::tc_fence_before();
      __syncthreads();

      // ---- a7 (erase reads): M^T = R^T T^T (own 64 columns); row i of M is r_i = Sbar_i^T k_i
      if (tid == 0 && !*sAbort) {
        ptx::tc_fence_after();
        constexpr uint32_t idM = ptx::idesc_bf16(128, 64, false, false);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          ptx::umma_bf16_ts(tmM, tmRb + kk * 8, ptx::sdesc_sw128(sb + OFF_T + kk * 32, 16, 1024), idM, kk > 0);
        ptx::umma_commit(bar(BAR_GB));
      }
      // ---- while M^T is computed: the next chunk's cumulative decay (its log_a tile landed
      //      during the solve); then its b tile may take the log_a slot
      if (has_next) {
        if (!kScalarDecay) waitb(bar(BAR_TMA_L), par ^ 1u);
        wide_next = elem_cumsum(par ^ 1u, t0 + C, nvalid_next, h, L);
        if (tid == kIssuer && !*sAbort) issue_tma_x(h, t0 + C);
      }
      waitb(bar(BAR_GB), par);
      ptx::tc_fence_after();
      {  // -M^T -> bf16 TMEM A operand
        uint32_t r[16], hb[8];
        ptx::tmem_ld16(tmM + lane_base + cg * 16, r);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 8; ++j) hb[j] = pack_bf16x2(-__uint_as_float(r[2 * j]), -__uint_as_float(r[2 * j + 1]));
        ptx::tmem_st8(tmMb + lane_base + cg * 8, hb);
        ptx::tmem_wait_st();
      }
      if (tid == kIssuer) ptx::bulk_wait_group_read0();  // the previous chunk's o store has read the staging
      ptx::tc_fence_before();
      __syncthreads();

      // ---- a7: the state-dependent remainder of O^T and dS
      if (tid == 0 && !*sAbort) {
        ptx::tc_fence_after();
        constexpr uint32_t idO = ptx::idesc_bf16(128, 64, false, false);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          if (!kCk)
            ptx::umma_bf16_ts(tmO, tmMb + kk * 8, ptx::sdesc_sw128(sb + (kXP ? OFF_QP : OFF_QX) + kk * 32, 16, 1024), idO, 1);
        ptx::umma_commit(bar(BAR_G4));  // O^T is complete: the epilogue need not wait for dS
        // dS^T += (-M^T) x_r: B = x_r as [tokens][dk] (MN-major, N = 128)
        constexpr uint32_t idS = ptx::idesc_bf16(128, 128, false, true);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          ptx::umma_bf16_ts(tmS, tmMb + kk * 8, ptx::sdesc_sw128(sb + OFF_XP + kk * 2048, 16384, 1024), idS, 1);
        ptx::umma_commit(bar(BAR_G5));  // the state is complete (waited for by the next S_r build)
      }
      // ---- while O^T and dS are finished: the next chunk's k_r, q_r, p_r (its k, q, v tiles
      //      landed during the solve, its w tile once dS = p_r^T V was done)
      if (has_next) {
        waitb(bar(BAR_TMA_A), par ^ 1u);
        if (!kScalarGates) waitb(bar(BAR_TMA_W), par ^ 1u);
        elem_scale(t0 + C, nvalid_next, h, L, ke2);
      }
      waitb(bar(BAR_G4), par);
      ptx::tc_fence_after();

      // ---- a8: outputs (the state was updated by the increment GEMMs)
      if (p.o) {
        // o^T: lane = dv channel `row`, columns = tokens [16 cg, 16 cg + 16)
        uint32_t r[16];
        ptx::tmem_ld16(tmO + lane_base + cg * 16, r);
        ptx::tmem_wait_ld();
        // staging: sub-blocks of [64 tokens][128 B] (64 bf16 or 32 fp32 channels), 8 KB each
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int i = cg * 16 + j;
          const float f = __uint_as_float(r[j]);
          if (sizeof(Tout) == 2) {
            const __nv_bfloat16 hv = __float2bfloat16_rn(f);
            sts_u16(sb + OFF_OS + (uint32_t)(row >> 6) * 8192u + (uint32_t)i * 128u + (uint32_t)(row & 63) * 2u,
                    *reinterpret_cast<const uint16_t *>(&hv));
          } else {
            sts_f32(sb + OFF_OS + (uint32_t)(row >> 5) * 8192u + (uint32_t)i * 128u + (uint32_t)(row & 31) * 4u, f);
          }
        }
      }
      // ---- the next chunk's x_r, once dS (the last reader of this chunk's x_r) is done
      if (has_next) {
        waitb(bar(BAR_G5), par);
        if (!kScalarGates) waitb(bar(BAR_TMA_X), par ^ 1u);
        elem_x(t0 + C, nvalid_next, h, ke2);
      }
      // one proxy fence per thread covers the o staging (read by the TMA store below) and the
      // next chunk's operands (read by its G1)
      ptx::fence_proxy_async_smem();
      ptx::tc_fence_before();
      __syncthreads();
      if (!p.o) {
        // no output requested (the checkpointing forward of the backward)
      } else if (nvalid == C) {
        // full chunk: asynchronous TMA store; the next chunk's epilogue rewrites the staging
        // area only after the issuing thread has seen these reads done (bulk_wait_group_read0)
        if (tid == kIssuer) {
          constexpr int kBoxC = sizeof(Tout) == 2 ? 64 : 32;
#pragma unroll
          for (int sbk = 0; sbk < D / kBoxC; ++sbk)
            ptx::tma_store_3d(&P.tm_o, sb + OFF_OS + (uint32_t)sbk * 8192u, sbk * kBoxC, h, t0);
          ptx::bulk_commit_group();
        }
      } else {
        // tail chunk: plain stores of the valid rows only
        constexpr int kRowBytes = D * (int)sizeof(Tout);
        constexpr int kU4 = kRowBytes / 16;
        uint8_t *go = static_cast<uint8_t *>(p.o);
        for (int e = tid; e < nvalid * kU4; e += kThreads) {
          const int i = e / kU4, uu = e % kU4;
          const uint4 val = lds_v4(sb + OFF_OS + (uint32_t)(uu >> 3) * 8192u + (uint32_t)i * 128u + (uint32_t)(uu & 7) * 16u);
          *reinterpret_cast<uint4 *>(go + ((size_t)(t0 + i) * H + h) * kRowBytes + uu * 16) = val;
        }
      }
      if (*sAbort) break;
    }

    // ---- a8: final state S = Diag(tau) Sacc, from S^T (thread: dv channel `row`, dk rows
    //      [32 cg, 32 cg + 32); each store instruction of a warp writes 32 consecutive dv entries).
    //      The last chunk's increment GEMMs must have landed (also before the next unit's S0).
    if (nchunks > 0) {
      waitb(bar(BAR_G5), (it & 1u) ^ 1u);
      ptx::tc_fence_after();
    }
    if (p.S_T && !*sAbort) {
      float *dst = p.S_T + ((size_t)unit * D + cg * 32) * D + row;
      const float *tp = sDLb((it & 1u) ^ 1u) + cg * 32;  // the last chunk's e^{L_C - L_ref}
      uint32_t r[32];
      ptx::tmem_ld32(tmS + lane_base + cg * 32, r);
      ptx::tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < 32; ++j) dst[(size_t)j * D] = (nchunks > 0 ? tp[j] : 1.f) * __uint_as_float(r[j]);
    }
    ptx::tc_fence_before();
    __syncthreads();
  }

  if (tid == kIssuer) ptx::bulk_wait_group0();
  if (*sAbort) {
    // wind-down after a timed-out wait (every wait of the loop then returned at once): let the
    // MMAs of the two issuing threads and the last armed phase of every TMA barrier finish,
    // each within the wait limit, before the tensor memory is freed and the CTA leaves
    if (tid == 0) {
      ptx::umma_commit(bar(BAR_DRAIN0));
      drain_bar(bar(BAR_DRAIN0), 0u, P.wait_ns);
#pragma unroll
      for (int b = BAR_TMA_A; b <= BAR_TMA_X; ++b)
        if (sIss[b] > 0u) drain_bar(bar(b), (sIss[b] - 1u) & 1u, P.wait_ns);
    }
    if (warp == kIssueWarp && lane == 0) {
      ptx::umma_commit(bar(BAR_DRAIN1));
      drain_bar(bar(BAR_DRAIN1), 0u, P.wait_ns);
    }
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

// o: [T_tot][H][128] of bf16 or fp32 viewed as (channel, head, token); box of 128 bytes of
// channels x 1 head x 64 tokens, unswizzled (matches the kernel's staging sub-blocks).
bool make_map_o(CUtensorMap *m, void *base, int64_t t_total, int H, bool bf16) {
  auto enc = get_encode();
  if (!enc) return false;
  const cuuint64_t es = bf16 ? 2 : 4;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)t_total};
  cuuint64_t strides[2] = {(cuuint64_t)D * es, (cuuint64_t)H * D * es};
  cuuint32_t box[3] = {bf16 ? 64u : 32u, 1, 64};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, base, dims,
                   strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                   CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <bool SD, bool SG, bool P3, bool PR, bool XP, typename Tout, bool CK = false>
cudaError_t launch_t(const TcParams &P, int grid, cudaStream_t stream) {
  auto kern = chunk_tc_kernel<SD, SG, P3, PR, XP, Tout, CK>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  kern<<<grid, kThreads, kSmemBytes, stream>>>(P);
  return cudaGetLastError();
}

template <bool P3, bool PR, bool XP>
cudaError_t launch_gates(const TcParams &P, int grid, cudaStream_t stream, bool sd, bool sg, bool obf) {
  if (sd && sg)
    return obf ? launch_t<true, true, P3, PR, XP, __nv_bfloat16>(P, grid, stream)
               : launch_t<true, true, P3, PR, XP, float>(P, grid, stream);
  if (sd)
    return obf ? launch_t<true, false, P3, PR, XP, __nv_bfloat16>(P, grid, stream)
               : launch_t<true, false, P3, PR, XP, float>(P, grid, stream);
  if (sg)
    return obf ? launch_t<false, true, P3, PR, XP, __nv_bfloat16>(P, grid, stream)
               : launch_t<false, true, P3, PR, XP, float>(P, grid, stream);
  return obf ? launch_t<false, false, P3, PR, XP, __nv_bfloat16>(P, grid, stream)
             : launch_t<false, false, P3, PR, XP, float>(P, grid, stream);
}

// the checkpointing forward: activated inputs (no prologue) and no o, so one output type
template <bool P3, bool XP>
cudaError_t launch_gates_ck(const TcParams &P, int grid, cudaStream_t stream, bool sd, bool sg) {
  using B = __nv_bfloat16;
  if (sd) return sg ? launch_t<true, true, P3, false, XP, B, true>(P, grid, stream)
                    : launch_t<true, false, P3, false, XP, B, true>(P, grid, stream);
  return sg ? launch_t<false, true, P3, false, XP, B, true>(P, grid, stream)
            : launch_t<false, false, P3, false, XP, B, true>(P, grid, stream);
}

}  // namespace

bool make_row_tile_map(CUtensorMap *m, const void *base, int64_t t_total, int H) {
  return make_map(m, base, t_total, H);
}

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
  const bool p3 = (p.flags & GDN2_GATE_FORM_P3) != 0;
  TcParams P;
  memset(&P, 0, sizeof(P));
  P.p = p;
  P.n_units = p.n_seqs * p.n_heads;
  P.counter = p.status + 1;
  P.wait_ns = kWaitTimeoutNs;
  if (P.n_units == 0) return cudaSuccess;
  const int64_t T = p.t_total > 0 ? p.t_total : 1;
  bool ok = make_map(&P.tm_q, p.q, T, p.n_heads) && make_map(&P.tm_k, p.k, T, p.n_heads) &&
            make_map(&P.tm_v, p.v, T, p.n_heads);
  if (ok && !sd) ok = make_map(&P.tm_g, p.log_a, T, p.n_heads);
  // tm_w feeds the first elementwise pass and tm_b the second; the gist.science form
  // needs its erase gate first and its value gate (w, d_v = d_k channels) second.
  const void *g_first = p3 ? p.b : (tied ? p.b : p.w);
  const void *g_second = p3 ? (tied ? p.b : p.w) : p.b;
  if (ok && !sg) ok = make_map(&P.tm_b, g_second, T, p.n_heads) && make_map(&P.tm_w, g_first, T, p.n_heads);
  if (ok && p.o) ok = make_map_o(&P.tm_o, p.o, T, p.n_heads, p.dtype_out == GDN2_BF16);
  if (!ok) {
    *why = "cuTensorMapEncodeTiled failed (driver entry point missing or bad tensor geometry)";
    return cudaErrorInvalidValue;
  }
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = P.n_units < sms ? P.n_units : sms;
  const bool obf = p.dtype_out == GDN2_BF16;
  const bool pr = (p.flags & GDN2_FUSED_PROLOGUE) != 0;
  uint64_t hook_ns = 0;
  if (take_debug_timeout(GDN2_DEBUG_CHUNK, &hook_ns)) {  // the timeout test hook, armed for this launch
    P.dbg_skip = 1;
    P.wait_ns = hook_ns;
  }
  if (p.ckpt) {
    if (pr || p.o) {
      *why = "the checkpointing forward takes activated inputs and writes no o";
      return cudaErrorNotSupported;
    }
    if (p3) return launch_gates_ck<true, true>(P, grid, stream, sd, sg);
    return tied ? launch_gates_ck<false, true>(P, grid, stream, sd, sg)
                : launch_gates_ck<false, false>(P, grid, stream, sd, sg);
  }
  // x_r == p_r in the gist.science form, and in the default form when w is b
  if (p3)
    return pr ? launch_gates<true, true, true>(P, grid, stream, sd, sg, obf)
              : launch_gates<true, false, true>(P, grid, stream, sd, sg, obf);
  if (tied)
    return pr ? launch_gates<false, true, true>(P, grid, stream, sd, sg, obf)
              : launch_gates<false, false, true>(P, grid, stream, sd, sg, obf);
  return pr ? launch_gates<false, true, false>(P, grid, stream, sd, sg, obf)
            : launch_gates<false, false, false>(P, grid, stream, sd, sg, obf);
}

}  // namespace gdn2
