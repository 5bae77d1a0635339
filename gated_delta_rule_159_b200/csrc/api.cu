// api.cu -- the extern "C" entry points declared in include/gdn2.h: argument
// validation, workspace layout, unit scheduling and kernel dispatch.  Nothing
// here computes the recurrence; every step of it runs in the kernels.
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <vector>

#include "internal.h"

namespace {

thread_local char g_err[512] = "";

int fail(int code, const char *fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return code;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

constexpr uint32_t kKnownFlags =
    GDN2_SCALAR_DECAY | GDN2_SCALAR_GATES | GDN2_TIED_GATES | GDN2_GATE_FORM_P3 | GDN2_FUSED_PROLOGUE;
constexpr size_t kWsHeader = 256;     // [0] status word, [1] unit counter
constexpr int kMaxSortedSeqs = 4096;  // above this the units run in index order

// Longest-first order of the (sequence, head) units of a packed batch: rank each
// sequence by length (ties by index) and list its heads at that rank.
__global__ void schedule_kernel(const int32_t *cu, int N, int H, int32_t *sched) {
  for (int n = threadIdx.x; n < N; n += blockDim.x) {
    const int len = cu[n + 1] - cu[n];
    int rank = 0;
    for (int m = 0; m < N; ++m) {
      const int lm = cu[m + 1] - cu[m];
      rank += (lm > len) || (lm == len && m < n);
    }
    for (int h = 0; h < H; ++h) sched[rank * H + h] = n * H + h;
  }
}

int check_dims(const gdn2_dims *d) {
  if (!d) return fail(GDN2_ERR_INVALID_ARG, "dims is NULL");
  if (d->reserved != 0) return fail(GDN2_ERR_INVALID_ARG, "dims.reserved must be 0");
  if (d->n_seqs < 1 || d->n_heads < 1 || d->seq_len < 0 || d->d_k < 1 || d->d_v < 1)
    return fail(GDN2_ERR_INVALID_ARG, "bad dims (n_seqs=%d n_heads=%d seq_len=%d d_k=%d d_v=%d)", d->n_seqs,
                d->n_heads, d->seq_len, d->d_k, d->d_v);
  if ((d->dtype_in != GDN2_BF16 && d->dtype_in != GDN2_F32) || (d->dtype_out != GDN2_BF16 && d->dtype_out != GDN2_F32))
    return fail(GDN2_ERR_INVALID_ARG, "bad dtype_in=%d / dtype_out=%d", d->dtype_in, d->dtype_out);
  if (d->flags & ~kKnownFlags) return fail(GDN2_ERR_INVALID_ARG, "unknown flag bits 0x%x", d->flags & ~kKnownFlags);
  if ((d->flags & GDN2_GATE_FORM_P3) && (d->flags & GDN2_TIED_GATES) && !(d->flags & GDN2_SCALAR_GATES) &&
      d->d_k != d->d_v)
    return fail(GDN2_ERR_INVALID_ARG, "tied per-channel gates in the GDN2_GATE_FORM_P3 form need d_k == d_v "
                "(b has d_k channels, w has d_v)");
  return GDN2_OK;
}

// Per-channel tensors are read by TMA or vector loads and need 16-byte alignment;
// the [T, H] scalar-gate arrays are read element by element and need only
// element alignment.
int check_inputs(const void *q, const void *k, const void *v, const void *log_a, const void *b, const void *w,
                 uint32_t flags, int dtype_in) {
  if (!q || !k || !v || !log_a || !b) return fail(GDN2_ERR_INVALID_ARG, "q, k, v, log_a and b must be non-NULL");
  if (!w && !(flags & GDN2_TIED_GATES)) return fail(GDN2_ERR_INVALID_ARG, "w is NULL without GDN2_TIED_GATES");
  const uintptr_t elem = dtype_in == GDN2_BF16 ? 2 : 4;
  const void *dense[3] = {q, k, v};
  for (const void *p : dense)
    if (!aligned16(p)) return fail(GDN2_ERR_INVALID_ARG, "input pointer %p is not 16-byte aligned", p);
  const bool sd = (flags & GDN2_SCALAR_DECAY) != 0, sg = (flags & GDN2_SCALAR_GATES) != 0;
  const void *gates[3] = {log_a, b, w};
  const bool scalar[3] = {sd, sg, sg};
  for (int i = 0; i < 3; ++i) {
    const uintptr_t a = reinterpret_cast<uintptr_t>(gates[i]);
    if (gates[i] && (scalar[i] ? (a % elem) != 0 : (a & 15u) != 0))
      return fail(GDN2_ERR_INVALID_ARG, "gate pointer %p is misaligned", gates[i]);
  }
  return GDN2_OK;
}

}  // namespace

namespace gdn2 {
int set_last_error(int code, const char *message) { return fail(code, "%s", message); }

namespace {
std::atomic<int> g_debug_site{0};
std::atomic<unsigned long long> g_debug_ns{0};
}  // namespace

bool take_debug_timeout(int site, uint64_t *wait_ns) {
  int armed = site;
  if (g_debug_site.load(std::memory_order_relaxed) != site ||
      !g_debug_site.compare_exchange_strong(armed, 0))
    return false;
  *wait_ns = g_debug_ns.load();
  return true;
}
}  // namespace gdn2

extern "C" {

int gdn2_version(void) { return 100; }

int gdn2_debug_timeout_once(int32_t site, uint64_t wait_ns) {
  g_err[0] = '\0';
  if (site != GDN2_DEBUG_CHUNK && site != GDN2_DEBUG_DECODE && site != GDN2_DEBUG_BWD)
    return fail(GDN2_ERR_INVALID_ARG, "unknown debug site %d", site);
  if (wait_ns < 1000ull || wait_ns > 10000000000ull)
    return fail(GDN2_ERR_INVALID_ARG, "wait_ns must lie in [1000, 1e10] (got %llu)", (unsigned long long)wait_ns);
  gdn2::g_debug_ns.store(wait_ns);
  gdn2::g_debug_site.store(site);
  return GDN2_OK;
}

const char *gdn2_last_error(void) { return g_err; }

size_t gdn2_chunk_fwd_workspace_size(const gdn2_dims *dims) {
  if (!dims || dims->n_seqs < 1 || dims->n_heads < 1) return 0;
  const size_t units = (size_t)dims->n_seqs * (size_t)dims->n_heads;
  return kWsHeader + ((units * sizeof(int32_t) + 255) / 256) * 256;
}

static int chunk_fwd_impl(const void *q, const void *k, const void *v, const void *log_a, const void *b,
                          const void *w, const float *S0, const int32_t *cu_seqlens, const int32_t *cu_seqlens_host,
                          void *o, float *S_T, const gdn2_dims *dims, void *workspace, size_t workspace_bytes,
                          gdn2_stream_t stream, bool reset_status, const int32_t *seg_bounds = nullptr);

int gdn2_chunk_fwd(const void *q, const void *k, const void *v, const void *log_a, const void *b, const void *w,
                   const float *S0, const int32_t *cu_seqlens, const int32_t *cu_seqlens_host, void *o, float *S_T,
                   const gdn2_dims *dims, void *workspace, size_t workspace_bytes, gdn2_stream_t stream) {
  return chunk_fwd_impl(q, k, v, log_a, b, w, S0, cu_seqlens, cu_seqlens_host, o, S_T, dims, workspace,
                        workspace_bytes, stream, true);
}

// seg_bounds (internal): [2 * dims->n_seqs] device (first, end) token of every unit sequence,
// which may leave gaps; dims->seq_len is then the packed token count the tensors span.
static int chunk_fwd_impl(const void *q, const void *k, const void *v, const void *log_a, const void *b,
                          const void *w, const float *S0, const int32_t *cu_seqlens, const int32_t *cu_seqlens_host,
                          void *o, float *S_T, const gdn2_dims *dims, void *workspace, size_t workspace_bytes,
                          gdn2_stream_t stream, bool reset_status, const int32_t *seg_bounds) {
  g_err[0] = '\0';
  int rc = check_dims(dims);
  if (rc) return rc;
  rc = check_inputs(q, k, v, log_a, b, w, dims->flags, dims->dtype_in);
  if (rc) return rc;
  if (!o || !aligned16(o)) return fail(GDN2_ERR_INVALID_ARG, "o must be non-NULL and 16-byte aligned");
  if ((S0 && !aligned16(S0)) || (S_T && !aligned16(S_T)))
    return fail(GDN2_ERR_INVALID_ARG, "S0 / S_T must be 16-byte aligned");
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return fail(GDN2_ERR_WORKSPACE, "workspace must be non-NULL and 256-byte aligned");
  const size_t need = gdn2_chunk_fwd_workspace_size(dims);
  if (workspace_bytes < need)
    return fail(GDN2_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", workspace_bytes, need);

  const int64_t t_total =
      (cu_seqlens || seg_bounds) ? (int64_t)dims->seq_len : (int64_t)dims->n_seqs * dims->seq_len;
  if (cu_seqlens_host) {
    if (!cu_seqlens) return fail(GDN2_ERR_INVALID_ARG, "cu_seqlens_host given without cu_seqlens");
    if (cu_seqlens_host[0] != 0 || cu_seqlens_host[dims->n_seqs] != t_total)
      return fail(GDN2_ERR_INVALID_ARG, "cu_seqlens_host must start at 0 and end at seq_len (= T_tot)");
    for (int n = 0; n < dims->n_seqs; ++n)
      if (cu_seqlens_host[n + 1] < cu_seqlens_host[n])
        return fail(GDN2_ERR_INVALID_ARG, "cu_seqlens_host is not non-decreasing at %d", n);
  }

  gdn2::ChunkProblem p;
  memset(&p, 0, sizeof(p));
  p.q = q; p.k = k; p.v = v; p.log_a = log_a; p.b = b; p.w = w;
  p.S0 = S0; p.cu_seqlens = cu_seqlens; p.o = o; p.S_T = S_T;
  p.n_seqs = dims->n_seqs; p.seq_len = dims->seq_len; p.n_heads = dims->n_heads;
  p.d_k = dims->d_k; p.d_v = dims->d_v; p.chunk = dims->chunk;
  p.dtype_in = dims->dtype_in; p.dtype_out = dims->dtype_out; p.flags = dims->flags;
  p.t_total = t_total;
  p.status = static_cast<int32_t *>(workspace);
  p.schedule = nullptr;
  p.seg_bounds = seg_bounds;

  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const bool tc = dims->d_k == 128 && dims->d_v == 128 && dims->chunk == 64 && dims->dtype_in == GDN2_BF16;
  const bool simt = dims->d_k <= 64 && dims->d_v <= 64 &&
                    (dims->chunk == 16 || dims->chunk == 32 || dims->chunk == 64);
  if (seg_bounds && !tc) return fail(GDN2_ERR_UNSUPPORTED, "segment bounds need the tensor-core path");
  if (!tc && !simt)
    return fail(GDN2_ERR_UNSUPPORTED,
                "no kernel for d_k=%d d_v=%d chunk=%d dtype_in=%d (supported: 128/128/64 bf16, or d<=64 with chunk "
                "16/32/64)",
                dims->d_k, dims->d_v, dims->chunk, dims->dtype_in);

  // header: [0] status word (kept across the passes of one split forward), [1] unit counter
  cudaError_t e = reset_status ? cudaMemsetAsync(workspace, 0, kWsHeader, s)
                               : cudaMemsetAsync(static_cast<char *>(workspace) + 4, 0, kWsHeader - 4, s);
  if (e != cudaSuccess) return fail(GDN2_ERR_CUDA, "cudaMemsetAsync(workspace): %s", cudaGetErrorString(e));
  if (tc && cu_seqlens && dims->n_seqs <= kMaxSortedSeqs) {
    int32_t *sched = reinterpret_cast<int32_t *>(static_cast<char *>(workspace) + kWsHeader);
    schedule_kernel<<<1, 1024, 0, s>>>(cu_seqlens, dims->n_seqs, dims->n_heads, sched);
    e = cudaGetLastError();
    if (e != cudaSuccess) return fail(GDN2_ERR_CUDA, "schedule launch: %s", cudaGetErrorString(e));
    p.schedule = sched;
  }
  if (tc) {
    const char *why = "";
    e = gdn2::launch_chunk_tc(p, s, &why);
    if (e == cudaErrorNotSupported) return fail(GDN2_ERR_UNSUPPORTED, "%s", why);
    if (e != cudaSuccess) return fail(GDN2_ERR_CUDA, "chunk_tc launch: %s (%s)", cudaGetErrorString(e), why);
  } else {
    e = gdn2::launch_chunk_simt(p, s);
    if (e != cudaSuccess) return fail(GDN2_ERR_CUDA, "chunk_simt launch: %s", cudaGetErrorString(e));
  }
  return GDN2_OK;
}

// gdn2_chunk_bwd workspace: [0, 256) header ([0] status, [1] forward unit counter, [2] backward
// unit counter), the unit schedule, the per-sequence checkpoint offsets, the final states
// (fp32), the checkpoints (per chunk and (sequence, head) the bf16 S_r and T tile images).
struct ChunkBwdLayout {
  size_t off_sched, off_ckoff, off_fin, off_ckpt, off_pro, total;
};
static ChunkBwdLayout chunk_bwd_layout(const gdn2_dims *dims, bool packed) {
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  const int64_t t_total = packed ? (int64_t)dims->seq_len : (int64_t)dims->n_seqs * dims->seq_len;
  const size_t units = (size_t)dims->n_seqs * dims->n_heads;
  ChunkBwdLayout L;
  L.off_sched = kWsHeader;
  L.off_ckoff = L.off_sched + up(units * sizeof(int32_t));
  L.off_fin = L.off_ckoff + up(((size_t)dims->n_seqs + 1) * sizeof(int64_t));
  L.off_ckpt = L.off_fin + units * 128 * 128 * sizeof(float);
  const size_t slots = gdn2::bwd_tc_ckpt_slots(dims->n_seqs, t_total, dims->n_heads, packed, dims->seq_len);
  L.total = L.off_ckpt + slots * gdn2::kBwdCkptSlotBytes;
  // with the fused prologue: activated bf16 copies of q, k (and of log_a, b, w: per channel or
  // per token) and the fp32 inverse norms of q and k per (token, head)
  L.off_pro = up(L.total);
  if (dims->flags & GDN2_FUSED_PROLOGUE) {
    const size_t rows = (size_t)t_total * dims->n_heads;
    const size_t gd = (dims->flags & GDN2_SCALAR_DECAY) ? 1 : 128, gg = (dims->flags & GDN2_SCALAR_GATES) ? 1 : 128;
    L.total = L.off_pro + up(rows * 128 * 2) * 2 + up(rows * gd * 2) + up(rows * gg * 2) * 2 + up(rows * 2 * sizeof(float));
  }
  return L;
}

static const char *chunk_bwd_unsupported(const gdn2_dims *d) {
  if (d->d_k != 128 || d->d_v != 128) return "gdn2_chunk_bwd needs d_k = d_v = 128";
  if (d->dtype_in != GDN2_BF16) return "gdn2_chunk_bwd needs bf16 inputs";
  return nullptr;
}

size_t gdn2_chunk_bwd_workspace_size(const gdn2_dims *dims, int32_t packed) {
  if (!dims || dims->n_seqs < 1 || dims->n_heads < 1 || dims->seq_len < 0) return 0;
  if (chunk_bwd_unsupported(dims)) return 0;
  return chunk_bwd_layout(dims, packed != 0).total;
}

int gdn2_chunk_bwd(const void *q, const void *k, const void *v, const void *log_a, const void *b, const void *w,
                   const float *S0, const int32_t *cu_seqlens, const void *dO, const float *dS_T, void *dq, void *dk,
                   void *dv, void *dlog_a, void *db, void *dw, float *dS0, const gdn2_dims *dims, void *workspace,
                   size_t workspace_bytes, gdn2_stream_t stream) {
  g_err[0] = '\0';
  int rc = check_dims(dims);
  if (rc) return rc;
  rc = check_inputs(q, k, v, log_a, b, w, dims->flags, dims->dtype_in);
  if (rc) return rc;
  if (const char *why = chunk_bwd_unsupported(dims)) return fail(GDN2_ERR_UNSUPPORTED, "%s", why);
  const bool tied = (dims->flags & GDN2_TIED_GATES) != 0;
  if (!dO || !dq || !dk || !dv || !dlog_a || !db || (!dw && !tied))
    return fail(GDN2_ERR_INVALID_ARG, "dO, dq, dk, dv, dlog_a, db (and dw without GDN2_TIED_GATES) must be non-NULL");
  if ((S0 && !aligned16(S0)) || (dS_T && !aligned16(dS_T)) || (dS0 && !aligned16(dS0)))
    return fail(GDN2_ERR_INVALID_ARG, "S0, dS_T and dS0 must be 16-byte aligned");
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return fail(GDN2_ERR_WORKSPACE, "workspace must be non-NULL and 256-byte aligned");
  if ((dims->flags & GDN2_FUSED_PROLOGUE) &&
      (!aligned16(dq) || !aligned16(dk) || !aligned16(dlog_a) || !aligned16(db) || (dw && !aligned16(dw))))
    return fail(GDN2_ERR_INVALID_ARG, "with GDN2_FUSED_PROLOGUE the gradients must be 16-byte aligned");
  const bool packed = cu_seqlens != nullptr;
  const ChunkBwdLayout lay = chunk_bwd_layout(dims, packed);
  if (workspace_bytes < lay.total)
    return fail(GDN2_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", workspace_bytes, lay.total);
  const int64_t t_total = packed ? (int64_t)dims->seq_len : (int64_t)dims->n_seqs * dims->seq_len;
  if (t_total >= (int64_t)1 << 31) return fail(GDN2_ERR_UNSUPPORTED, "gdn2_chunk_bwd needs T_tot < 2^31");

  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  char *ws = static_cast<char *>(workspace);
  int32_t *status = reinterpret_cast<int32_t *>(ws);
  cudaError_t e = cudaMemsetAsync(ws, 0, kWsHeader, s);
  if (e != cudaSuccess) return fail(GDN2_ERR_CUDA, "cudaMemsetAsync(workspace): %s", cudaGetErrorString(e));
  const int32_t *sched = nullptr;
  int64_t *ckoff = nullptr;
  if (packed) {
    if (dims->n_seqs <= kMaxSortedSeqs) {
      int32_t *sp = reinterpret_cast<int32_t *>(ws + lay.off_sched);
      schedule_kernel<<<1, 1024, 0, s>>>(cu_seqlens, dims->n_seqs, dims->n_heads, sp);
      e = cudaGetLastError();
      if (e != cudaSuccess) return fail(GDN2_ERR_CUDA, "schedule launch: %s", cudaGetErrorString(e));
      sched = sp;
    }
    ckoff = reinterpret_cast<int64_t *>(ws + lay.off_ckoff);
    e = gdn2::launch_ckpt_offsets(cu_seqlens, dims->n_seqs, ckoff, s);
    if (e != cudaSuccess) return fail(GDN2_ERR_CUDA, "checkpoint offsets launch: %s", cudaGetErrorString(e));
  }
  void *ckpt = ws + lay.off_ckpt;
  float *S_fin = reinterpret_cast<float *>(ws + lay.off_fin);
  // raw inputs as given; with the fused prologue the passes below run on activated copies
  const void *aq = q, *ak = k, *ala = log_a, *ab = b, *aw = w;
  uint32_t aflags = dims->flags;
  gdn2::PrologueCopiesBf16 pc{};
  gdn2::BwdProblem raw;
  memset(&raw, 0, sizeof(raw));
  raw.q = q; raw.k = k; raw.log_a = log_a; raw.b = b; raw.w = tied ? nullptr : w;
  raw.dq = dq; raw.dk = dk; raw.dlog_a = dlog_a; raw.db = db; raw.dw = tied ? nullptr : dw;
  raw.n_heads = dims->n_heads; raw.t_total = t_total; raw.dtype_out = dims->dtype_out; raw.flags = dims->flags;
  if (dims->flags & GDN2_FUSED_PROLOGUE) {
    auto up = [](size_t x) { return (x + 255) / 256 * 256; };
    const size_t rows = (size_t)t_total * dims->n_heads;
    const size_t gd = (dims->flags & GDN2_SCALAR_DECAY) ? 1 : 128, gg = (dims->flags & GDN2_SCALAR_GATES) ? 1 : 128;
    char *base = ws + lay.off_pro;
    pc.q = reinterpret_cast<__nv_bfloat16 *>(base);
    base += up(rows * 256);
    pc.k = reinterpret_cast<__nv_bfloat16 *>(base);
    base += up(rows * 256);
    pc.log_a = reinterpret_cast<__nv_bfloat16 *>(base);
    base += up(rows * gd * 2);
    pc.b = reinterpret_cast<__nv_bfloat16 *>(base);
    base += up(rows * gg * 2);
    pc.w = reinterpret_cast<__nv_bfloat16 *>(base);
    base += up(rows * gg * 2);
    pc.inv_norm = reinterpret_cast<float *>(base);
    e = gdn2::launch_prolog_act(raw, pc, s);
    if (e != cudaSuccess) return fail(GDN2_ERR_CUDA, "prologue launch: %s", cudaGetErrorString(e));
    aq = pc.q; ak = pc.k; ala = pc.log_a; ab = pc.b; aw = tied ? nullptr : pc.w;
    aflags &= ~(uint32_t)GDN2_FUSED_PROLOGUE;
  }

  // the forward, writing every chunk's S_r tile and the final states instead of o
  gdn2::ChunkProblem f;
  memset(&f, 0, sizeof(f));
  f.q = aq; f.k = ak; f.v = v; f.log_a = ala; f.b = ab; f.w = aw;
  f.S0 = S0; f.cu_seqlens = cu_seqlens; f.o = nullptr; f.S_T = S_fin;
  f.n_seqs = dims->n_seqs; f.seq_len = dims->seq_len; f.n_heads = dims->n_heads;
  f.d_k = 128; f.d_v = 128; f.chunk = 64;
  f.dtype_in = GDN2_BF16; f.dtype_out = dims->dtype_out; f.flags = aflags;
  f.t_total = t_total;
  f.status = status;
  f.schedule = sched;
  f.ckpt = ckpt;
  f.ckpt_off = ckoff;
  const char *why = "";
  e = gdn2::launch_chunk_tc(f, s, &why);
  if (e == cudaErrorNotSupported) return fail(GDN2_ERR_UNSUPPORTED, "%s", why);
  if (e != cudaSuccess) return fail(GDN2_ERR_CUDA, "chunk_tc launch: %s (%s)", cudaGetErrorString(e), why);

  gdn2::BwdProblem p;
  memset(&p, 0, sizeof(p));
  p.q = aq; p.k = ak; p.v = v; p.log_a = ala; p.b = ab; p.w = tied ? nullptr : aw;
  p.S0 = S0; p.cu_seqlens = cu_seqlens; p.dO = dO; p.dS_T = dS_T;
  p.dq = dq; p.dk = dk; p.dv = dv; p.dlog_a = dlog_a; p.db = db; p.dw = tied ? nullptr : dw; p.dS0 = dS0;
  p.n_seqs = dims->n_seqs; p.seq_len = dims->seq_len; p.n_heads = dims->n_heads;
  p.d_k = 128; p.d_v = 128; p.t_total = t_total;
  p.dtype_in = GDN2_BF16; p.dtype_out = dims->dtype_out; p.flags = aflags;
  e = gdn2::launch_bwd_tc(p, ckpt, S_fin, ckoff, sched, status, status + 2, s);
  if (e != cudaSuccess) return fail(GDN2_ERR_CUDA, "bwd_tc launch: %s", cudaGetErrorString(e));
  if (dims->flags & GDN2_FUSED_PROLOGUE) {  // gradients of the raw inputs
    e = gdn2::launch_prolog_chain(raw, pc.inv_norm, s);
    if (e != cudaSuccess) return fail(GDN2_ERR_CUDA, "prologue chain-rule launch: %s", cudaGetErrorString(e));
  }
  return GDN2_OK;
}

size_t gdn2_bwd_workspace_size(const gdn2_dims *dims, int32_t packed) {
  if (!dims || dims->n_seqs < 1 || dims->n_heads < 1 || dims->seq_len < 0 || dims->d_k < 1 || dims->d_v < 1)
    return 0;
  if (dims->d_v != 16 && dims->d_v != 32 && dims->d_v != 64 && dims->d_v != 128) return 0;
  const int64_t t_total = packed ? (int64_t)dims->seq_len : (int64_t)dims->n_seqs * dims->seq_len;
  return gdn2::bwd_workspace_bytes(dims->n_seqs, t_total, dims->n_heads, dims->d_k, dims->d_v, dims->flags);
}

int gdn2_bwd(const void *q, const void *k, const void *v, const void *log_a, const void *b, const void *w,
             const float *S0, const int32_t *cu_seqlens, const void *dO, const float *dS_T, void *dq, void *dk,
             void *dv, void *dlog_a, void *db, void *dw, float *dS0, const gdn2_dims *dims, void *workspace,
             size_t workspace_bytes, gdn2_stream_t stream) {
  g_err[0] = '\0';
  int rc = check_dims(dims);
  if (rc) return rc;
  rc = check_inputs(q, k, v, log_a, b, w, dims->flags, dims->dtype_in);
  if (rc) return rc;
  if (dims->d_k > 128 || (dims->d_v != 16 && dims->d_v != 32 && dims->d_v != 64 && dims->d_v != 128))
    return fail(GDN2_ERR_UNSUPPORTED, "gdn2_bwd supports d_k <= 128 and d_v in {16, 32, 64, 128} (got %d, %d)",
                dims->d_k, dims->d_v);
  const bool tied = (dims->flags & GDN2_TIED_GATES) != 0;
  if (!dO || !dq || !dk || !dv || !dlog_a || !db || (!dw && !tied))
    return fail(GDN2_ERR_INVALID_ARG, "dO, dq, dk, dv, dlog_a, db (and dw without GDN2_TIED_GATES) must be non-NULL");
  if ((S0 && !aligned16(S0)) || (dS_T && !aligned16(dS_T)) || (dS0 && !aligned16(dS0)))
    return fail(GDN2_ERR_INVALID_ARG, "S0, dS_T and dS0 must be 16-byte aligned");
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return fail(GDN2_ERR_WORKSPACE, "workspace must be non-NULL and 256-byte aligned");
  const int64_t t_total = cu_seqlens ? (int64_t)dims->seq_len : (int64_t)dims->n_seqs * dims->seq_len;
  const size_t need = gdn2::bwd_workspace_bytes(dims->n_seqs, t_total, dims->n_heads, dims->d_k, dims->d_v,
                                                dims->flags);
  if (workspace_bytes < need)
    return fail(GDN2_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", workspace_bytes, need);
  gdn2::BwdProblem p;
  memset(&p, 0, sizeof(p));
  p.q = q; p.k = k; p.v = v; p.log_a = log_a; p.b = b; p.w = w;
  p.S0 = S0; p.cu_seqlens = cu_seqlens; p.dO = dO; p.dS_T = dS_T;
  p.dq = dq; p.dk = dk; p.dv = dv; p.dlog_a = dlog_a; p.db = db; p.dw = tied ? nullptr : dw; p.dS0 = dS0;
  p.n_seqs = dims->n_seqs; p.seq_len = dims->seq_len; p.n_heads = dims->n_heads;
  p.d_k = dims->d_k; p.d_v = dims->d_v; p.t_total = t_total;
  p.dtype_in = dims->dtype_in; p.dtype_out = dims->dtype_out; p.flags = dims->flags;
  gdn2::bwd_carve(p, workspace);
  cudaError_t e = gdn2::launch_bwd(p, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(GDN2_ERR_CUDA, "bwd launch: %s", cudaGetErrorString(e));
  return GDN2_OK;
}

int gdn2_decode_status(gdn2_stream_t stream) {
  g_err[0] = '\0';
  int32_t st = 0;
  const int e = gdn2::read_decode_status(reinterpret_cast<cudaStream_t>(stream), &st);
  if (e != 0) return fail(GDN2_ERR_CUDA, "reading the decode status: %s", cudaGetErrorString((cudaError_t)e));
  if (st == gdn2::kStatusTimeout) return fail(GDN2_ERR_TIMEOUT, "a bounded wait of the decode kernel timed out");
  if (st != 0) return fail(GDN2_ERR_CUDA, "unknown device status %d", st);
  return GDN2_OK;
}

static gdn2::SplitPlan split_plan_for(const gdn2_dims *dims, int32_t n_split) {
  const gdn2::SplitPlan p0 = gdn2::split_plan(dims->n_seqs, dims->seq_len, dims->n_heads, n_split, dims->dtype_in,
                                              dims->dtype_out, 0);
  gdn2_dims inner = *dims;
  inner.n_seqs = p0.n_segs;
  inner.seq_len = dims->n_seqs * dims->seq_len;
  return gdn2::split_plan(dims->n_seqs, dims->seq_len, dims->n_heads, n_split, dims->dtype_in, dims->dtype_out,
                          gdn2_chunk_fwd_workspace_size(&inner));
}

size_t gdn2_chunk_fwd_split_workspace_size(const gdn2_dims *dims, int32_t n_split) {
  if (!dims || dims->n_seqs < 1 || dims->n_heads < 1 || dims->seq_len < 0 || n_split < 1) return 0;
  return split_plan_for(dims, n_split).total;
}

int gdn2_chunk_fwd_split(const void *q, const void *k, const void *v, const void *log_a, const void *b,
                         const void *w, const float *S0, void *o, float *S_T, const gdn2_dims *dims, int32_t n_split,
                         void *workspace, size_t workspace_bytes, gdn2_stream_t stream) {
  g_err[0] = '\0';
  int rc = check_dims(dims);
  if (rc) return rc;
  if (n_split < 1) return fail(GDN2_ERR_INVALID_ARG, "n_split must be >= 1 (got %d)", n_split);
  if (dims->d_k != 128 || dims->d_v != 128 || dims->chunk != 64 || dims->dtype_in != GDN2_BF16)
    return fail(GDN2_ERR_UNSUPPORTED, "gdn2_chunk_fwd_split needs d_k = d_v = 128, chunk 64 and bf16 inputs");
  if ((int64_t)dims->n_seqs * dims->seq_len >= ((int64_t)1 << 31))
    return fail(GDN2_ERR_UNSUPPORTED, "gdn2_chunk_fwd_split needs fewer than 2^31 tokens");
  rc = check_inputs(q, k, v, log_a, b, w, dims->flags, dims->dtype_in);
  if (rc) return rc;
  if (!o || !aligned16(o)) return fail(GDN2_ERR_INVALID_ARG, "o must be non-NULL and 16-byte aligned");
  if ((S0 && !aligned16(S0)) || (S_T && !aligned16(S_T)))
    return fail(GDN2_ERR_INVALID_ARG, "S0 / S_T must be 16-byte aligned");
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return fail(GDN2_ERR_WORKSPACE, "workspace must be non-NULL and 256-byte aligned");
  const size_t need = gdn2_chunk_fwd_split_workspace_size(dims, n_split);
  if (workspace_bytes < need)
    return fail(GDN2_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", workspace_bytes, need);
  const int N = dims->n_seqs, T = dims->seq_len, H = dims->n_heads;
  if ((int64_t)N * T == 0) {  // nothing to run: S_T = S0
    cudaStream_t s0 = reinterpret_cast<cudaStream_t>(stream);
    if (!S_T) return GDN2_OK;
    const size_t bytes = (size_t)N * H * 128 * 128 * sizeof(float);
    const cudaError_t e = S0 ? cudaMemcpyAsync(S_T, S0, bytes, cudaMemcpyDeviceToDevice, s0)
                             : cudaMemsetAsync(S_T, 0, bytes, s0);
    return e == cudaSuccess ? GDN2_OK : fail(GDN2_ERR_CUDA, "S_T for empty sequences: %s", cudaGetErrorString(e));
  }
  char *ws = static_cast<char *>(workspace);
  gdn2::SplitArgs a;
  a.plan = split_plan_for(dims, n_split);
  a.N = N; a.T = T; a.H = H; a.dtype_out = dims->dtype_out;
  a.cu = reinterpret_cast<int32_t *>(ws + a.plan.off_cu);
  a.starts = reinterpret_cast<float *>(ws + a.plan.off_start);
  a.F = reinterpret_cast<float *>(ws + a.plan.off_F);
  a.G = reinterpret_cast<float *>(ws + a.plan.off_G);
  a.S_T = S_T;
  a.S0 = S0;
  a.o = o;
  void *zero_v = ws + a.plan.off_zero_v;
  void *o2 = ws + a.plan.off_o2;
  a.o2 = o2;
  void *inner_ws = ws + a.plan.off_inner;
  const size_t inner_bytes = a.plan.off_cu - a.plan.off_inner;
  if (a.plan.n_per_seq == 1)  // one segment per sequence: the plain forward
    return chunk_fwd_impl(q, k, v, log_a, b, w, S0, nullptr, nullptr, o, S_T, dims, inner_ws, inner_bytes, stream,
                          true);
  gdn2_dims inner = *dims;
  inner.n_seqs = a.plan.n_segs;
  inner.seq_len = N * T;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const size_t vbytes = (size_t)N * T * H * 128 * (dims->dtype_in == GDN2_BF16 ? 2 : 4);
  cudaError_t e = cudaMemsetAsync(zero_v, 0, vbytes, s);
  if (e == cudaSuccess) e = gdn2::launch_split_helpers(0, a, s);
  if (e == cudaSuccess) e = gdn2::launch_split_helpers(1, a, s);
  if (e != cudaSuccess) return fail(GDN2_ERR_CUDA, "split setup: %s", cudaGetErrorString(e));
  // pass 1: zero starts (S0 in each sequence's first segment): o and the end states G
  rc = chunk_fwd_impl(q, k, v, log_a, b, w, a.starts, a.cu, nullptr, o, a.G, &inner, inner_ws, inner_bytes, stream,
                      true);
  if (rc) return rc;
  // pass 2: identity starts, v = 0: the transitions F
  e = gdn2::launch_split_helpers(2, a, s);
  if (e != cudaSuccess) return fail(GDN2_ERR_CUDA, "split identities: %s", cudaGetErrorString(e));
  rc = chunk_fwd_impl(q, k, zero_v, log_a, b, w, a.starts, a.cu, nullptr, o2, a.F, &inner, inner_ws, inner_bytes,
                      stream, false);
  if (rc) return rc;
  // combine: true start states; S_T
  e = gdn2::launch_split_helpers(3, a, s);
  if (e != cudaSuccess) return fail(GDN2_ERR_CUDA, "split combine: %s", cudaGetErrorString(e));
  // pass 3: the outputs' part that comes from the start states, added to o
  rc = chunk_fwd_impl(q, k, zero_v, log_a, b, w, a.starts, a.cu, nullptr, o2, nullptr, &inner, inner_ws, inner_bytes,
                      stream, false);
  if (rc) return rc;
  e = gdn2::launch_split_helpers(4, a, s);
  if (e != cudaSuccess) return fail(GDN2_ERR_CUDA, "split add: %s", cudaGetErrorString(e));
  return GDN2_OK;
}

static size_t up256(size_t x) { return (x + 255) / 256 * 256; }

// ---------------------------------------------------------------- packed varlen split
// Plan of gdn2_chunk_fwd_split_varlen from the host copy of cu_seqlens.  tau = the balanced
// share of 64-token chunks per SM; a sequence of more than 3 tau chunks is cut into segments of
// about tau chunks (whole chunks), raised until all segment units fit in the SMs when that is
// possible.  Passes (one chunk-kernel launch each): 2 = segments of split sequences from the
// identity (their E = F + G); 1 = every segment from 0 (unsplit sequences from S0): G and the
// provisional o; combine; 3 = split segments that start from a non-zero state, re-run from it:
// the final o.
struct VarlenPlan {
  int N = 0, H = 0, NS = 0, N2 = 0, N3 = 0;
  bool any_split = false;
  std::vector<int32_t> ints;  // cu1 [NS + 1] | src1 [NS] | src2 [N2] | b2 [2 N2] | b3 [2 N3] | info [4 N]
  size_t i_cu1 = 0, i_src1 = 0, i_src2 = 0, i_b2 = 0, i_b3 = 0, i_info = 0;
  size_t off_ints = 0, off_G = 0, off_E = 0, off_S3 = 0, total = 0, inner = 0;
};

static VarlenPlan varlen_plan(const gdn2_dims *d, const int32_t *cu, int n_sm, bool has_S0) {
  VarlenPlan P;
  const int N = d->n_seqs, H = d->n_heads;
  P.N = N;
  P.H = H;
  std::vector<int64_t> chunks(N);
  int64_t total = 0, cmax = 0;
  for (int n = 0; n < N; ++n) {
    chunks[n] = ((int64_t)cu[n + 1] - cu[n] + 63) / 64;
    total += chunks[n];
    cmax = chunks[n] > cmax ? chunks[n] : cmax;
  }
  int64_t tau = (total * H + n_sm - 1) / (n_sm > 0 ? n_sm : 1);
  if (tau < 1) tau = 1;
  std::vector<int> m(N, 1);
  for (int iter = 0; iter < 16; ++iter) {
    int64_t units = 0;
    for (int n = 0; n < N; ++n) {
      m[n] = chunks[n] > 3 * tau ? (int)((chunks[n] + tau - 1) / tau) : 1;
      units += (int64_t)m[n] * H;
    }
    if (units <= n_sm || 3 * tau >= cmax) break;
    tau = (tau * units + n_sm - 1) / n_sm;  // fewer, longer segments
  }
  std::vector<int32_t> cu1{0}, src1, src2, b2, b3, info;
  for (int n = 0; n < N; ++n) {
    const int32_t bos = cu[n], eos = cu[n + 1];
    const int first1 = (int)src1.size(), first2 = (int)src2.size(), first3 = (int)b3.size() / 2;
    int segs = 1;
    if (m[n] > 1) {
      const int64_t per = (chunks[n] + m[n] - 1) / m[n];  // chunks per segment
      segs = 0;
      for (int64_t a = bos; a < eos; a += per * 64) {
        const int32_t e = (int32_t)(a + per * 64 < eos ? a + per * 64 : eos);
        cu1.push_back(e);
        src1.push_back(-1);  // from 0
        src2.push_back(-2);  // from the identity
        b2.push_back((int32_t)a);
        b2.push_back(e);
        if (segs > 0 || has_S0) {
          b3.push_back((int32_t)a);
          b3.push_back(e);
        }
        ++segs;
      }
      P.any_split = true;
    } else {
      cu1.push_back(eos);
      src1.push_back(has_S0 ? n : -1);
    }
    info.push_back(segs);
    info.push_back(first1);
    info.push_back(first2);
    info.push_back(first3);
  }
  P.NS = (int)src1.size();
  P.N2 = (int)src2.size();
  P.N3 = (int)b3.size() / 2;
  auto put = [&](const std::vector<int32_t> &v) {
    const size_t at = P.ints.size();
    P.ints.insert(P.ints.end(), v.begin(), v.end());
    return at;
  };
  P.i_cu1 = put(cu1);
  P.i_src1 = put(src1);
  P.i_src2 = put(src2);
  P.i_b2 = put(b2);
  P.i_b3 = put(b3);
  P.i_info = put(info);
  // workspace: the passes' own workspace (sized for the largest pass) | plan | G | E | starts3
  gdn2_dims inner = *d;
  inner.n_seqs = P.NS > 0 ? P.NS : 1;
  const size_t state = (size_t)H * 128 * 128 * sizeof(float);
  P.inner = up256(gdn2_chunk_fwd_workspace_size(&inner));
  P.off_ints = P.inner;
  P.off_G = P.off_ints + up256(P.ints.size() * sizeof(int32_t));
  P.off_E = P.off_G + up256((size_t)P.NS * state);
  P.off_S3 = P.off_E + up256((size_t)P.N2 * state);
  P.total = P.off_S3 + up256((size_t)P.N3 * state);
  return P;
}

static int sm_count() {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return 148;
  return sms;
}

static int check_varlen_cu(const gdn2_dims *dims, const int32_t *cu_host) {
  if (!cu_host) return fail(GDN2_ERR_INVALID_ARG, "cu_seqlens_host is required (the plan is made on the host)");
  if (cu_host[0] != 0 || cu_host[dims->n_seqs] != dims->seq_len)
    return fail(GDN2_ERR_INVALID_ARG, "cu_seqlens_host must start at 0 and end at seq_len (= T_tot)");
  for (int n = 0; n < dims->n_seqs; ++n)
    if (cu_host[n + 1] < cu_host[n]) return fail(GDN2_ERR_INVALID_ARG, "cu_seqlens_host is not non-decreasing at %d", n);
  return GDN2_OK;
}

size_t gdn2_chunk_fwd_split_varlen_workspace_size(const gdn2_dims *dims, const int32_t *cu_seqlens_host) {
  if (!dims || dims->n_seqs < 1 || dims->n_heads < 1 || dims->seq_len < 0 || !cu_seqlens_host) return 0;
  if (cu_seqlens_host[0] != 0 || cu_seqlens_host[dims->n_seqs] != dims->seq_len) return 0;
  for (int n = 0; n < dims->n_seqs; ++n)
    if (cu_seqlens_host[n + 1] < cu_seqlens_host[n]) return 0;
  return varlen_plan(dims, cu_seqlens_host, sm_count(), true).total;  // S0 present: the larger plan
}

int gdn2_chunk_fwd_split_varlen(const void *q, const void *k, const void *v, const void *log_a, const void *b,
                                const void *w, const float *S0, const int32_t *cu_seqlens,
                                const int32_t *cu_seqlens_host, void *o, float *S_T, const gdn2_dims *dims,
                                void *workspace, size_t workspace_bytes, gdn2_stream_t stream) {
  g_err[0] = '\0';
  int rc = check_dims(dims);
  if (rc) return rc;
  if (dims->d_k != 128 || dims->d_v != 128 || dims->chunk != 64 || dims->dtype_in != GDN2_BF16)
    return fail(GDN2_ERR_UNSUPPORTED, "gdn2_chunk_fwd_split_varlen needs d_k = d_v = 128, chunk 64 and bf16 inputs");
  if (!cu_seqlens) return fail(GDN2_ERR_INVALID_ARG, "cu_seqlens must be non-NULL");
  rc = check_varlen_cu(dims, cu_seqlens_host);
  if (rc) return rc;
  rc = check_inputs(q, k, v, log_a, b, w, dims->flags, dims->dtype_in);
  if (rc) return rc;
  if (!o || !aligned16(o)) return fail(GDN2_ERR_INVALID_ARG, "o must be non-NULL and 16-byte aligned");
  if ((S0 && !aligned16(S0)) || (S_T && !aligned16(S_T)))
    return fail(GDN2_ERR_INVALID_ARG, "S0 / S_T must be 16-byte aligned");
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return fail(GDN2_ERR_WORKSPACE, "workspace must be non-NULL and 256-byte aligned");
  const size_t need = gdn2_chunk_fwd_split_varlen_workspace_size(dims, cu_seqlens_host);
  if (workspace_bytes < need)
    return fail(GDN2_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", workspace_bytes, need);
  const VarlenPlan P = varlen_plan(dims, cu_seqlens_host, sm_count(), S0 != nullptr);
  if (!P.any_split)  // nothing is long enough to split: the plain forward
    return chunk_fwd_impl(q, k, v, log_a, b, w, S0, cu_seqlens, cu_seqlens_host, o, S_T, dims, workspace,
                          P.inner, stream, true);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  char *ws = static_cast<char *>(workspace);
  int32_t *pi = reinterpret_cast<int32_t *>(ws + P.off_ints);
  float *G = reinterpret_cast<float *>(ws + P.off_G);
  float *E = reinterpret_cast<float *>(ws + P.off_E);
  float *S3 = reinterpret_cast<float *>(ws + P.off_S3);
  const int H = dims->n_heads;
  cudaError_t e = gdn2::write_ints(pi, P.ints.data(), P.ints.size(), s);
  if (e == cudaSuccess) e = gdn2::launch_fill_starts(E, pi + P.i_src2, nullptr, P.N2, H, s);
  if (e == cudaSuccess) e = gdn2::launch_fill_starts(G, pi + P.i_src1, S0, P.NS, H, s);
  if (e != cudaSuccess) return fail(GDN2_ERR_CUDA, "varlen split setup: %s", cudaGetErrorString(e));
  // pass 2: split segments from the identity (their o rows are rewritten by passes 1 and 3)
  gdn2_dims d2 = *dims;
  d2.n_seqs = P.N2;
  rc = chunk_fwd_impl(q, k, v, log_a, b, w, E, nullptr, nullptr, o, E, &d2, ws, P.inner, stream, true,
                      pi + P.i_b2);
  if (rc) return rc;
  // pass 1: every segment (split ones from 0, unsplit sequences from S0)
  gdn2_dims d1 = *dims;
  d1.n_seqs = P.NS;
  std::vector<int32_t> cu1_host(P.ints.begin() + P.i_cu1, P.ints.begin() + P.i_cu1 + P.NS + 1);
  rc = chunk_fwd_impl(q, k, v, log_a, b, w, G, pi + P.i_cu1, cu1_host.data(), o, G, &d1, ws, P.inner, stream,
                      false);
  if (rc) return rc;
  e = gdn2::launch_combine_varlen(pi + P.i_info, E, G, S3, S0, S_T, dims->n_seqs, H, s);
  if (e != cudaSuccess) return fail(GDN2_ERR_CUDA, "varlen split combine: %s", cudaGetErrorString(e));
  // pass 3: the split segments that start from a non-zero state, from that state: the final o
  if (P.N3 == 0) return GDN2_OK;
  gdn2_dims d3 = *dims;
  d3.n_seqs = P.N3;
  return chunk_fwd_impl(q, k, v, log_a, b, w, S3, nullptr, nullptr, o, nullptr, &d3, ws, P.inner, stream, false,
                        pi + P.i_b3);
}

// ---------------------------------------------------------------- one segment per rank
// Workspace of gdn2_segment_maps / gdn2_segment_correct: the inner forward's workspace, a zero
// v, scratch outputs and (maps only) the identity start states.
struct SegLayout {
  size_t off_zero_v, off_o2, off_ident, total;
};
static SegLayout seg_layout(const gdn2_dims *d, bool maps) {
  SegLayout L;
  const size_t tok = (size_t)d->n_seqs * (size_t)d->seq_len * (size_t)d->n_heads;
  const size_t in_e = d->dtype_in == GDN2_BF16 ? 2 : 4, out_e = d->dtype_out == GDN2_BF16 ? 2 : 4;
  L.off_zero_v = up256(gdn2_chunk_fwd_workspace_size(d));
  L.off_o2 = L.off_zero_v + up256(tok * (size_t)d->d_v * in_e);
  L.off_ident = L.off_o2 + up256(tok * (size_t)d->d_v * out_e);
  L.total = L.off_ident + (maps ? up256((size_t)d->n_seqs * d->n_heads * d->d_k * d->d_v * sizeof(float)) : 0);
  return L;
}

static int check_segment_call(const gdn2_dims *dims, const void *workspace, size_t workspace_bytes, size_t need) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if (dims->d_k != 128 || dims->d_v != 128 || dims->chunk != 64 || dims->dtype_in != GDN2_BF16)
    return fail(GDN2_ERR_UNSUPPORTED, "the segment calls need d_k = d_v = 128, chunk 64 and bf16 inputs");
  if ((int64_t)dims->n_seqs * dims->seq_len >= ((int64_t)1 << 31))
    return fail(GDN2_ERR_UNSUPPORTED, "the segment calls need fewer than 2^31 tokens");
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return fail(GDN2_ERR_WORKSPACE, "workspace must be non-NULL and 256-byte aligned");
  if (workspace_bytes < need) return fail(GDN2_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", workspace_bytes, need);
  return GDN2_OK;
}

size_t gdn2_segment_maps_workspace_size(const gdn2_dims *dims) {
  if (!dims || dims->n_seqs < 1 || dims->n_heads < 1 || dims->seq_len < 0) return 0;
  return seg_layout(dims, true).total;
}

size_t gdn2_segment_correct_workspace_size(const gdn2_dims *dims) {
  if (!dims || dims->n_seqs < 1 || dims->n_heads < 1 || dims->seq_len < 0) return 0;
  return seg_layout(dims, false).total;
}

int gdn2_segment_maps(const void *q, const void *k, const void *v, const void *log_a, const void *b, const void *w,
                      const float *S0, void *o, float *F, float *G, const gdn2_dims *dims, void *workspace,
                      size_t workspace_bytes, gdn2_stream_t stream) {
  g_err[0] = '\0';
  int rc = check_segment_call(dims, workspace, workspace_bytes, gdn2_segment_maps_workspace_size(dims));
  if (rc) return rc;
  if (dims->seq_len > 0) {  // every check before the first launch (an empty segment reads no input)
    rc = check_inputs(q, k, v, log_a, b, w, dims->flags, dims->dtype_in);
    if (rc) return rc;
    if (!o || !aligned16(o)) return fail(GDN2_ERR_INVALID_ARG, "o must be non-NULL and 16-byte aligned");
  }
  if (S0 && !aligned16(S0)) return fail(GDN2_ERR_INVALID_ARG, "S0 must be 16-byte aligned");
  if (!F || !G || !aligned16(F) || !aligned16(G)) return fail(GDN2_ERR_INVALID_ARG, "F and G must be non-NULL and 16-byte aligned");
  const SegLayout L = seg_layout(dims, true);
  char *ws = static_cast<char *>(workspace);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int units = dims->n_seqs * dims->n_heads;
  const size_t state_bytes = (size_t)units * 128 * 128 * sizeof(float);
  float *ident = reinterpret_cast<float *>(ws + L.off_ident);
  cudaError_t e = gdn2::launch_identities(ident, units, s);
  if (e != cudaSuccess) return fail(GDN2_ERR_CUDA, "identity states: %s", cudaGetErrorString(e));
  if (dims->seq_len == 0) {  // an empty segment maps S to S: F = I, G = S0 (or 0)
    e = cudaMemcpyAsync(F, ident, state_bytes, cudaMemcpyDeviceToDevice, s);
    if (e == cudaSuccess)
      e = S0 ? cudaMemcpyAsync(G, S0, state_bytes, cudaMemcpyDeviceToDevice, s) : cudaMemsetAsync(G, 0, state_bytes, s);
    return e == cudaSuccess ? GDN2_OK : fail(GDN2_ERR_CUDA, "empty segment: %s", cudaGetErrorString(e));
  }
  const size_t inner_bytes = L.off_zero_v;
  // o and G: the segment from its given start (S0, or 0)
  rc = chunk_fwd_impl(q, k, v, log_a, b, w, S0, nullptr, nullptr, o, G, dims, ws, inner_bytes, stream, true);
  if (rc) return rc;
  // F: the segment from the identity with v = 0
  const size_t vbytes = (size_t)dims->n_seqs * dims->seq_len * dims->n_heads * 128 * 2;
  e = cudaMemsetAsync(ws + L.off_zero_v, 0, vbytes, s);
  if (e != cudaSuccess) return fail(GDN2_ERR_CUDA, "zero v: %s", cudaGetErrorString(e));
  return chunk_fwd_impl(q, k, ws + L.off_zero_v, log_a, b, w, ident, nullptr, nullptr, ws + L.off_o2, F, dims, ws,
                        inner_bytes, stream, false);
}

int gdn2_affine_prefix(const float *F_all, const float *G_all, float *start, float *S_T, int32_t n_seqs,
                       int32_t n_heads, int32_t n_segs, int32_t seg, gdn2_stream_t stream) {
  g_err[0] = '\0';
  if (!F_all || !G_all) return fail(GDN2_ERR_INVALID_ARG, "F_all and G_all must be non-NULL");
  if (n_seqs < 1 || n_heads < 1 || n_segs < 1 || seg < 0 || seg >= n_segs)
    return fail(GDN2_ERR_INVALID_ARG, "bad sizes (n_seqs=%d n_heads=%d n_segs=%d seg=%d)", n_seqs, n_heads, n_segs, seg);
  if (!start && !S_T) return GDN2_OK;
  const size_t per_seg = (size_t)n_seqs * n_heads;
  const cudaError_t e = gdn2::launch_prefix(F_all, G_all, per_seg, (size_t)n_heads, start, S_T, seg, n_segs, n_seqs,
                                            n_heads, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? GDN2_OK : fail(GDN2_ERR_CUDA, "affine prefix: %s", cudaGetErrorString(e));
}

int gdn2_segment_correct(const void *q, const void *k, const void *log_a, const void *b, const void *w,
                         const float *start, void *o, const gdn2_dims *dims, void *workspace, size_t workspace_bytes,
                         gdn2_stream_t stream) {
  g_err[0] = '\0';
  int rc = check_segment_call(dims, workspace, workspace_bytes, gdn2_segment_correct_workspace_size(dims));
  if (rc) return rc;
  if (dims->seq_len == 0) return GDN2_OK;  // nothing to correct
  rc = check_inputs(q, k, q, log_a, b, w, dims->flags, dims->dtype_in);  // (v is not read: q stands in)
  if (rc) return rc;
  if (!start || !aligned16(start)) return fail(GDN2_ERR_INVALID_ARG, "start must be non-NULL and 16-byte aligned");
  if (!o || !aligned16(o)) return fail(GDN2_ERR_INVALID_ARG, "o must be non-NULL and 16-byte aligned");
  const SegLayout L = seg_layout(dims, false);
  char *ws = static_cast<char *>(workspace);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const size_t n_out = (size_t)dims->n_seqs * dims->seq_len * dims->n_heads * 128;
  cudaError_t e = cudaMemsetAsync(ws + L.off_zero_v, 0, n_out * 2, s);
  if (e != cudaSuccess) return fail(GDN2_ERR_CUDA, "zero v: %s", cudaGetErrorString(e));
  rc = chunk_fwd_impl(q, k, ws + L.off_zero_v, log_a, b, w, start, nullptr, nullptr, ws + L.off_o2, nullptr, dims, ws,
                      L.off_zero_v, stream, true);
  if (rc) return rc;
  e = gdn2::launch_add(o, ws + L.off_o2, n_out, dims->dtype_out, s);
  return e == cudaSuccess ? GDN2_OK : fail(GDN2_ERR_CUDA, "o += correction: %s", cudaGetErrorString(e));
}

int gdn2_check_status(const void *workspace, gdn2_stream_t stream) {
  g_err[0] = '\0';
  if (!workspace) return fail(GDN2_ERR_INVALID_ARG, "workspace is NULL");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return fail(GDN2_ERR_CUDA, "cudaStreamSynchronize: %s", cudaGetErrorString(e));
  int32_t st = 0;
  e = cudaMemcpy(&st, workspace, sizeof(st), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return fail(GDN2_ERR_CUDA, "reading the status word: %s", cudaGetErrorString(e));
  if (st == gdn2::kStatusTimeout) return fail(GDN2_ERR_TIMEOUT, "a bounded device wait timed out");
  if (st == gdn2::kStatusRange)
    return fail(GDN2_ERR_RANGE, "a chunk's decay range exceeds what gdn2_chunk_bwd handles; use gdn2_bwd");
  if (st != 0) return fail(GDN2_ERR_CUDA, "unknown device status %d", st);
  return GDN2_OK;
}

int gdn2_decode_step(const void *q, const void *k, const void *v, const void *log_a, const void *b, const void *w,
                     float *S, void *o, const gdn2_dims *dims, gdn2_stream_t stream) {
  g_err[0] = '\0';
  int rc = check_dims(dims);
  if (rc) return rc;
  if (dims->seq_len != 1) return fail(GDN2_ERR_INVALID_ARG, "gdn2_decode_step needs seq_len == 1");
  rc = check_inputs(q, k, v, log_a, b, w, dims->flags, dims->dtype_in);
  if (rc) return rc;
  if (!S || !aligned16(S) || !o || !aligned16(o))
    return fail(GDN2_ERR_INVALID_ARG, "S and o must be non-NULL and 16-byte aligned");
  if (dims->d_k > 128 || (dims->d_v != 16 && dims->d_v != 32 && dims->d_v != 64 && dims->d_v != 128))
    return fail(GDN2_ERR_UNSUPPORTED, "decode supports d_k <= 128 and d_v in {16, 32, 64, 128} (got %d, %d)",
                dims->d_k, dims->d_v);
  gdn2::DecodeProblem p;
  p.q = q; p.k = k; p.v = v; p.log_a = log_a; p.b = b; p.w = w;
  p.S = S; p.o = o;
  p.n_seqs = dims->n_seqs; p.n_heads = dims->n_heads; p.d_k = dims->d_k; p.d_v = dims->d_v;
  p.dtype_in = dims->dtype_in; p.dtype_out = dims->dtype_out; p.flags = dims->flags;
  p.state_idx = nullptr;
  p.n_slots = 0;
  cudaError_t e = gdn2::launch_decode(p, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(GDN2_ERR_CUDA, "decode launch: %s", cudaGetErrorString(e));
  return GDN2_OK;
}

int gdn2_decode_step_indexed(const void *q, const void *k, const void *v, const void *log_a, const void *b,
                             const void *w, float *S_pool, int32_t n_slots, const int32_t *state_idx, void *o,
                             const gdn2_dims *dims, gdn2_stream_t stream) {
  g_err[0] = '\0';
  int rc = check_dims(dims);
  if (rc) return rc;
  if (dims->seq_len != 1) return fail(GDN2_ERR_INVALID_ARG, "gdn2_decode_step_indexed needs seq_len == 1");
  rc = check_inputs(q, k, v, log_a, b, w, dims->flags, dims->dtype_in);
  if (rc) return rc;
  if (!S_pool || !aligned16(S_pool) || !o || !aligned16(o))
    return fail(GDN2_ERR_INVALID_ARG, "S_pool and o must be non-NULL and 16-byte aligned");
  if (!state_idx || reinterpret_cast<uintptr_t>(state_idx) % 4 != 0)
    return fail(GDN2_ERR_INVALID_ARG, "state_idx must be a non-NULL, 4-byte aligned device int32 array");
  if (n_slots < 1) return fail(GDN2_ERR_INVALID_ARG, "n_slots must be >= 1 (got %d)", n_slots);
  if (dims->d_k > 128 || (dims->d_v != 16 && dims->d_v != 32 && dims->d_v != 64 && dims->d_v != 128))
    return fail(GDN2_ERR_UNSUPPORTED, "decode supports d_k <= 128 and d_v in {16, 32, 64, 128} (got %d, %d)",
                dims->d_k, dims->d_v);
  gdn2::DecodeProblem p;
  p.q = q; p.k = k; p.v = v; p.log_a = log_a; p.b = b; p.w = w;
  p.S = S_pool; p.o = o;
  p.n_seqs = dims->n_seqs; p.n_heads = dims->n_heads; p.d_k = dims->d_k; p.d_v = dims->d_v;
  p.dtype_in = dims->dtype_in; p.dtype_out = dims->dtype_out; p.flags = dims->flags;
  p.state_idx = state_idx;
  p.n_slots = n_slots;
  cudaError_t e = gdn2::launch_decode(p, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(GDN2_ERR_CUDA, "decode launch: %s", cudaGetErrorString(e));
  return GDN2_OK;
}

}  // extern "C"
