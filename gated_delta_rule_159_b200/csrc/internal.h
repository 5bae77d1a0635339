// internal.h -- host-side launch interfaces between the C-ABI layer (api.cu)
// and the kernel translation units.  Not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/gdn2.h"

namespace gdn2 {

// Resolved problem for one chunk_fwd call (validated by api.cu).
struct ChunkProblem {
  const void *q, *k, *v, *log_a, *b, *w;
  const float *S0;
  const int32_t *cu_seqlens;  // device, may be null (equal lengths)
  void *o;
  float *S_T;
  int n_seqs, seq_len, n_heads, d_k, d_v, chunk;
  int dtype_in, dtype_out;
  uint32_t flags;
  int64_t t_total;
  // Device workspace: status word + optional unit schedule.
  int32_t *status;          // one int32, zeroed by the launcher before the kernel runs
  const int32_t *schedule;  // [n_units] unit ids, longest first, or null (identity order)
  // Optional [2 * n_seqs] device array of (first token, end token) per sequence; when set it
  // replaces cu_seqlens for the unit bounds, so the sequences may leave gaps between them
  // (the split forward's passes over a subset of segments).  Tensor-core path only.
  const int32_t *seg_bounds;
  // Optional checkpoint buffer for the backward (tensor-core path only): per chunk a slot of
  // kBwdCkptSlotBytes with the bf16 S_r = Diag(e^{L_ref}) S tile image (the chunk kernel's
  // swizzled [d_k][d_v] layout) and the bf16 T tile, the slots of a unit laid out as
  // tc::ckpt_first_slot says; ckpt_off [n_seqs + 1]
  // (int64) is the first slot of each sequence divided by n_heads, or NULL for equal lengths.
  // With ckpt set, o may be NULL (no output written).
  void *ckpt;
  const int64_t *ckpt_off;
};

struct DecodeProblem {
  const void *q, *k, *v, *log_a, *b, *w;
  float *S;
  void *o;
  int n_seqs, n_heads, d_k, d_v;
  int dtype_in, dtype_out;
  uint32_t flags;
  const int32_t *state_idx;  // NULL: sequence n owns state n; else slot state_idx[n] of S
  int n_slots;               // slots in S when state_idx is set
  uint64_t wait_ns;          // limit of the streaming kernel's bounded waits (set by launch_decode)
  int dbg_skip;              // timeout test hook: CTA 0 arms its first load group without issuing it
};

struct BwdProblem {
  const void *q, *k, *v, *log_a, *b, *w;  // forward inputs (dtype_in)
  const float *S0;                        // [N, H, d_k, d_v] or NULL
  const int32_t *cu_seqlens;              // device [N + 1] or NULL
  const void *dO;                         // [T_tot, H, d_v] (dtype_out)
  const float *dS_T;                      // [N, H, d_k, d_v] or NULL
  void *dq, *dk, *dv, *dlog_a, *db, *dw;  // gradients (dtype_out), shaped like the inputs
  float *dS0;                             // [N, H, d_k, d_v] or NULL
  float *ckpt, *part, *dz;                // workspace pieces (bwd_carve)
  float *prolog;                          // workspace for the fused prologue's copies, or NULL
  const float *inv_norm;                  // [T_tot, H, 2] 1/|q|, 1/|k| when the prologue ran, else NULL
  int n_seqs, seq_len, n_heads, d_k, d_v;
  int64_t t_total;
  int dtype_in, dtype_out;
  uint32_t flags;
};

// Bytes of one backward checkpoint slot (per chunk and (sequence, head)): the bf16 S_r tile
// image (32 KB) and the bf16 T = (I + A)^-1 tile image (8 KB) the checkpointing forward writes.
constexpr size_t kBwdCkptSlotBytes = 128 * 128 * 2 + 64 * 64 * 2;

// Status word values written by kernels (0 = fine).
constexpr int32_t kStatusTimeout = 1;
// A chunk of the tensor-core backward has a decay range beyond its factored form.
constexpr int32_t kStatusRange = 2;

// Activated fp32 copies of the inputs written by the backward's prologue pass.
struct PrologueCopies {
  float *q, *k, *v, *log_a, *b, *w, *inv_norm;
};

size_t bwd_workspace_bytes(int64_t n_seqs, int64_t t_total, int n_heads, int d_k, int d_v, uint32_t flags);
void bwd_carve(BwdProblem &p, void *workspace);
cudaError_t launch_bwd(const BwdProblem &p, cudaStream_t stream);

// Chunked tensor-core backward (bwd_tc.cu; d_k = d_v = 128, bf16 inputs, per-channel gates in
// the default placement, tied or not).  Checkpoint slots a call needs (an upper bound for
// packed batches), the per-sequence slot offsets for packed batches, and the reverse kernel
// over the S_r tiles a checkpointing forward wrote (ChunkProblem::ckpt) and its final states.
size_t bwd_tc_ckpt_slots(int64_t n_seqs, int64_t t_total, int n_heads, bool packed, int seq_len);
cudaError_t launch_ckpt_offsets(const int32_t *cu_seqlens, int n_seqs, int64_t *off, cudaStream_t stream);
cudaError_t launch_bwd_tc(const BwdProblem &p, const void *ckpt, const float *S_fin, const int64_t *ckpt_off,
                          const int32_t *schedule, int32_t *status, int32_t *counter, cudaStream_t stream);
// The fused prologue of gdn2_chunk_bwd: activated bf16 copies of q, k, log_a, b, w (w NULL with
// tied gates) and the inverse norms 1/|q|, 1/|k| per (token, head); afterwards the activations'
// chain rule in place on the gradients (p's inputs are the raw ones).
struct PrologueCopiesBf16 {
  __nv_bfloat16 *q, *k, *log_a, *b, *w;
  float *inv_norm;
};
cudaError_t launch_prolog_act(const BwdProblem &p, const PrologueCopiesBf16 &c, cudaStream_t stream);
cudaError_t launch_prolog_chain(const BwdProblem &p, const float *inv_norm, cudaStream_t stream);

// Sequence-parallel forward (seqpar.cu): segments of seg_len tokens, workspace offsets.
struct SplitPlan {
  int seg_len, n_per_seq, n_segs;
  size_t off_inner, off_cu, off_start, off_F, off_G, off_zero_v, off_o2, total;
};
struct SplitArgs {
  SplitPlan plan;
  int N, T, H, dtype_out;
  int32_t *cu;
  float *starts, *F, *G, *S_T;
  const float *S0;
  void *o;
  const void *o2;
};
// inner_bytes: workspace of the inner chunked forwards over all segments
SplitPlan split_plan(int N, int T, int H, int n_split, int dtype_in, int dtype_out, size_t inner_bytes);
// what: 0 segment bounds, 1 pass-1 starts, 2 identity starts, 3 combine, 4 o += o2
cudaError_t launch_split_helpers(int what, const SplitArgs &a, cudaStream_t stream);
// Helpers of the per-rank segment calls: `units` 128 x 128 identities; o += o2 (n elements);
// the start state of segment `upto` and the end state after n_segs segments (see prefix_kernel).
cudaError_t launch_identities(float *dst, int units, cudaStream_t stream);
// Packed varlen split helpers: host-planned int32 values to the device (kernel parameters,
// no stream synchronisation); start states (src[u] = -2 identity, -1 zero, n >= 0 S0[n]);
// the serial combine per (sequence, head) from seq_info[4 n] = {m, pass-1, pass-2, pass-3
// index of its first segment}.
cudaError_t write_ints(int32_t *dst, const int32_t *vals, size_t n, cudaStream_t stream);
cudaError_t launch_fill_starts(float *dst, const int32_t *src, const float *S0, int units, int H,
                               cudaStream_t stream);
cudaError_t launch_combine_varlen(const int32_t *seq_info, const float *E, const float *G, float *starts3,
                                  const float *S0, float *S_T, int N, int H, cudaStream_t stream);
cudaError_t launch_add(void *o, const void *o2, size_t n, int dtype_out, cudaStream_t stream);
cudaError_t launch_prefix(const float *F, const float *G, size_t seg_stride, size_t seq_stride, float *start,
                          float *S_T, int upto, int n_segs, int N, int H, cudaStream_t stream);

// Record `message` as this thread's gdn2_last_error() text and return `code`.
int set_last_error(int code, const char *message);

// The one-shot timeout test hook (gdn2_debug_timeout_once): true, with the armed wait limit,
// when the next launch of the kernel at `site` (GDN2_DEBUG_CHUNK / GDN2_DEBUG_DECODE) is to
// run it; the hook is then disarmed.
bool take_debug_timeout(int site, uint64_t *wait_ns);

cudaError_t launch_decode(const DecodeProblem &p, cudaStream_t stream);
// Synchronise `stream`, read and clear the decode status word; returns a cudaError_t value.
int read_decode_status(cudaStream_t stream, int32_t *out);
cudaError_t launch_chunk_simt(const ChunkProblem &p, cudaStream_t stream);
// Tensor-core path (d_k = d_v = 128, C = 64, bf16 in).  Returns cudaErrorNotSupported
// when the problem is outside what it handles.
cudaError_t launch_chunk_tc(const ChunkProblem &p, cudaStream_t stream, const char **why);
// Tensor map of a [t_total][H][128] bf16 tensor viewed as (channel, head, token): boxes of 64
// channels x 1 head x 64 tokens with the 128-byte swizzle (the tile layout of the tensor-core
// kernels).  False when the driver entry point is missing or the geometry is rejected.
bool make_row_tile_map(CUtensorMap *m, const void *base, int64_t t_total, int H);

}  // namespace gdn2
