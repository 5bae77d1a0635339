/*
 * gdn2.h -- C ABI of libgdn2.so: the Gated DeltaNet-2 token-mixer forward on
 * NVIDIA B200 (sm_100a).
 *
 * The operation (per head, state S of d_k x d_v in fp32), for every token t:
 *
 *   decay       Sbar = Diag(a_t) S_{t-1},   a_t = exp(log_a_t) in (0, 1]^{d_k}
 *   erase read  r_t  = Sbar^T k_t
 *   erase       S'   = Sbar - (b_t . k_t) r_t^T
 *   write       S_t  = S'   + (w_t . k_t) v_t^T
 *   read        o_t  = S_t^T q_t
 *
 * Sources: gist.science "Gated DeltaNet-2: Decoupling Erase and Write in
 * Linear Attention", Methodologie 1 (channel-wise erase gate b_t and write gate
 * w_t, channel-wise decay D_t = Diag(alpha_t) from KDA); alanhou.org "Core
 * Mechanism" (b_t erases, w_t writes; O(1) recurrent inference and a chunkwise
 * WY algorithm for training); neelmishra.github.io "Gated DeltaNet", section
 * "Decay first, then compute the write error" (key x value orientation; the
 * erase read uses the decayed state); cours.spawnkit.ai session 16, worked trace
 * (read after the update).  Where those pages differ on which side the gates
 * sit, this library follows the form above by default (erase outer factor
 * b.k, erase read with k, write outer factor w.k) and offers the gist.science
 * equation as GDN2_GATE_FORM_P3:
 *
 *   S_t = (I - k_t (b_t . k_t)^T) Diag(a_t) S_{t-1} + k_t (w_t . v_t)^T,
 *   o_t = S_t^T q_t,
 *
 * where the erase read uses b.k, the erase and write outer factors are k and
 * the write gate w_t has d_v channels and scales the value.
 *
 * Conventions for every entry point:
 *  - All tensor pointers are DEVICE pointers owned by the caller; the library
 *    never allocates or frees them.  Tensors are dense row-major with the
 *    shapes given below; every base pointer must be 16-byte aligned, except
 *    the [T, H] scalar-gate arrays of GDN2_SCALAR_DECAY / GDN2_SCALAR_GATES,
 *    which need only the alignment of their element type.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *    stream) and never synchronise the device.  A non-zero status means
 *    nothing was launched (argument errors) or the launch failed (CUDA
 *    errors); gdn2_last_error() then describes it.
 *  - Values are not validated.  Preconditions: finite inputs; log_a <= 0 (the
 *    decay is bounded in (0, 1], cours.spawnkit.ai session 16 "Stability");
 *    b, w in [0, 1]; q and k L2-normalised by the caller (no 1/sqrt(d_k) scale
 *    is applied).  Any finite log_a <= 0 is in range: the tensor-core chunked
 *    path factors each chunk's decay around a per-channel reference when every
 *    channel decays by at most 128 nats over the chunk, and runs a chunk with a
 *    wider decay range token by token (neelmishra.github.io, "What makes the
 *    architecture more than a recurrence": chunk sizes and intermediate
 *    numerical ranges).
 */
#ifndef GDN2_H
#define GDN2_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Opaque CUDA stream handle; binary-compatible with cudaStream_t. */
typedef struct CUstream_st *gdn2_stream_t;

/* Status codes returned by every entry point. */
enum gdn2_status {
  GDN2_OK = 0,
  GDN2_ERR_INVALID_ARG = -1,  /* null/misaligned pointer, bad dims, bad cu_seqlens_host */
  GDN2_ERR_UNSUPPORTED = -2,  /* valid request the library has no kernel for */
  GDN2_ERR_CUDA = -3,         /* a CUDA runtime call or kernel launch failed */
  GDN2_ERR_TIMEOUT = -4,      /* a bounded device-side wait gave up (reported by gdn2_check_status) */
  GDN2_ERR_WORKSPACE = -5,    /* workspace pointer NULL or smaller than the queried size */
  GDN2_ERR_RANGE = -6         /* gdn2_chunk_bwd met a chunk whose decay range is beyond its
                                 factored form (reported by gdn2_check_status) */
};

/* Element types of the per-token inputs (dtype_in) and of o (dtype_out). */
enum gdn2_dtype { GDN2_BF16 = 0, GDN2_F32 = 1 };

/* Flags (dims.flags). */
enum gdn2_flags {
  GDN2_SCALAR_DECAY = 1u,  /* log_a is [T_tot, H]: one decay per token and head (a = alpha 1) */
  GDN2_SCALAR_GATES = 2u,  /* b and w are [T_tot, H]: one erase and one write gate per token and head */
  GDN2_TIED_GATES = 4u,    /* w is b (the w pointer is ignored and may be NULL) */
  GDN2_GATE_FORM_P3 = 8u,  /* gist.science gate placement (above): w is [T_tot, H, d_v]; with
                              GDN2_TIED_GATES and per-channel gates it needs d_k == d_v */
  GDN2_FUSED_PROLOGUE = 16u /* q, k, log_a, b, w carry pre-activations and the kernels apply the
                              mixer's activations (neelmishra.github.io, "What makes the architecture
                              more than a recurrence" and "Read the limiting cases"):
                              q <- q / sqrt(|q|^2 + 1e-6), k likewise (over d_k);
                              log_a <- log sigmoid(log_a); b <- sigmoid(b); w <- sigmoid(w). */
};

/*
 * Problem description shared by both entry points.
 *   n_seqs     N, number of sequences (>= 1).
 *   seq_len    tokens per sequence when cu_seqlens == NULL (all N equal);
 *              total packed tokens T_tot when cu_seqlens != NULL.
 *              gdn2_decode_step requires seq_len == 1.
 *   n_heads    H.
 *   d_k, d_v   head dimensions.
 *   chunk      C, chunk length of the chunked path (ignored by decode).
 *   dtype_in   enum gdn2_dtype of q, k, v, log_a, b, w.
 *   dtype_out  enum gdn2_dtype of o.
 *   flags      enum gdn2_flags, OR-ed.
 */
typedef struct gdn2_dims {
  int32_t n_seqs;
  int32_t seq_len;
  int32_t n_heads;
  int32_t d_k;
  int32_t d_v;
  int32_t chunk;
  int32_t dtype_in;
  int32_t dtype_out;
  uint32_t flags;
  int32_t reserved; /* must be 0 */
} gdn2_dims;

/*
 * gdn2_chunk_fwd -- chunked (prefill) forward over N packed sequences.
 *
 * Computes o and the final state S_T of the recurrence above for every
 * (sequence, head) with the chunkwise-parallel WY form (alanhou.org "Core
 * Mechanism": decay absorbed into asymmetric erase factors; gist.science
 * Methodologie 3: lower-triangular (I + T)^-1 solve giving erase-side and
 * write-side auxiliaries).  The result equals the token-by-token recurrence up
 * to rounding.
 *
 * Arguments (T_tot = N * seq_len without cu_seqlens):
 *   q, k         [T_tot, H, d_k]  dtype_in
 *   v            [T_tot, H, d_v]  dtype_in
 *   log_a        [T_tot, H, d_k]  dtype_in, log of the decay (<= 0); [T_tot, H] with GDN2_SCALAR_DECAY
 *   b, w         [T_tot, H, d_k]  dtype_in, erase / write gates; [T_tot, H] with GDN2_SCALAR_GATES;
 *                w may be NULL with GDN2_TIED_GATES; w is [T_tot, H, d_v] with GDN2_GATE_FORM_P3
 *   S0           [N, H, d_k, d_v] fp32 initial states, or NULL for zeros.  May alias S_T.
 *   cu_seqlens   device int32 [N + 1] token offsets (0 = cu[0] <= ... <= cu[N] = T_tot), or NULL
 *   cu_seqlens_host  optional host copy of cu_seqlens used to schedule the longest sequences
 *                first; NULL lets the device order them.  Must match cu_seqlens when given.
 *   o            [T_tot, H, d_v]  dtype_out (written); must not alias an input.
 *   S_T          [N, H, d_k, d_v] fp32 final states (written), or NULL to skip them.
 *   workspace    device scratch of at least gdn2_chunk_fwd_workspace_size(dims) bytes,
 *                256-byte aligned, owned by the caller; its contents need not be initialised
 *                and must not be used by another call running concurrently on the GPU.
 * Supported: d_k = d_v = 128, C = 64, bf16 in, bf16 or fp32 out (tensor-core path);
 *            d_k, d_v <= 64, C in {16, 32, 64}, bf16 or fp32 in (small-head path).
 * Errors: GDN2_ERR_INVALID_ARG, GDN2_ERR_UNSUPPORTED, GDN2_ERR_WORKSPACE, GDN2_ERR_CUDA.
 */
int gdn2_chunk_fwd(const void *q, const void *k, const void *v,
                   const void *log_a, const void *b, const void *w,
                   const float *S0, const int32_t *cu_seqlens, const int32_t *cu_seqlens_host,
                   void *o, float *S_T, const gdn2_dims *dims,
                   void *workspace, size_t workspace_bytes, gdn2_stream_t stream);

/* Bytes of device workspace gdn2_chunk_fwd needs for `dims` (0 if dims are invalid). */
size_t gdn2_chunk_fwd_workspace_size(const gdn2_dims *dims);

/*
 * gdn2_check_status -- synchronises `stream`, then reads the device status word
 * that gdn2_chunk_fwd left in `workspace` (bounded waits inside the kernel
 * record a timeout there instead of hanging; gdn2_chunk_bwd also records a chunk
 * beyond its decay range there).  Returns GDN2_OK, GDN2_ERR_TIMEOUT, GDN2_ERR_RANGE
 * or GDN2_ERR_CUDA.  Optional: a caller that never checks loses nothing but the
 * diagnosis.
 */
int gdn2_check_status(const void *workspace, gdn2_stream_t stream);

/*
 * gdn2_decode_step -- one recurrent step (alanhou.org "Core Mechanism": inference
 * runs as a pure RNN with O(1) memory per token) for N sequences, updating the
 * states in place: every state is read once and written once.
 *   q, k, log_a, b, w  [N, H, d_k] dtype_in ([N, H] for the scalar flags;
 *                      w is [N, H, d_v] with GDN2_GATE_FORM_P3)
 *   v                  [N, H, d_v] dtype_in
 *   S                  [N, H, d_k, d_v] fp32, read and overwritten in place
 *   o                  [N, H, d_v] dtype_out
 * dims.seq_len must be 1.  Supported: d_k <= 128, d_v in {16, 32, 64, 128},
 * bf16 or fp32 in, fp32 or bf16 out.
 * Errors: GDN2_ERR_INVALID_ARG, GDN2_ERR_UNSUPPORTED, GDN2_ERR_CUDA.
 */
int gdn2_decode_step(const void *q, const void *k, const void *v,
                     const void *log_a, const void *b, const void *w,
                     float *S, void *o, const gdn2_dims *dims, gdn2_stream_t stream);

/*
 * gdn2_chunk_fwd_split -- gdn2_chunk_fwd for long sequences when the (sequence,
 * head) units alone would leave SMs idle: every sequence is cut into up to
 * n_split segments (whole 64-token chunks) that run side by side.  The
 * recurrence is affine in its state (neelmishra.github.io, "What makes the
 * architecture more than a recurrence": the affine-composition view holds once
 * each transition includes decay): a segment maps its start state S_s to
 * F S_s + G and its outputs split into a part from S_s = 0 and a part from S_s
 * with v = 0.  Three chunked passes over all segments (start 0; start I with
 * v = 0, giving F; the combined true starts with v = 0) and a serial combine
 * per (sequence, head) give the same o and S_T as gdn2_chunk_fwd up to
 * rounding, for about three times its work.
 * Arguments as gdn2_chunk_fwd for N = dims.n_seqs equal sequences of
 * dims.seq_len tokens (no cu_seqlens); n_split >= 1.
 * Supported: d_k = d_v = 128, chunk 64, bf16 inputs.  workspace: at least
 * gdn2_chunk_fwd_split_workspace_size(dims, n_split) bytes, 256-byte aligned;
 * gdn2_check_status(workspace) reports a timed-out wait of any of the passes.
 * Errors: GDN2_ERR_INVALID_ARG, GDN2_ERR_UNSUPPORTED, GDN2_ERR_WORKSPACE, GDN2_ERR_CUDA.
 */
int gdn2_chunk_fwd_split(const void *q, const void *k, const void *v,
                         const void *log_a, const void *b, const void *w,
                         const float *S0, void *o, float *S_T, const gdn2_dims *dims, int32_t n_split,
                         void *workspace, size_t workspace_bytes, gdn2_stream_t stream);

/* Bytes of workspace gdn2_chunk_fwd_split needs (0 if the arguments are invalid). */
size_t gdn2_chunk_fwd_split_workspace_size(const gdn2_dims *dims, int32_t n_split);

/*
 * gdn2_chunk_fwd_split_varlen -- gdn2_chunk_fwd over a packed varlen batch in which some
 * sequences are much longer than the balanced share of work per SM: those sequences are
 * cut into whole-chunk segments that run side by side (the affine-composition view of
 * neelmishra.github.io, "What makes the architecture more than a recurrence", as in
 * gdn2_chunk_fwd_split), the others run whole.  The plan is made on the host from
 * cu_seqlens_host: with tau the balanced number of 64-token chunks per SM, a sequence of
 * more than 3 tau chunks is cut into segments of about tau chunks.  Four device steps:
 * the split sequences' segments from the identity state (E = F + G per segment); every
 * segment from the zero state (unsplit sequences from S0): G and provisional outputs; a
 * serial combine per (sequence, head) (F = E - G, S <- F S + G, giving S_T and every
 * segment's true start); the split segments with a non-zero start re-run from it, which
 * writes their final outputs.  The split sequences cost about three times their work;
 * when no sequence qualifies the call is the plain gdn2_chunk_fwd.  Same o and S_T as
 * gdn2_chunk_fwd up to rounding.
 * Arguments as gdn2_chunk_fwd with cu_seqlens; cu_seqlens_host is required here.
 * Supported: d_k = d_v = 128, chunk 64, bf16 inputs.  workspace: at least
 * gdn2_chunk_fwd_split_varlen_workspace_size(dims, cu_seqlens_host) bytes (the plan, and so
 * the size, depends on the lengths and on the current device's SM count), 256-byte aligned;
 * gdn2_check_status(workspace) reports a timed-out wait of any pass.
 * Errors: GDN2_ERR_INVALID_ARG, GDN2_ERR_UNSUPPORTED, GDN2_ERR_WORKSPACE, GDN2_ERR_CUDA.
 */
int gdn2_chunk_fwd_split_varlen(const void *q, const void *k, const void *v,
                                const void *log_a, const void *b, const void *w,
                                const float *S0, const int32_t *cu_seqlens, const int32_t *cu_seqlens_host,
                                void *o, float *S_T, const gdn2_dims *dims,
                                void *workspace, size_t workspace_bytes, gdn2_stream_t stream);

/* Bytes of workspace gdn2_chunk_fwd_split_varlen needs (0 if the arguments are invalid). */
size_t gdn2_chunk_fwd_split_varlen_workspace_size(const gdn2_dims *dims, const int32_t *cu_seqlens_host);

/*
 * Sequence parallelism across ranks (one process per GPU): rank r of R holds tokens
 * [r L, (r + 1) L) of each of N equal sequences (all heads) and runs, on its own GPU,
 *
 *   1. gdn2_segment_maps: its outputs o from the start state 0 (rank 0: the true S0),
 *      and its segment's affine map S_end = F S_start + G (the same affine view as
 *      gdn2_chunk_fwd_split: F is the end state from S_start = I with v = 0, G the end
 *      state from the start above);
 *   2. an all-gather of every rank's F and G (the caller's collective, e.g. NCCL), laid
 *      out [R][N][H][128][128] fp32;
 *   3. gdn2_affine_prefix: its true start state S_s(r) = F_{r-1} S_s(r-1) + G_{r-1},
 *      S_s(0) = 0 (rank 0's outputs and G already include S0), and, when S_T is given,
 *      the end state of the whole sequences;
 *   4. gdn2_segment_correct (ranks r > 0): o += the outputs of its segment from S_s(r)
 *      with v = 0.
 * Together they give gdn2_chunk_fwd's o (each rank its tokens) and S_T up to rounding.
 * dims describe the rank's local segment: N = dims.n_seqs sequences of dims.seq_len
 * tokens, no cu_seqlens.  Supported: d_k = d_v = 128, chunk 64, bf16 inputs.  All
 * pointers are device pointers owned by the caller; workspaces are 256-byte aligned
 * and at least the size the matching *_workspace_size call returns.
 * Errors: GDN2_ERR_INVALID_ARG, GDN2_ERR_UNSUPPORTED, GDN2_ERR_WORKSPACE, GDN2_ERR_CUDA.
 *
 * gdn2_segment_maps: q, k, v, log_a, b, w, S0 (may be NULL), o as gdn2_chunk_fwd with
 * 4-D-equivalent layout [N * L, H, d]; F, G: [N][H][128][128] fp32 outputs.  An empty
 * segment (dims.seq_len = 0) reads no input: F = I, G = S0 (or 0).
 */
int gdn2_segment_maps(const void *q, const void *k, const void *v,
                      const void *log_a, const void *b, const void *w,
                      const float *S0, void *o, float *F, float *G, const gdn2_dims *dims,
                      void *workspace, size_t workspace_bytes, gdn2_stream_t stream);
size_t gdn2_segment_maps_workspace_size(const gdn2_dims *dims);

/*
 * gdn2_affine_prefix: F_all, G_all [n_segs][n_seqs][n_heads][128][128] fp32 (segment
 * `seg` = rank `seg`); start (may be NULL): [n_seqs][n_heads][128][128] fp32, receives
 * S_s(seg) (zeros for seg 0); S_T (may be NULL): receives the state after all n_segs
 * segments.  One CTA per (sequence, head), serial over the segments.
 */
int gdn2_affine_prefix(const float *F_all, const float *G_all, float *start, float *S_T,
                       int32_t n_seqs, int32_t n_heads, int32_t n_segs, int32_t seg,
                       gdn2_stream_t stream);

/*
 * gdn2_segment_correct: o (dims.dtype_out, [N * L, H, 128]) += the outputs of the
 * segment run from `start` ([N][H][128][128] fp32) with v = 0; q, k, log_a, b, w as
 * gdn2_chunk_fwd (v is not needed).
 */
int gdn2_segment_correct(const void *q, const void *k, const void *log_a, const void *b, const void *w,
                         const float *start, void *o, const gdn2_dims *dims,
                         void *workspace, size_t workspace_bytes, gdn2_stream_t stream);
size_t gdn2_segment_correct_workspace_size(const gdn2_dims *dims);

/*
 * gdn2_decode_status -- synchronise `stream`, then report whether any decode
 * step since the last call gave up a bounded device-side wait (the d_k = d_v =
 * 128 decode streams each state through shared memory with bulk copies and
 * waits at most 1 s for each).  Returns GDN2_OK or GDN2_ERR_TIMEOUT (and clears
 * the record), or GDN2_ERR_CUDA.  Optional, like gdn2_check_status.
 */
int gdn2_decode_status(gdn2_stream_t stream);

/*
 * gdn2_decode_step_indexed -- gdn2_decode_step for continuous batching: the N
 * sequences of this step live in a pool of state slots and sequence n reads and
 * updates slot state_idx[n].  The per-step operation is the same recurrent
 * step (alanhou.org "Core Mechanism": O(1) state per sequence at inference);
 * the pages define no batching scheme, the indirection is this library's.
 *   q, k, v, log_a, b, w, o   as gdn2_decode_step, N = dims.n_seqs rows
 *   S_pool      [n_slots, H, d_k, d_v] fp32 device, updated in place (only the
 *               slots named by state_idx are touched)
 *   n_slots     number of slots in S_pool (>= 1)
 *   state_idx   device int32 [N]: slot of sequence n.  An entry outside
 *               [0, n_slots) marks a padding row: its o row is set to zero and
 *               no state is read or written.  Two rows naming the same slot in
 *               one call race on that slot (the result is undefined).
 * Errors: GDN2_ERR_INVALID_ARG, GDN2_ERR_UNSUPPORTED, GDN2_ERR_CUDA.
 */
int gdn2_decode_step_indexed(const void *q, const void *k, const void *v,
                             const void *log_a, const void *b, const void *w,
                             float *S_pool, int32_t n_slots, const int32_t *state_idx, void *o,
                             const gdn2_dims *dims, gdn2_stream_t stream);

/*
 * gdn2_bwd -- gradients of the forward (gdn2_chunk_fwd with the same inputs)
 * for training.  The method's training path runs a gate-aware backward of its
 * chunked form (gist.science Methodologie 3; alanhou.org "Core Mechanism"),
 * whose formula the pages do not print; the gradient is fixed by the forward,
 * and this call computes it by reverse-mode differentiation of the recurrence
 * token by token (fp32), recomputing the states from checkpoints kept every 4
 * tokens in the workspace.  It returns the gradients of
 *     sum_t <dO_t, o_t> + sum_n <dS_T[n], S_T[n]>.
 * Arguments (T_tot as for gdn2_chunk_fwd; all device pointers, caller-owned):
 *   q, k, v, log_a, b, w, S0, cu_seqlens   the forward's inputs, same layouts and flags
 *                                         (dims.chunk is ignored)
 *   dO       [T_tot, H, d_v] dtype_out    gradient of o
 *   dS_T     [N, H, d_k, d_v] fp32 or NULL (zero)
 *   dq, dk, dlog_a, db, dw, dv            written, dtype_out, each shaped like its input
 *                                         (scalar-flag gates give [T_tot, H]); with
 *                                         GDN2_TIED_GATES the w gradient is added into db
 *                                         and dw may be NULL
 *   dS0      [N, H, d_k, d_v] fp32 or NULL to skip
 *   workspace  >= gdn2_bwd_workspace_size(dims) bytes, 256-byte aligned, uninitialised
 *              is fine; one call at a time per workspace
 * Supported: d_k <= 128, d_v in {16, 32, 64, 128}, bf16 or fp32 in and out.
 * Errors: GDN2_ERR_INVALID_ARG, GDN2_ERR_UNSUPPORTED, GDN2_ERR_WORKSPACE, GDN2_ERR_CUDA.
 */
int gdn2_bwd(const void *q, const void *k, const void *v,
             const void *log_a, const void *b, const void *w,
             const float *S0, const int32_t *cu_seqlens,
             const void *dO, const float *dS_T,
             void *dq, void *dk, void *dv, void *dlog_a, void *db, void *dw, float *dS0,
             const gdn2_dims *dims, void *workspace, size_t workspace_bytes, gdn2_stream_t stream);

/* Bytes of device workspace gdn2_bwd needs for `dims` (0 if dims are unsupported).
 * packed != 0: the call passes cu_seqlens, so dims.seq_len is T_tot; packed == 0:
 * N equal sequences of dims.seq_len tokens. */
size_t gdn2_bwd_workspace_size(const gdn2_dims *dims, int32_t packed);

/*
 * gdn2_chunk_bwd -- the gradients gdn2_bwd returns, computed in the chunked form on the
 * tensor cores.  The method trains through its chunked form with a gate-aware backward
 * (gist.science Methodologie 3, "Poortbewuste terugwaartse pass"); the pages print no
 * formula for it, and this call differentiates the chunk algebra of gdn2_chunk_fwd:
 *   1. a pass of the chunked forward writes each 64-token chunk's start state (as the
 *      bf16 operand tile the chunk uses) and the final state (fp32) to the workspace;
 *      o is not written;
 *   2. one reverse pass per (sequence, head), last chunk first, recomputes each chunk's
 *      auxiliaries from its start state and forms every gradient of the chunk with
 *      bf16 tensor-core products accumulated in fp32, carrying dLoss/dS (fp32) from chunk
 *      to chunk; the chain rule through the decay and the gates runs in the same pass.
 * It returns the gradients of  sum_t <dO_t, o_t> + sum_n <dS_T[n], S_T[n]>  with the
 * precision of the bf16-input chunked forward (the products take bf16 operands), not the
 * fp32 precision of gdn2_bwd.
 * Arguments, layouts and ownership: as gdn2_bwd.  dims.chunk is ignored.
 * Supported: d_k = d_v = 128, bf16 inputs, dtype_out (dO and the gradients) bf16 or fp32;
 * either gate placement (GDN2_GATE_FORM_P3), GDN2_TIED_GATES, GDN2_SCALAR_DECAY and
 * GDN2_SCALAR_GATES (each alone or both), and GDN2_FUSED_PROLOGUE (the passes then run on
 * activated bf16 copies of q, k, log_a, b, w kept in the workspace, and the activations'
 * chain rule is applied to the gradients at the end).  T_tot >= 2^31 gives
 * GDN2_ERR_UNSUPPORTED (gdn2_bwd covers it).
 * Range: every chunk must keep each channel's in-chunk decay L_0 - L_63 within 128 nats
 * (the forward's factored form).  A chunk beyond it is not computed: the call records
 * GDN2_ERR_RANGE for gdn2_check_status(workspace) and that (sequence, head)'s gradients are
 * undefined; gdn2_bwd handles any range.
 * workspace  >= gdn2_chunk_bwd_workspace_size(dims, packed) bytes, 256-byte aligned; one
 *            call at a time per workspace.  It holds the checkpoints: 40 KB per chunk and
 *            (sequence, head) (the bf16 S_r and T tiles), plus one fp32 final state each, and
 *            with the fused prologue the activated copies.
 * Errors: GDN2_ERR_INVALID_ARG, GDN2_ERR_UNSUPPORTED, GDN2_ERR_WORKSPACE, GDN2_ERR_CUDA;
 * gdn2_check_status reports GDN2_ERR_TIMEOUT (a bounded device wait) or GDN2_ERR_RANGE.
 */
int gdn2_chunk_bwd(const void *q, const void *k, const void *v,
                   const void *log_a, const void *b, const void *w,
                   const float *S0, const int32_t *cu_seqlens,
                   const void *dO, const float *dS_T,
                   void *dq, void *dk, void *dv, void *dlog_a, void *db, void *dw, float *dS0,
                   const gdn2_dims *dims, void *workspace, size_t workspace_bytes, gdn2_stream_t stream);

/* Bytes of device workspace gdn2_chunk_bwd needs (0 if dims are unsupported); packed as
 * for gdn2_bwd_workspace_size (for packed batches an upper bound from T_tot and N). */
size_t gdn2_chunk_bwd_workspace_size(const gdn2_dims *dims, int32_t packed);

/*
 * gdn2_chunk_fwd_noalloc -- gdn2_chunk_fwd for callers that cannot allocate
 * device memory.  (The paper has no counterpart; this is a deployment aid.)
 *
 * Some callers cannot call cudaMalloc: a plugin inside a host framework whose
 * allocator owns all device memory (e.g. a serving engine that reserves nearly
 * all of HBM up front), or code on a path where cudaMalloc's implicit device
 * synchronisation is not allowed.  This entry point takes the same arguments
 * as gdn2_chunk_fwd minus the workspace, and uses instead a fixed scratch
 * array of 256 + 4 * GDN2_NOALLOC_MAX_UNITS bytes compiled into the library:
 * every GPU that loads libgdn2.so holds it until the process exits.  It calls
 * no cudaMalloc, cudaFree or other allocating routine.  The caller still owns
 * and passes all inputs and outputs.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current) and caches it; make
 *     that first call before any stream capture.
 *   - All calls share the one array and it keeps the last call's contents; the
 *     call clears the parts that must start at zero itself.  Calls whose
 *     executions overlap on the GPU (different streams, or concurrent host
 *     threads on one device) race on the array: serialise them.
 *   - Problems with more than GDN2_NOALLOC_MAX_UNITS (sequence, head) units
 *     are rejected with GDN2_ERR_UNSUPPORTED and a message naming the limit.
 * Errors: as gdn2_chunk_fwd, plus GDN2_ERR_UNSUPPORTED for the size limit.
 */
#define GDN2_NOALLOC_MAX_UNITS 16384
int gdn2_chunk_fwd_noalloc(const void *q, const void *k, const void *v,
                           const void *log_a, const void *b, const void *w,
                           const float *S0, const int32_t *cu_seqlens, const int32_t *cu_seqlens_host,
                           void *o, float *S_T, const gdn2_dims *dims, gdn2_stream_t stream);

/*
 * gdn2_chunk_fwd_noalloc_status -- gdn2_check_status for gdn2_chunk_fwd_noalloc:
 * synchronises `stream`, then reads the status word that the last
 * gdn2_chunk_fwd_noalloc on the current device left in the fixed array (the
 * caller holds no pointer to it).  Returns GDN2_OK (also when no such call has
 * run on this device), GDN2_ERR_TIMEOUT or GDN2_ERR_CUDA.  The next
 * gdn2_chunk_fwd_noalloc clears the word, so read it before that call.
 */
int gdn2_chunk_fwd_noalloc_status(gdn2_stream_t stream);

/*
 * gdn2_debug_timeout_once -- test hook for the failure detection of the bounded
 * device-side waits; not for production use.  It arms a one-shot fault for the
 * next launch of the kernel named by `site`:
 *   GDN2_DEBUG_CHUNK   the tensor-core chunk kernel (gdn2_chunk_fwd and the calls
 *                      built on it),
 *   GDN2_DEBUG_DECODE  the streaming decode kernel (d_k = d_v = 128),
 *   GDN2_DEBUG_BWD     the reverse kernel of gdn2_chunk_bwd (its checkpointing
 *                      forward runs normally).
 * In that launch every bounded wait uses the limit `wait_ns` instead of 1 s, and
 * the first CTA announces the bytes of its first load group to its mbarrier but
 * issues none of the copies, so its wait runs out: the kernel records
 * GDN2_ERR_TIMEOUT in its status word (read by gdn2_check_status /
 * gdn2_decode_status), lets the copies and MMAs it did issue finish (each wait
 * bounded by the same limit), frees its tensor memory and returns.  No copy is
 * left in flight, no address is faulted, and the outputs of that launch are
 * undefined.  The hook is per process and consumed by the first matching
 * launch; the pages have no counterpart (failure detection is this library's).
 * Errors: GDN2_ERR_INVALID_ARG for an unknown site or wait_ns outside
 * [1000, 10^10].
 */
enum gdn2_debug_site { GDN2_DEBUG_CHUNK = 1, GDN2_DEBUG_DECODE = 2, GDN2_DEBUG_BWD = 3 };
int gdn2_debug_timeout_once(int32_t site, uint64_t wait_ns);

/* Thread-local description of the last non-zero status on this thread ("" if none). */
const char *gdn2_last_error(void);

/* Library version, major * 10000 + minor * 100 + patch. */
int gdn2_version(void);

#ifdef __cplusplus
} /* extern "C" */
#endif

#endif /* GDN2_H */
