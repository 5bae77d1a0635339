// internal.h -- host-side launch interfaces between the C-ABI layer (api.cu)
// and the kernel translation units.  Not part of the public ABI.
#pragma once

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
};

struct DecodeProblem {
  const void *q, *k, *v, *log_a, *b, *w;
  float *S;
  void *o;
  int n_seqs, n_heads, d_k, d_v;
  int dtype_in, dtype_out;
  uint32_t flags;
};

// Status word values written by kernels (0 = fine).
constexpr int32_t kStatusTimeout = 1;

// Record `message` as this thread's gdn2_last_error() text and return `code`.
int set_last_error(int code, const char *message);

cudaError_t launch_decode(const DecodeProblem &p, cudaStream_t stream);
cudaError_t launch_chunk_simt(const ChunkProblem &p, cudaStream_t stream);
// Tensor-core path (d_k = d_v = 128, C = 64, bf16 in).  Returns cudaErrorNotSupported
// when the problem is outside what it handles.
cudaError_t launch_chunk_tc(const ChunkProblem &p, cudaStream_t stream, const char **why);

}  // namespace gdn2
