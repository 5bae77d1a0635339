// noalloc.cu -- gdn2_chunk_fwd_noalloc: the chunked forward for callers that
// cannot allocate device memory.
//
// gdn2_chunk_fwd needs a small device workspace (a status word, the unit
// counter of its persistent kernel and the longest-first unit schedule) that
// the caller allocates.  Some callers cannot: a plugin running inside a host
// framework whose allocator owns all device memory (for example a serving
// engine that reserves nearly all of HBM for its caches up front), or code on
// a path where cudaMalloc and its implicit device synchronisation are not
// allowed.  This entry point uses instead a fixed scratch array that lives in
// the library's own device image: every GPU that loads libgdn2.so holds it
// until the process exits.  It calls no cudaMalloc, cudaFree or any
// allocating routine; it hands the array to the ordinary gdn2_chunk_fwd.
//
// In host code the array's name is only a stand-in for the device symbol, so
// its device address is looked up once per device with cudaGetSymbolAddress
// (with that device current) and cached.
#include <cuda_runtime.h>

#include <cstdio>
#include <mutex>

#include "internal.h"

namespace {

// 256-byte header (status word, unit counter) + one int32 per (sequence, head) unit, the
// schedule part rounded up to 256 bytes exactly as gdn2_chunk_fwd_workspace_size rounds it,
// so that a request at the limit always fits.
constexpr size_t kNoAllocScheduleBytes = ((4 * (size_t)GDN2_NOALLOC_MAX_UNITS + 255) / 256) * 256;
constexpr size_t kNoAllocScratchBytes = 256 + kNoAllocScheduleBytes;
static_assert(kNoAllocScratchBytes >= 256 + 4 * (size_t)GDN2_NOALLOC_MAX_UNITS, "scratch too small");
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_setup_mutex;
void *g_scratch_ptr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device (looked up once per device).
// With lookup == false a device that has never run the entry point reports NULL.
int scratch_for_current_device(void **out, bool lookup = true) {
  char msg[256];
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    snprintf(msg, sizeof(msg), "gdn2_chunk_fwd_noalloc: cudaGetDevice: %s", cudaGetErrorString(e));
    return gdn2::set_last_error(GDN2_ERR_CUDA, msg);
  }
  if (dev < 0 || dev >= kMaxDevices) {
    snprintf(msg, sizeof(msg), "gdn2_chunk_fwd_noalloc: device %d is beyond the %d devices it supports", dev,
             kMaxDevices);
    return gdn2::set_last_error(GDN2_ERR_UNSUPPORTED, msg);
  }
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (!g_scratch_ptr[dev] && lookup) {
    void *ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
    if (e != cudaSuccess || ptr == nullptr) {
      snprintf(msg, sizeof(msg), "gdn2_chunk_fwd_noalloc: cudaGetSymbolAddress of the scratch array failed: %s",
               cudaGetErrorString(e));
      return gdn2::set_last_error(GDN2_ERR_CUDA, msg);
    }
    g_scratch_ptr[dev] = ptr;
  }
  *out = g_scratch_ptr[dev];
  return GDN2_OK;
}

}  // namespace

extern "C" int gdn2_chunk_fwd_noalloc(const void *q, const void *k, const void *v, const void *log_a, const void *b,
                                      const void *w, const float *S0, const int32_t *cu_seqlens,
                                      const int32_t *cu_seqlens_host, void *o, float *S_T, const gdn2_dims *dims,
                                      gdn2_stream_t stream) {
  if (dims && (long long)dims->n_seqs * (long long)dims->n_heads > (long long)GDN2_NOALLOC_MAX_UNITS) {
    char msg[256];
    snprintf(msg, sizeof(msg),
             "gdn2_chunk_fwd_noalloc: %d sequences x %d heads = %lld units exceeds the fixed scratch limit of %d "
             "units; use gdn2_chunk_fwd with a caller-allocated workspace",
             dims->n_seqs, dims->n_heads, (long long)dims->n_seqs * (long long)dims->n_heads,
             GDN2_NOALLOC_MAX_UNITS);
    return gdn2::set_last_error(GDN2_ERR_UNSUPPORTED, msg);
  }
  void *scratch = nullptr;
  const int rc = scratch_for_current_device(&scratch);
  if (rc != GDN2_OK) return rc;
  return gdn2_chunk_fwd(q, k, v, log_a, b, w, S0, cu_seqlens, cu_seqlens_host, o, S_T, dims, scratch,
                        kNoAllocScratchBytes, stream);
}

// Status of the last gdn2_chunk_fwd_noalloc on the current device: its bounded device waits
// record a timeout in word 0 of the fixed array, which the caller has no pointer to.
extern "C" int gdn2_chunk_fwd_noalloc_status(gdn2_stream_t stream) {
  void *scratch = nullptr;
  int rc = scratch_for_current_device(&scratch, false);
  if (rc != GDN2_OK) return rc;
  if (!scratch) return GDN2_OK;  // no call has run on this device
  return gdn2_check_status(scratch, stream);
}
