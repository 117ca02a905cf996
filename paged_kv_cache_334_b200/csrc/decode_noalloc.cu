// decode_noalloc.cu -- pa_decode_noalloc: decode without a caller workspace.
//
// For callers that are not allowed to allocate device memory (plugins inside
// an engine that owns all device memory, latency-bound loops where
// cudaMalloc / cudaFree may stall the device), the decode scratch space comes
// from the fixed array below instead of a caller-provided workspace.  The
// array is part of the library's device image: each GPU that loads libpa
// holds it until the process exits.  Nothing here calls cudaMalloc, cudaFree
// or any allocating library routine.
//
// Host code must not use `pa_noalloc_scratch` as a pointer: on the host the
// name only stands for the symbol.  Its device address is looked up once per
// device with cudaGetSymbolAddress (with that device current) and kept.
#include <mutex>
#include <stdio.h>

#include "../../include/pa.h"
#include "pa_launch.h"

namespace pa {
// api.cu: pa_decode on the page-stream / partition kernels only (the
// tensor-core path for groups of 64 or 128 heads needs more scratch).
size_t decode_workspace_bytes_streamed(const pa_cache_desc *cache, int32_t batch,
                                       int32_t num_q_heads, int32_t max_blocks_per_seq);
pa_status decode_streamed(const pa_cache_desc *cache, void *out, const void *q,
                          const void *key_cache, const void *value_cache,
                          const int32_t *block_tables, const int32_t *context_lens,
                          int32_t batch, int32_t num_q_heads, int32_t max_blocks_per_seq,
                          float scale, void *workspace, size_t workspace_bytes,
                          int32_t *err_word, pa_stream_t stream);
}  // namespace pa

namespace {

constexpr size_t kScratchBytes = PA_DECODE_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char pa_noalloc_scratch[kScratchBytes];

std::mutex g_setup_mutex;
void *g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device (set up on the
// first call for that device).
pa_status scratch_address(void **addr) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    char msg[256];
    snprintf(msg, sizeof msg, "pa_decode_noalloc: cudaGetDevice failed: %s",
             cudaGetErrorString(e));
    pa::set_last_error_message(msg);
    return PA_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) {
    pa::set_last_error_message("pa_decode_noalloc: device ordinal out of range");
    return PA_ERR_UNSUPPORTED;
  }
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (g_scratch_addr[dev] == nullptr) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, pa_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) {
      char msg[256];
      snprintf(msg, sizeof msg,
               "pa_decode_noalloc: cudaGetSymbolAddress of the scratch array failed: %s",
               cudaGetErrorString(e));
      pa::set_last_error_message(msg);
      return PA_ERR_CUDA;
    }
    g_scratch_addr[dev] = p;
  }
  *addr = g_scratch_addr[dev];
  return PA_OK;
}

}  // namespace

extern "C" pa_status pa_decode_noalloc(const pa_cache_desc *cache, void *out,
                                       const void *q, const void *key_cache,
                                       const void *value_cache,
                                       const int32_t *block_tables,
                                       const int32_t *context_lens,
                                       int32_t batch, int32_t num_q_heads,
                                       int32_t max_blocks_per_seq, float scale,
                                       int32_t *err_word, pa_stream_t stream) {
  const size_t need =
      pa::decode_workspace_bytes_streamed(cache, batch, num_q_heads, max_blocks_per_seq);
  if (need > kScratchBytes) {
    char msg[256];
    snprintf(msg, sizeof msg,
             "pa_decode_noalloc: these sizes need %zu bytes of scratch but the built-in "
             "scratch holds %zu bytes; use pa_decode with a workspace",
             need, kScratchBytes);
    pa::set_last_error_message(msg);
    return PA_ERR_UNSUPPORTED;
  }
  if (need == 0 || batch == 0) {
    // Invalid arguments or an empty batch: pa_decode reports / does nothing.
    return pa::decode_streamed(cache, out, q, key_cache, value_cache, block_tables,
                               context_lens, batch, num_q_heads, max_blocks_per_seq, scale,
                               nullptr, 0, err_word, stream);
  }
  void *scratch = nullptr;
  pa_status s = scratch_address(&scratch);
  if (s != PA_OK) return s;
  // The previous call's leftovers must not be taken for zeroed counters.
  cudaError_t e = cudaMemsetAsync(scratch, 0, need, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) {
    char msg[256];
    snprintf(msg, sizeof msg, "pa_decode_noalloc: clearing the scratch failed: %s",
             cudaGetErrorString(e));
    pa::set_last_error_message(msg);
    return PA_ERR_CUDA;
  }
  return pa::decode_streamed(cache, out, q, key_cache, value_cache, block_tables,
                             context_lens, batch, num_q_heads, max_blocks_per_seq, scale,
                             scratch, kScratchBytes, err_word, stream);
}
