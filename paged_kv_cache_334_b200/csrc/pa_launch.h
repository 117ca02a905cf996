// pa_launch.h -- internal launchers behind the C ABI (host side).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace pa {

// Arguments of the decode kernels, validated by the C ABI layer.
struct DecodeArgs {
  const void *q;
  void *out;  // pa_decode only
  const void *key_cache;
  const void *value_cache;
  const int32_t *block_tables;
  const int32_t *context_lens;
  float *part_max;   // [B, Hq, max_parts]
  float *part_sum;   // [B, Hq, max_parts]
  float *part_out;   // [B, Hq, max_parts, D]
  int32_t *counters; // [B * Hkv * head_tiles]; pa_decode only
  int32_t *err_word;
  int32_t dtype;
  int32_t num_blocks, block_size, num_kv_heads, head_dim;
  int32_t batch, num_q_heads, max_blocks;
  int32_t part_tokens, max_parts;
  float scale;
  bool merge;  // true: pa_decode (single-partition output + last-CTA merge)
};

// Query heads handled together by one CTA for a GQA group of `group` heads.
int decode_head_tile(int group);

cudaError_t launch_write_kv(int32_t dtype, int32_t block_size,
                            int32_t num_blocks, int64_t row_bytes,
                            void *key_cache, void *value_cache,
                            const void *k_new, const void *v_new,
                            const int64_t *slot_mapping, int32_t num_tokens,
                            int32_t *err_word, cudaStream_t stream);

cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t stream);

// Set the text pa_last_error_message() returns on the calling host thread.
void set_last_error_message(const char *msg);

cudaError_t launch_reduce(void *out, const float *part_max,
                          const float *part_sum, const float *part_out,
                          const int32_t *context_lens, int32_t batch,
                          int32_t num_q_heads, int32_t head_dim,
                          int32_t partition_tokens, int32_t max_partitions,
                          int32_t out_dtype, int32_t *err_word,
                          cudaStream_t stream);

}  // namespace pa
