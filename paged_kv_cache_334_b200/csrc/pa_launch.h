// pa_launch.h -- internal launchers behind the C ABI (host side).
#pragma once

#include <cuda.h>
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
  // pa_forward_decode: a sequence whose new-token slot is not the one its
  // table gives position ctx - 1 is flagged PA_DEVERR_SLOT and zeroed.
  const int64_t *slot_mapping;
  int32_t dtype;
  int32_t num_blocks, block_size, num_kv_heads, head_dim;
  int32_t batch, num_q_heads, max_blocks;
  int32_t part_tokens, max_parts;
  float scale;
  bool merge;  // true: pa_decode (single-partition output + last-CTA merge)
};

namespace stream {

constexpr int kMaxStages = 4;
constexpr int kMaxPPS = 8;              // virtual pages per stage
constexpr int kVPageBytes = 32 * 1024;  // largest virtual page (whole token rows)
constexpr int kMaxGrid = 192;           // CTAs (one per SM); sizes the workspace
constexpr int kHdrBytes = 8192;         // barriers, descriptors, score exchange
constexpr int kSmemLimit = 232448;      // opt-in shared memory per CTA on sm_100

// Arguments of the persistent decode kernel (decode_stream.cuh).
struct Params {
  // 3-D tiled views (head_dim, token row of the pool, KV head) of the caches,
  // boxes of 64 elements x vbs tokens x all KV heads, 128-byte swizzle; used
  // when `tile` is set (bf16, vbs >= 16).
  CUtensorMap tmap_k;
  CUtensorMap tmap_v;
  const void *q;
  void *out;
  void *key_cache;    // written only by the fused cache write (slot_mapping set)
  void *value_cache;
  // Fused cache write (pa_forward_decode), all NULL for pa_decode: row b of
  // k_new / v_new ([batch][Hkv][D]) goes to slot_mapping[b] when that is the
  // slot of position context_lens[b] - 1 of sequence b.
  const void *k_new;
  const void *v_new;
  const int64_t *slot_mapping;
  const int32_t *block_tables;
  const int32_t *context_lens;
  float *part_ml;     // [kMaxGrid * 2][Hq][2]: (max in log2 units, normaliser)
  float *part_o;      // [kMaxGrid * 2][Hq][D]: normalised partial output
  int32_t *seq_merge;  // [batch][4]: first contributing CTA, contributors, slot of the first
  int32_t *err_word;
  // Split-K mode (pa_decode_splitk) when sk_o is set: sequence b's
  // partition u (part_pages virtual pages) writes sk_max / sk_sum [b][hq][u]
  // (max in natural units, normaliser) and sk_o [b][hq][u][D] (normalised
  // output), max_parts partitions per row; out, part_* and seq_merge unused.
  float *sk_max, *sk_sum, *sk_o;
  int32_t part_pages, max_parts;
  // Suffix mode (shared-prefix decode): the first tok_offset tokens of every
  // sequence are left out (block_tables then points tok_offset / block_size
  // entries into each row, rows table_stride entries apart, max_blocks of
  // them usable) and each (sequence, query head) result goes to seq_ml (max
  // in log2 units, normaliser) and seq_o (normalised output) instead of out.
  float *seq_ml;
  float *seq_o;
  int32_t tok_offset, table_stride;
  int32_t num_blocks, block_size, num_kv_heads, num_q_heads, max_blocks, batch;
  int32_t vbs, log2_vbs, log2_vpp;  // virtual page tokens; log2 of pages per block
  int32_t log2_bs;                  // log2 of block_size
  // 8-token blocks on the tile path: a virtual page of 16 tokens is two
  // blocks, copied as one box per (block, tensor, 64-wide d half)
  int32_t pair;
  int32_t row_bytes;                // one token row, all KV heads (global layout)
  int32_t row_pitch;                // bytes between token rows in a shared-memory stage
  int32_t vpage_stride;             // vbs * row_pitch
  int32_t q_bytes;                  // Hq * D * elt
  int32_t pps, stages, stage_bytes, hdr_bytes;
  int32_t grid;
  int32_t group;                    // query heads per KV head
  int32_t heads_per_warp;           // query heads one consumer warp serves (<= 8)
  int32_t warps_per_kv;             // consumer warps per KV head
  int32_t tile;                     // 1: tensor copies of swizzled boxes, else row copies
  int32_t box_bytes;                // bytes of one box (64 x vbs x Hkv bf16)
  int32_t n_dhalf;                  // boxes per page per tensor (head_dim / 64)
  // FP8 pages: one box of 128 codes x vbs x Hkv per page and tensor, from
  // which the consumers build fp16 fragments of the code values;
  // scale_log2 then includes k_scale and out_scale is v_scale
  int32_t fp8;
  float out_scale;
  float k_scale, v_scale;  // FP8 pages: the fused write's quantisation scales
  float scale_log2;
};

cudaError_t launch_bf16(const Params &p, int head_dim, int group, int hkv, size_t smem,
                        cudaStream_t stream);
// FP8 pages (head_dim 128, up to 8 query heads per KV head, 4 or 8 KV heads).
cudaError_t launch_fp8(const Params &p, int hkv, size_t smem, cudaStream_t stream);
// Second kernel of pa_decode: merge the partials of sequences split across CTAs.
cudaError_t launch_merge_bf16(const Params &p, int head_dim, cudaStream_t stream);
cudaError_t launch_merge_f32(const Params &p, int head_dim, cudaStream_t stream);
cudaError_t launch_f32(const Params &p, int head_dim, int group, int hkv, size_t smem,
                       cudaStream_t stream);

}  // namespace stream

// Arguments of the shared-prefix kernel (prefix.cu).
constexpr int kMaxPrefixBlocks = 2048;
struct PrefixParams {
  // 3-D tiled views: q (head_dim, query head, sequence) with boxes of 64 x
  // group x 128 / group, and the caches (head_dim, token row, KV head) with
  // boxes of 64 x block_size x 1; all with 128-byte swizzle.
  CUtensorMap tmap_q;
  CUtensorMap tmap_k;
  CUtensorMap tmap_v;
  const int32_t *block_tables;  // rows of table_stride entries; the prefix is row 0's first entries
  const int32_t *context_lens;
  const float *seq_ml;          // [batch][Hq] (max in log2 units, normaliser) of each suffix
  const float *seq_o;           // [batch][Hq][D] normalised suffix output
  // Suffixes left by the suffix kernel (suffix.cu): when `merge` is set,
  // (sequence, KV head) pair i's record merge[4i..4i+3] = (first CTA, number
  // of CTAs n, slot of the first CTA, bad); n == 1: the result is in
  // seq_ml / seq_o, n >= 2: in part_ml / part_o rows (CTA * 2 + slot) * Hq + hq,
  // n == 0: no suffix.  NULL: seq_ml / seq_o hold every row's suffix.
  const int32_t *merge;
  const float *part_ml, *part_o;
  void *out;
  int32_t *err_word;
  int32_t batch, num_q_heads, num_kv_heads, group, block_size, table_stride, prefix_blocks,
      num_blocks;
  float scale_log2;
};
size_t prefix_smem_bytes(int head_dim);
cudaError_t launch_prefix(const PrefixParams &p, int head_dim, cudaStream_t stream);

// Arguments of the suffix kernel (suffix.cu): the tokens past the shared
// prefix of every (sequence, KV head) pair on the tensor cores, for groups
// of 64 or 128 query heads per KV head.
struct SuffixParams {
  CUtensorMap tmap_q;  // q (head_dim, query head, sequence), boxes of 64 x group x 1
  CUtensorMap tmap_k;  // caches as in PrefixParams
  CUtensorMap tmap_v;
  // fp32 (head_dim, row) views of seq_o and part_o with boxes of 32 x group
  // and 128-byte swizzle: the epilogue's tiled stores (group 64)
  CUtensorMap tmap_seq_o;
  CUtensorMap tmap_part_o;
  const int32_t *block_tables;
  const int32_t *context_lens;
  float *seq_ml, *seq_o;    // pairs inside one CTA's range: [batch][Hq][2], [batch][Hq][D]
  float *part_ml, *part_o;  // cut pairs: [grid * 2][Hq][2], [grid * 2][Hq][D]
  int32_t *merge;           // [batch * Hkv][4], as read by the prefix kernel
  // pa_forward_decode: sequence b's newest token must sit in slot_mapping[b]
  // as the table gives position ctx - 1, else PA_DEVERR_SLOT and its output
  // is zeroed (NULL: no check)
  const int64_t *slot_mapping;
  int32_t *err_word;
  int32_t batch, num_q_heads, num_kv_heads, group, block_size, table_stride, prefix_blocks,
      num_blocks, grid;
  float scale_log2;
};
size_t suffix_smem_bytes(int head_dim, int group);
cudaError_t launch_suffix(const SuffixParams &p, int head_dim, cudaStream_t stream);
// pa_decode on the tensor-core path (no prefix): each (sequence, KV head)
// pair's rows from its result or its partials, as bf16 `out` rows.
cudaError_t launch_finish(const SuffixParams &p, void *out, int head_dim, cudaStream_t stream);

// Arguments of the paged prefill kernel (prefill.cu).
constexpr int kMaxPrefillBlocks = 4096;  // table entries per sequence (max_blocks_per_seq)
struct PrefillParams {
  CUtensorMap tmap_q;  // q (head_dim, query head, token), boxes of 64 x group x 128 / group
  CUtensorMap tmap_k;  // caches as in PrefixParams
  CUtensorMap tmap_v;
  const int32_t *block_tables;  // [batch][table_stride]
  const int32_t *context_lens;  // [batch]: history including the new tokens
  const int32_t *query_start;   // [batch + 1]: sequence b's new tokens are q rows [qs[b], qs[b+1])
  void *out;                    // [num_tokens][Hq][D] bf16
  int32_t *err_word;
  int32_t batch, num_tokens, num_q_heads, num_kv_heads, group, block_size, table_stride,
      num_blocks;
  int32_t tiles_per_seq;  // ceil(max_query_len * group / 128): grid x
  float scale_log2;
};
size_t prefill_smem_bytes(int head_dim);
cudaError_t launch_prefill(const PrefillParams &p, int head_dim, cudaStream_t stream);

// Query heads handled together by one CTA for a GQA group of `group` heads.
int decode_head_tile(int group);

// With block_tables / context_lens set (num_tokens = batch, token b = the
// newest token of sequence b), a token is written only when its slot is the
// one the table gives position context_lens[b] - 1; others are flagged.
// FP8 pages (dtype PA_DTYPE_FP8_E4M3): row_bytes is a cache row of codes,
// the new rows are bf16 and are quantised with k_scale / v_scale.
cudaError_t launch_write_kv(int32_t dtype, int32_t block_size,
                            int32_t num_blocks, int64_t row_bytes,
                            void *key_cache, void *value_cache,
                            const void *k_new, const void *v_new,
                            const int64_t *slot_mapping, int32_t num_tokens,
                            int32_t *err_word, cudaStream_t stream,
                            const int32_t *block_tables = nullptr,
                            const int32_t *context_lens = nullptr, int32_t max_blocks = 0,
                            float k_scale = 1.f, float v_scale = 1.f);

cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t stream);

// Set the text pa_last_error_message() returns on the calling host thread.
void set_last_error_message(const char *msg);

// Threads of one pa_reduce CTA (one CTA per sequence and query head).
constexpr int kReduceThreads = 512;
cudaError_t launch_reduce(void *out, const float *part_max,
                          const float *part_sum, const float *part_out,
                          const int32_t *context_lens, int32_t batch,
                          int32_t num_q_heads, int32_t head_dim,
                          int32_t partition_tokens, int32_t max_partitions,
                          int32_t out_dtype, int32_t *err_word,
                          cudaStream_t stream);

}  // namespace pa
