/*
 * pa.h -- C ABI of libpa: attention over a paged KV cache on NVIDIA B200
 * (sm_100a): single-query decode (pa_decode and its variants) and chunked
 * prefill with the causal mask (pa_prefill).
 *
 * The operations follow three public pages:
 *   [route]    "From correct to faster: the PagedAttention optimisation
 *              route" (yjxyzxyz.cn, article oHue8hrF);
 *   [teaching] "Implementing teaching PagedAttention: reading the historical
 *              KV cache from the block table" (yjxyzxyz.cn, article wVdUWYLj);
 *   [serving]  "Operators and compilers: inference attention and KV kernels"
 *              (charles2530.github.io, 2025-09-30).
 *
 * Conventions shared by every call
 * --------------------------------
 * - Every pointer argument except `cache` is a DEVICE pointer on the current
 *   CUDA device, owned by the caller; the library keeps no reference after
 *   the call returns, allocates no memory and never synchronises.  Work is
 *   enqueued on `stream` (a cudaStream_t; NULL = the legacy default stream)
 *   and runs asynchronously: outputs are valid once the stream reaches the
 *   call.
 * - Arrays are dense, row-major, exactly as written:
 *     key_cache, value_cache  [num_blocks, block_size, num_kv_heads, head_dim]
 *     q, out                  [batch, num_q_heads, head_dim] (pa_prefill:
 *                             [num_tokens, num_q_heads, head_dim])
 *     k_new, v_new            [num_tokens, num_kv_heads, head_dim]
 *     block_tables            [batch, max_blocks_per_seq] int32
 *     context_lens            [batch] int32
 *     slot_mapping            [num_tokens] int64
 *   Caches, q, out, k_new, v_new and partial outputs must be 16-byte
 *   aligned.  Elements are fp32 or bf16 (cache->dtype); q, k_new, v_new and
 *   out have the cache's dtype; partials are always fp32.
 * - Query head hq reads KV head hq / (num_q_heads / num_kv_heads)
 *   (contiguous GQA / MQA groups; [serving] section 7 "Why MQA / GQA change
 *   serving performance").
 * - Synchronous errors are returned: PA_ERR_INVALID_ARG for bad sizes,
 *   null or misaligned pointers; PA_ERR_UNSUPPORTED for a shape with no
 *   compiled kernel (head_dim not 64/128, block_size not a power of two
 *   in [1, 256], more than 512 query heads per KV head); PA_ERR_CUDA when
 *   a launch fails.  pa_last_error_message() gives the detail.
 * - Errors that depend on device data are not returned: a block id outside
 *   [0, num_blocks) among a sequence's visible pages, a context length
 *   outside [0, max_blocks_per_seq * block_size], or a slot at or past
 *   num_blocks * block_size set a PA_DEVERR_* bit in *err_word (an int32
 *   in device memory, may be NULL) with an atomic OR; the affected
 *   sequence's output is written as zeros (a bad slot is skipped).  The
 *   caller reads the word after its own synchronisation.  No kernel traps.
 */
#ifndef PA_H_
#define PA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef void *pa_stream_t; /* a cudaStream_t */

typedef enum pa_status {
  PA_OK = 0,
  PA_ERR_INVALID_ARG = 1,
  PA_ERR_UNSUPPORTED = 2,
  PA_ERR_CUDA = 3
} pa_status;

typedef enum pa_dtype { PA_DTYPE_F32 = 0, PA_DTYPE_BF16 = 1, PA_DTYPE_FP8_E4M3 = 2 } pa_dtype;

/*
 * FP8 pages (PA_DTYPE_FP8_E4M3).  The pages name quantised KV only as a
 * later addition; the reading taken: the caches hold codes of the OCP 8-bit
 * floating point format E4M3 in its "fn" form (1 sign bit, 4 exponent bits
 * with bias 7, 3 mantissa bits, subnormals at exponent 0, no infinities,
 * S.1111.111 is NaN, largest finite magnitude 448), and a key_cache entry
 * stands for code * k_scale, a value_cache entry for code * v_scale (one
 * scale per tensor, pa_cache_desc).  q, out, k_new and v_new are bf16.
 * pa_write_kv_cache stores the code nearest to x / scale (the division in
 * IEEE single precision, ties to the even mantissa, magnitudes at or above
 * 448 saturating to 448).  Served by pa_write_kv_cache, pa_decode,
 * pa_forward_decode, pa_decode_noalloc and pa_decode_splitk for head_dim
 * 128, block_size >= 16, 4 or 8 KV heads and at most 8 query heads per KV
 * head; other calls and shapes return PA_ERR_UNSUPPORTED.  Decode converts the codes exactly
 * and multiplies them in fp16 tiles (fp32 accumulation), so q must lie
 * within fp16's range (|q| < 65504).
 */

/* Bits OR'd into *err_word by kernels that meet bad device data. */
#define PA_DEVERR_BLOCK_ID 1
#define PA_DEVERR_CONTEXT_LEN 2
#define PA_DEVERR_SLOT 4
/* A pipeline wait inside a kernel gave up (never expected; the outputs of
 * that call are incomplete and its workspace must be zero-filled again). */
#define PA_DEVERR_TIMEOUT 8
/* pa_decode_shared_prefix: a sequence whose table does not start with the
 * shared prefix pages or whose context is shorter than the prefix. */
#define PA_DEVERR_PREFIX 16

/* Shape of the physical KV cache pool ([teaching] section "First define a
 * simple KV cache layout": [num_blocks, block_size, num_heads, head_dim],
 * with num_heads = the number of KV heads). */
typedef struct pa_cache_desc {
  int32_t num_blocks;
  int32_t block_size;
  int32_t num_kv_heads;
  int32_t head_dim;
  int32_t dtype; /* pa_dtype */
  /* PA_DTYPE_FP8_E4M3 only (ignored for the other dtypes): the values the
   * codes of key_cache / value_cache stand for are code * k_scale and
   * code * v_scale; both finite and > 0. */
  float k_scale;
  float v_scale;
} pa_cache_desc;

/* Version of this ABI (major * 10000 + minor * 100 + patch); 200 added the
 * scales of pa_cache_desc and PA_DTYPE_FP8_E4M3, 300 added pa_prefill. */
int32_t pa_version(void);

/* Static text for a status code. */
const char *pa_status_string(int32_t status);

/* Detail of the last non-OK status returned on the calling host thread. */
const char *pa_last_error_message(void);

/*
 * pa_write_kv_cache -- store the current tokens' K/V rows in their slots.
 *
 * [teaching] section "Writing slots and reading the block table must
 * agree": the Block Manager reserves a slot (physical_block_id,
 * block_offset) for the current token and its K/V are written there before
 * attention reads it as history.  Slot encoding: slot_mapping[i] =
 * physical_block_id * block_size + block_offset; a negative slot means
 * "no token" and is skipped.  For each i with 0 <= slot < num_blocks *
 * block_size, key_cache[slot / block_size, slot % block_size, :, :] =
 * k_new[i] and the same for value_cache / v_new, as a byte copy.  A slot
 * past the pool sets PA_DEVERR_SLOT and is skipped.  num_tokens == 0 is a
 * no-op.  Two tokens with the same slot race (last writer undefined).
 */
pa_status pa_write_kv_cache(const pa_cache_desc *cache, void *key_cache,
                            void *value_cache, const void *k_new,
                            const void *v_new, const int64_t *slot_mapping,
                            int32_t num_tokens, int32_t *err_word,
                            pa_stream_t stream);

/*
 * pa_decode_workspace_bytes -- size of the scratch memory pa_decode needs
 * for these sizes (0 on invalid arguments).
 */
size_t pa_decode_workspace_bytes(const pa_cache_desc *cache, int32_t batch,
                                 int32_t num_q_heads,
                                 int32_t max_blocks_per_seq);

/*
 * pa_decode -- fused paged decode attention.
 *
 * For every sequence b and query head hq, with h = hq / (Hq / Hkv):
 * for t in [0, context_lens[b]): logical_block_id = t / block_size,
 * block_offset = t % block_size, physical_block_id =
 * block_tables[b, logical_block_id] ([teaching] section "From logical
 * token to physical block"); s_t = scale * dot(q[b, hq], K_t[h]); out[b,
 * hq] = sum_t softmax(s)_t * V_t[h] ([route] section "What the attention
 * kernel really does").  One pass over the history with an online softmax
 * (running max and normaliser), the block-table lookup done inside the
 * kernel, no gathered K/V and no stored score vector ([route] sections
 * "The core idea of high-performance PagedAttention" and "What the
 * attention kernel really does").  The decode query attends to exactly the
 * given history, so there is no mask argument ([teaching] section "Where
 * is the attention mask").  context_lens[b] == 0 gives a zero output.
 * Table entries past ceil(context_lens[b] / block_size) are never read.
 *
 * scale is usually 1 / sqrt(head_dim).  workspace: device memory of at
 * least pa_decode_workspace_bytes(...) bytes, 256-byte aligned, ZERO-FILLED
 * before its first use; every call leaves it ready for the next one, so one
 * buffer serves any number of stream-ordered calls.  Calls that overlap on
 * the GPU must not share a workspace.  A call may run as more than one
 * kernel; the later ones are launched with programmatic stream
 * serialisation and wait for the earlier ones.  bf16 caches with 64 or 128
 * query heads per KV head (head_dim 64 or 128, block_size 8..128) are
 * computed on the tensor cores in tiles of 128 tokens (the serving page's
 * section 4.1: many queries per KV page make the work a dense
 * contraction); the result is the same up to rounding.
 */
pa_status pa_decode(const pa_cache_desc *cache, void *out, const void *q,
                    const void *key_cache, const void *value_cache,
                    const int32_t *block_tables, const int32_t *context_lens,
                    int32_t batch, int32_t num_q_heads,
                    int32_t max_blocks_per_seq, float scale, void *workspace,
                    size_t workspace_bytes, int32_t *err_word,
                    pa_stream_t stream);

/*
 * pa_forward_decode -- one decode step: store each sequence's newest token,
 * then attend over its whole history, in one call.
 *
 * The attention backend's decode entry takes the query, the cache pool, the
 * block tables, the context lengths and the slot mapping together ([route]
 * section "FlashAttention, FlashInfer and engineering reuse"): it writes the
 * current token's K/V by slot mapping and reads the history by block table
 * ([teaching] section "How PagedAttention plugs into mini vLLM").
 *
 * k_new, v_new are [batch, num_kv_heads, head_dim]: row b is the newest
 * token of sequence b, at position context_lens[b] - 1 (context_lens
 * include it).  slot_mapping is [batch] int64.  For each b with
 * slot_mapping[b] >= 0 the row is stored exactly as pa_write_kv_cache
 * would, PROVIDED that slot_mapping[b] is the slot the block table gives
 * position context_lens[b] - 1 (physical block block_tables[b, (ctx-1) /
 * block_size], offset (ctx-1) % block_size, both in range); any other
 * non-negative slot sets PA_DEVERR_SLOT, that row is not stored and
 * sequence b's output is written as zeros (its history would be
 * incomplete).  slot_mapping[b] < 0 stores nothing.  Then out = pa_decode of the same
 * arguments, with the stored rows visible.  A cache position that another
 * sequence's visible history also maps (a shared page) must not be written
 * in the same call: the order of that write and that read is unspecified.
 *
 * The result equals pa_write_kv_cache(..., num_tokens = batch) followed by
 * pa_decode whenever every slot passes the check.  Workspace, streams and
 * the remaining errors are those of pa_decode.  The row is stored inside the
 * decode kernel, by the warp that loads the token's page, just before it
 * loads it; for shapes outside the persistent kernel's set (see pa_decode's
 * implementation notes in the library source) a separate write kernel with
 * the same check runs first.
 */
pa_status pa_forward_decode(const pa_cache_desc *cache, void *out, const void *q,
                            void *key_cache, void *value_cache, const void *k_new,
                            const void *v_new, const int64_t *slot_mapping,
                            const int32_t *block_tables, const int32_t *context_lens,
                            int32_t batch, int32_t num_q_heads, int32_t max_blocks_per_seq,
                            float scale, void *workspace, size_t workspace_bytes,
                            int32_t *err_word, pa_stream_t stream);

/*
 * pa_decode_shared_prefix -- pa_decode for a batch whose sequences all start
 * with the same pages (a shared prompt prefix).
 *
 * [serving] section 6 "Prefix caching": requests with a common prefix share
 * its KV pages.  Here the prefix is the first prefix_blocks entries of
 * block_tables row 0, and every sequence's table must start with the same
 * entries and every context_lens[b] must be >= prefix_blocks * block_size.
 * out is the same as pa_decode's (up to rounding); internally the suffix
 * past the prefix is decoded per sequence and the prefix, read by every
 * (sequence, query head) of a KV head, runs as dense tensor-core tiles of
 * 128 rows x 128 prefix tokens (tcgen05) whose epilogue merges the two
 * parts with the running-max rescaling ([route] section "The core idea of
 * high-performance PagedAttention").
 *
 * A sequence whose table or length does not contain the prefix sets
 * PA_DEVERR_PREFIX and its output is zeroed; a bad prefix block id sets
 * PA_DEVERR_BLOCK_ID and zeroes every output.  Shapes: bf16, head_dim 64
 * or 128, query heads per KV head dividing 128, block_size 8..128 (a power
 * of two), prefix_blocks <= 2048; with fewer than 64 query heads per KV
 * head also a shape pa_decode serves with its persistent page-stream kernel
 * (else PA_ERR_UNSUPPORTED).  With 64 or 128 heads per KV head the suffix
 * runs on the tensor cores too.  prefix_blocks == 0 is
 * pa_decode.  workspace: at least pa_decode_shared_prefix_workspace_bytes
 * bytes, 256-byte aligned, zero-filled before first use (as pa_decode's).
 */
size_t pa_decode_shared_prefix_workspace_bytes(const pa_cache_desc *cache, int32_t batch,
                                               int32_t num_q_heads, int32_t max_blocks_per_seq,
                                               int32_t prefix_blocks);
pa_status pa_decode_shared_prefix(const pa_cache_desc *cache, void *out, const void *q,
                                  const void *key_cache, const void *value_cache,
                                  const int32_t *block_tables, const int32_t *context_lens,
                                  int32_t batch, int32_t num_q_heads, int32_t max_blocks_per_seq,
                                  int32_t prefix_blocks, float scale, void *workspace,
                                  size_t workspace_bytes, int32_t *err_word, pa_stream_t stream);

/*
 * pa_prefill -- paged (chunked) prefill attention with the causal mask.
 *
 * [teaching] section "Where is the attention mask": in prefill every prompt
 * token sees itself and the tokens before it; [route] section "decode
 * attention and prefill attention are different": prefill processes a whole
 * prompt, or a chunk of it, at once.  Sequence b brings
 * n_b = query_start[b+1] - query_start[b] new tokens, rows query_start[b] ..
 * query_start[b+1]-1 of q and out.  Their K/V rows must already be stored at
 * their slots (pa_write_kv_cache); the history of sequence b holds
 * context_lens[b] tokens including them, so new token j sits at position
 * p = context_lens[b] - n_b + j and
 *   out[row, hq, :] = sum_{t <= p} softmax_t(scale * q[row, hq, :] . K_t) V_t
 * with K_t, V_t read through row b of block_tables (KV head hq / G).  With
 * context_lens[b] == n_b this is a plain causal prompt prefill; with more it
 * is a later chunk of a chunked prefill.
 *
 * Arrays: q, out [num_tokens, num_q_heads, head_dim] bf16; query_start
 * [batch + 1] int32, non-decreasing, query_start[batch] <= num_tokens;
 * block_tables [batch, max_blocks_per_seq]; context_lens [batch].
 * max_query_len must be >= every n_b: the grid covers that many tokens per
 * sequence.  Rows of out outside every sequence's range are not written.
 *
 * Data errors (flagged in *err_word): a query_start range outside
 * [0, num_tokens] or decreasing sets PA_DEVERR_CONTEXT_LEN and writes none
 * of that sequence's rows; n_b > context_lens[b], n_b > max_query_len or
 * context_lens[b] > max_blocks_per_seq * block_size sets
 * PA_DEVERR_CONTEXT_LEN and zeroes the rows of the sequence that the grid
 * covers; a block id outside [0, num_blocks) among the sequence's first
 * ceil(context_lens[b] / block_size) entries sets PA_DEVERR_BLOCK_ID and
 * zeroes its rows.  A sequence with n_b == 0 is not read.
 *
 * Shapes: bf16, head_dim 64 or 128, query heads per KV head dividing 128,
 * block_size 8..128, max_blocks_per_seq <= 4096 (else PA_ERR_UNSUPPORTED).
 * batch, num_tokens or max_query_len == 0 is a no-op.  The work runs as
 * tcgen05 tiles of 128 (query token, query head) rows x 128 KV tokens with
 * the online softmax; no workspace.
 */
pa_status pa_prefill(const pa_cache_desc *cache, void *out, const void *q,
                     const void *key_cache, const void *value_cache,
                     const int32_t *block_tables, const int32_t *context_lens,
                     const int32_t *query_start, int32_t batch, int32_t num_tokens,
                     int32_t num_q_heads, int32_t max_blocks_per_seq, int32_t max_query_len,
                     float scale, int32_t *err_word, pa_stream_t stream);

/*
 * pa_decode_noalloc -- pa_decode for callers that cannot allocate device
 * memory.
 *
 * The pages have no counterpart to this entry point.  It serves callers of
 * this library that may not call cudaMalloc and so cannot hand pa_decode a
 * workspace: code running as a plugin or callback inside a host engine that
 * owns every byte of device memory through its own pool (an allocation
 * behind the pool's back can fail or break its accounting), and decode loops
 * with hard latency budgets, where cudaMalloc / cudaFree may wait for the
 * whole device to go idle.
 *
 * Arguments, semantics, results and error reporting are those of pa_decode,
 * minus the workspace.  The scratch space is a fixed array of
 * PA_DECODE_NOALLOC_SCRATCH_BYTES bytes of device memory inside libpa; every
 * GPU that loads the library holds it until the process exits.  This call
 * allocates nothing (no cudaMalloc, cudaFree or allocating library routine).
 *
 * - Kernels: those of pa_decode, except that bf16 caches with 64 or 128
 *   query heads per KV head run on the page-stream kernel (16 query heads
 *   per consumer warp) instead of the tensor-core tile kernel, whose scratch
 *   (per-row results of the whole batch) would not fit.
 * - Limit: the call needs the scratch pa_decode needs on those kernels.
 *   That is pa_decode_workspace_bytes(cache, batch, num_q_heads,
 *   max_blocks_per_seq) for every shape except the 64 / 128 query-head
 *   groups above, where it is the page-stream kernel's fixed per-SM
 *   partials, 2 * 192 * num_q_heads * (head_dim + 2) * 4 bytes plus 16
 *   bytes per sequence (about 12.8 MB at 64 heads of head_dim 128).  When it
 *   exceeds PA_DECODE_NOALLOC_SCRATCH_BYTES the call returns
 *   PA_ERR_UNSUPPORTED (see pa_last_error_message) and enqueues no work; use
 *   pa_decode with a workspace for such sizes.
 * - Set-up: the first call on a device looks up the array's device address
 *   for that device (the calling thread's current device) and remembers it.
 *   Make that first call on each device before any stream capture.
 * - Sharing: all calls on a device use the same array, and it keeps what the
 *   last call left in it.  Each call clears the bytes it needs (an
 *   asynchronous memset on `stream`) before the decode kernel runs.  Calls
 *   that overlap on the GPU (other streams, or other host threads without
 *   ordering between them) race on the array and give wrong results; order
 *   them on one stream.
 */
#define PA_DECODE_NOALLOC_SCRATCH_BYTES (16u * 1024u * 1024u)

pa_status pa_decode_noalloc(const pa_cache_desc *cache, void *out,
                            const void *q, const void *key_cache,
                            const void *value_cache,
                            const int32_t *block_tables,
                            const int32_t *context_lens, int32_t batch,
                            int32_t num_q_heads, int32_t max_blocks_per_seq,
                            float scale, int32_t *err_word,
                            pa_stream_t stream);

/*
 * pa_decode_splitk -- per-partition partial results for long contexts.
 *
 * Partition p of sequence b covers tokens [p * partition_tokens,
 * min((p + 1) * partition_tokens, context_lens[b])).  For every
 * non-empty partition and query head, with s_t as in pa_decode:
 *   part_max[b, hq, p] = max_t s_t
 *   part_sum[b, hq, p] = sum_t exp(s_t - part_max)
 *   part_out[b, hq, p, :] = sum_t exp(s_t - part_max) V_t[h] / part_sum
 * i.e. the running maximum and normaliser of the online softmax of [route]
 * section "What the attention kernel really does", kept per partition.
 * Partitions p in [ceil(context_lens[b] / partition_tokens),
 * max_partitions) get part_max = -inf, part_sum = 0, part_out = 0.  A
 * partition that meets a bad block id gets part_sum = -1 (and sets
 * PA_DEVERR_BLOCK_ID); a sequence with a bad context length gets empty
 * partials everywhere (and sets PA_DEVERR_CONTEXT_LEN).
 * Shapes: part_max, part_sum [batch, num_q_heads, max_partitions];
 * part_out [batch, num_q_heads, max_partitions, head_dim]; all fp32.
 * partition_tokens must be a positive multiple of block_size;
 * max_partitions must be >= ceil(max_blocks_per_seq * block_size /
 * partition_tokens).  No workspace: on the shapes of pa_decode's persistent
 * page-stream kernel, when partition_tokens is a multiple of its page (16
 * tokens for bf16 caches of 8-token blocks, 32 for FP8 caches, else at most
 * block_size), the partitions of all sequences form one stream cut into one
 * range per SM at partition boundaries, so each partition is computed whole
 * by one CTA and written once; other shapes and partition sizes run one CTA
 * per (partition, KV head, head tile) and allow at most 1024 blocks per
 * partition; FP8 caches need the page stream (PA_ERR_UNSUPPORTED otherwise).
 */
pa_status pa_decode_splitk(const pa_cache_desc *cache, const void *q,
                           const void *key_cache, const void *value_cache,
                           const int32_t *block_tables,
                           const int32_t *context_lens, int32_t batch,
                           int32_t num_q_heads, int32_t max_blocks_per_seq,
                           float scale, int32_t partition_tokens,
                           int32_t max_partitions, float *part_max,
                           float *part_sum, float *part_out, int32_t *err_word,
                           pa_stream_t stream);

/*
 * pa_reduce -- merge per-partition partials into the output.
 *
 * For each (b, hq), over partitions p < min(ceil(context_lens[b] /
 * partition_tokens), max_partitions) with part_sum > 0:
 * M = max_p part_max, w_p = part_sum * exp(part_max - M),
 * out[b, hq, :] = sum_p w_p part_out[p] / sum_p w_p -- the rescaling rule
 * of the online softmax applied across partitions.  Zero output when no
 * partition is non-empty or when any of them has part_sum < 0 (a bad
 * block id upstream).  A context length < 0 or past max_partitions *
 * partition_tokens sets PA_DEVERR_CONTEXT_LEN and gives zeros.  out has
 * dtype `out_dtype`.  head_dim a multiple of 4, at most 1024; up to about
 * 56000 partitions (else PA_ERR_UNSUPPORTED).
 */
pa_status pa_reduce(void *out, const float *part_max, const float *part_sum,
                    const float *part_out, const int32_t *context_lens,
                    int32_t batch, int32_t num_q_heads, int32_t head_dim,
                    int32_t partition_tokens, int32_t max_partitions,
                    int32_t out_dtype, int32_t *err_word, pa_stream_t stream);

#ifdef __cplusplus
} /* extern "C" */
#endif

#endif /* PA_H_ */
