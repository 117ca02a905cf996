// write_kv.cu -- cache write by slot mapping.
//
// Page "Implementing teaching PagedAttention: reading the historical KV cache
// from the block table", section "Writing slots and reading the block table
// must agree": the current token's K/V rows go to the slot the Block Manager
// reserved for it, (physical_block_id, block_offset), encoded here as
// slot = physical_block_id * block_size + block_offset.
//
// One CTA per (new token, row slice); each thread moves 16-byte vectors, so a
// row (num_kv_heads * head_dim elements) is copied with coalesced loads and
// stores.  Bit-exact: the bytes are moved, never converted.
#include "pa_common.cuh"
#include "pa_launch.h"

namespace pa {
namespace {

// Whether token `token`'s slot may be written: inside the pool and, in a
// decode step (block_tables set), the slot the table gives position ctx - 1.
__device__ __forceinline__ bool slot_ok(int64_t token, int64_t slot, int64_t num_slots,
                                        const int32_t *__restrict__ block_tables,
                                        const int32_t *__restrict__ context_lens,
                                        int32_t max_blocks, int32_t block_size,
                                        int32_t num_blocks) {
  bool ok = slot < num_slots;
  if (ok && block_tables != nullptr) {
    const int32_t ctx = context_lens[token];
    ok = ctx > 0 && (int64_t)ctx <= (int64_t)max_blocks * block_size;
    if (ok) {
      const int32_t pos = ctx - 1;
      const int32_t pb = block_tables[token * (int64_t)max_blocks + pos / block_size];
      ok = pb >= 0 && pb < num_blocks && slot == (int64_t)pb * block_size + pos % block_size;
    }
  }
  return ok;
}

__global__ void __launch_bounds__(128)
write_kv_kernel(uint4 *__restrict__ key_cache, uint4 *__restrict__ value_cache,
                const uint4 *__restrict__ k_new, const uint4 *__restrict__ v_new,
                const int64_t *__restrict__ slot_mapping, int64_t num_slots,
                int64_t row_vecs, int32_t *err_word,
                const int32_t *__restrict__ block_tables,
                const int32_t *__restrict__ context_lens, int32_t max_blocks,
                int32_t block_size, int32_t num_blocks) {
  // The decode kernel that usually follows waits for this grid to finish
  // (griddepcontrol.wait) before it reads anything; letting it launch now
  // overlaps its start-up with this copy.
  asm volatile("griddepcontrol.launch_dependents;");
  const int64_t token = blockIdx.x;
  const int64_t slot = slot_mapping[token];
  if (slot < 0) return;
  // decode step: token b is sequence b's newest, at position ctx - 1; only
  // the slot the block table gives that position is accepted
  const bool ok = slot_ok(token, slot, num_slots, block_tables, context_lens, max_blocks,
                          block_size, num_blocks);
  if (!ok) {
    if (blockIdx.y == 0 && threadIdx.x == 0) set_error(err_word, PA_DEVERR_SLOT);
    return;
  }
  const int64_t src = token * row_vecs;
  const int64_t dst = slot * row_vecs;
  for (int64_t i = blockIdx.y * (int64_t)blockDim.x + threadIdx.x; i < row_vecs;
       i += (int64_t)gridDim.y * blockDim.x) {
    key_cache[dst + i] = k_new[src + i];
    value_cache[dst + i] = v_new[src + i];
  }
}

// FP8 pages: the new rows arrive as bf16 (row_elems per token); each group
// of 16 elements is divided by its tensor's scale and quantised to E4M3
// codes (bf16x16_to_e4m3), one 16-byte store of codes per group.
__global__ void __launch_bounds__(128)
write_kv_fp8_kernel(uint4 *__restrict__ key_cache, uint4 *__restrict__ value_cache,
                    const uint4 *__restrict__ k_new, const uint4 *__restrict__ v_new,
                    const int64_t *__restrict__ slot_mapping, int64_t num_slots,
                    int64_t row_groups, float k_scale, float v_scale, int32_t *err_word,
                    const int32_t *__restrict__ block_tables,
                    const int32_t *__restrict__ context_lens, int32_t max_blocks,
                    int32_t block_size, int32_t num_blocks) {
  asm volatile("griddepcontrol.launch_dependents;");
  const int64_t token = blockIdx.x;
  const int64_t slot = slot_mapping[token];
  if (slot < 0) return;
  if (!slot_ok(token, slot, num_slots, block_tables, context_lens, max_blocks, block_size,
               num_blocks)) {
    if (blockIdx.y == 0 && threadIdx.x == 0) set_error(err_word, PA_DEVERR_SLOT);
    return;
  }
  for (int64_t i = blockIdx.y * (int64_t)blockDim.x + threadIdx.x; i < row_groups;
       i += (int64_t)gridDim.y * blockDim.x) {
    const int64_t src = (token * row_groups + i) * 2;  // two 16-byte bf16 vectors per group
    const int64_t dst = slot * row_groups + i;
    key_cache[dst] = bf16x16_to_e4m3(k_new[src], k_new[src + 1], k_scale);
    value_cache[dst] = bf16x16_to_e4m3(v_new[src], v_new[src + 1], v_scale);
  }
}

}  // namespace

cudaError_t launch_write_kv(int32_t dtype, int32_t block_size,
                            int32_t num_blocks, int64_t row_bytes,
                            void *key_cache, void *value_cache,
                            const void *k_new, const void *v_new,
                            const int64_t *slot_mapping, int32_t num_tokens,
                            int32_t *err_word, cudaStream_t stream,
                            const int32_t *block_tables, const int32_t *context_lens,
                            int32_t max_blocks, float k_scale, float v_scale) {
  if (num_tokens == 0) return cudaSuccess;
  if (dtype == PA_DTYPE_FP8_E4M3) {
    // row_bytes: one cache row of codes (= elements)
    const int64_t groups = row_bytes / 16;
    const int threads = 128;
    int64_t gy = (groups + threads - 1) / threads;
    if (gy > 64) gy = 64;
    dim3 grid((unsigned)num_tokens, (unsigned)gy);
    write_kv_fp8_kernel<<<grid, threads, 0, stream>>>(
        static_cast<uint4 *>(key_cache), static_cast<uint4 *>(value_cache),
        static_cast<const uint4 *>(k_new), static_cast<const uint4 *>(v_new), slot_mapping,
        (int64_t)num_blocks * block_size, groups, k_scale, v_scale, err_word, block_tables,
        context_lens, max_blocks, block_size, num_blocks);
    return cudaGetLastError();
  }
  const int64_t row_vecs = row_bytes / 16;
  const int threads = 128;
  int64_t gy = (row_vecs + threads - 1) / threads;
  if (gy > 64) gy = 64;
  dim3 grid((unsigned)num_tokens, (unsigned)gy);
  write_kv_kernel<<<grid, threads, 0, stream>>>(
      static_cast<uint4 *>(key_cache), static_cast<uint4 *>(value_cache),
      static_cast<const uint4 *>(k_new), static_cast<const uint4 *>(v_new),
      slot_mapping, (int64_t)num_blocks * block_size, row_vecs, err_word, block_tables,
      context_lens, max_blocks, block_size, num_blocks);
  return cudaGetLastError();
}

}  // namespace pa
