// reduce.cu -- merge of per-partition partials (pa_reduce).
//
// Each partition p of a sequence carries the running maximum m_p, the
// normaliser l_p and the normalised partial output o_p of the online
// softmax (page "From correct to faster: the PagedAttention optimisation
// route", section "What the attention kernel really does").  Merging uses the
// same rescaling rule across partitions:
//   M = max_p m_p,  w_p = l_p * exp(m_p - M),  out = sum_p w_p o_p / sum_p w_p.
// One CTA per (sequence, query head); thread d handles output element d.
#include <math.h>

#include "pa_common.cuh"
#include "pa_launch.h"

namespace pa {
namespace {

template <typename TO>
__global__ void __launch_bounds__(128)
reduce_kernel(void *__restrict__ out, const float *__restrict__ part_max,
              const float *__restrict__ part_sum,
              const float *__restrict__ part_out,
              const int32_t *__restrict__ context_lens, int32_t num_q_heads,
              int32_t head_dim, int32_t partition_tokens,
              int32_t max_partitions, int32_t *err_word) {
  const int64_t bh = blockIdx.x;
  const int64_t b = bh / num_q_heads;
  const int ctx = context_lens[b];
  const bool bad_len =
      ctx < 0 || (int64_t)ctx > (int64_t)max_partitions * partition_tokens;
  if (bad_len && (bh % num_q_heads) == 0 && threadIdx.x == 0)
    set_error(err_word, PA_DEVERR_CONTEXT_LEN);
  const int np = bad_len ? 0 : (ctx + partition_tokens - 1) / partition_tokens;
  const float *pm = part_max + bh * max_partitions;
  const float *pl = part_sum + bh * max_partitions;
  float M = -INFINITY;
  bool any_bad = false;
  for (int p = 0; p < np; ++p) {
    const float l = pl[p];
    if (l < 0.f) any_bad = true;
    if (l > 0.f) M = fmaxf(M, pm[p]);
  }
  const bool zero = any_bad || M == -INFINITY;
  for (int d = threadIdx.x; d < head_dim; d += blockDim.x) {
    float o = 0.f;
    if (!zero) {
      float W = 0.f, O = 0.f;
      for (int p = 0; p < np; ++p) {
        const float l = pl[p];
        if (!(l > 0.f)) continue;
        const float w = l * exp2f((pm[p] - M) * kLog2e);
        W += w;
        O += w * part_out[(bh * max_partitions + p) * head_dim + d];
      }
      o = O / W;
    }
    Elem<TO>::store1(out, bh * head_dim + d, o);
  }
}

}  // namespace

cudaError_t launch_reduce(void *out, const float *part_max,
                          const float *part_sum, const float *part_out,
                          const int32_t *context_lens, int32_t batch,
                          int32_t num_q_heads, int32_t head_dim,
                          int32_t partition_tokens, int32_t max_partitions,
                          int32_t out_dtype, int32_t *err_word,
                          cudaStream_t stream) {
  const int64_t blocks = (int64_t)batch * num_q_heads;
  if (blocks == 0) return cudaSuccess;
  if (out_dtype == PA_DTYPE_BF16)
    reduce_kernel<__nv_bfloat16><<<(unsigned)blocks, 128, 0, stream>>>(
        out, part_max, part_sum, part_out, context_lens, num_q_heads, head_dim,
        partition_tokens, max_partitions, err_word);
  else
    reduce_kernel<float><<<(unsigned)blocks, 128, 0, stream>>>(
        out, part_max, part_sum, part_out, context_lens, num_q_heads, head_dim,
        partition_tokens, max_partitions, err_word);
  return cudaGetLastError();
}

}  // namespace pa
