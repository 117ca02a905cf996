// reduce.cu -- merge of per-partition partials (pa_reduce).
//
// Each partition p of a sequence carries the running maximum m_p, the
// normaliser l_p and the normalised partial output o_p of the online
// softmax (page "From correct to faster: the PagedAttention optimisation
// route", section "What the attention kernel really does").  Merging uses the
// same rescaling rule across partitions:
//   M = max_p m_p,  w_p = l_p * exp(m_p - M),  out = sum_p w_p o_p / sum_p w_p.
//
// One CTA per (sequence, query head).  The work is a read of the row's
// partials (max_partitions x head_dim fp32, 128 KB for 256 partitions of
// head_dim 128), so it is laid out for memory-level parallelism: every
// thread loads partition maxima and normalisers at once and the CTA reduces
// them in shared memory; then the threads split into groups of head_dim / 4
// (one 16-byte column each), group g summing partitions g, g + G, ... with
// independent loads in flight, and the groups' sums are added in shared
// memory.
#include <math.h>

#include "pa_common.cuh"
#include "pa_launch.h"

namespace pa {
namespace {

template <typename TO>
__global__ void __launch_bounds__(kReduceThreads)
reduce_kernel(void *__restrict__ out, const float *__restrict__ part_max,
              const float *__restrict__ part_sum,
              const float *__restrict__ part_out,
              const int32_t *__restrict__ context_lens, int32_t num_q_heads,
              int32_t head_dim, int32_t partition_tokens,
              int32_t max_partitions, int32_t *err_word) {
  extern __shared__ __align__(16) float smem[];
  // [max_partitions] weights, then [groups][head_dim] group sums
  float *wts = smem;
  float4 *gsum = reinterpret_cast<float4 *>(smem + ((max_partitions + 3) & ~3));
  __shared__ float red_m[kReduceThreads / 32];
  __shared__ float red_w[kReduceThreads / 32];
  __shared__ int red_bad[kReduceThreads / 32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t bh = blockIdx.x;
  const int64_t b = bh / num_q_heads;
  const int ctx = context_lens[b];
  const bool bad_len =
      ctx < 0 || (int64_t)ctx > (int64_t)max_partitions * partition_tokens;
  if (bad_len && (bh % num_q_heads) == 0 && tid == 0)
    set_error(err_word, PA_DEVERR_CONTEXT_LEN);
  const int np = bad_len ? 0 : (ctx + partition_tokens - 1) / partition_tokens;
  const float *pm = part_max + bh * max_partitions;
  const float *pl = part_sum + bh * max_partitions;

  // 1. M = max over non-empty partitions, and whether any partition is bad
  float m = -INFINITY;
  int bad = 0;
  for (int p = tid; p < np; p += kReduceThreads) {
    const float l = pl[p];
    bad |= l < 0.f;
    if (l > 0.f) m = fmaxf(m, pm[p]);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    bad |= __shfl_xor_sync(0xffffffffu, bad, o);
  }
  if (lane == 0) {
    red_m[warp] = m;
    red_bad[warp] = bad;
  }
  __syncthreads();
  float M = -INFINITY;
  bad = 0;
  for (int w = 0; w < kReduceThreads / 32; ++w) {
    M = fmaxf(M, red_m[w]);
    bad |= red_bad[w];
  }
  const bool zero = bad || M == -INFINITY;

  // 2. the weights w_p = l_p exp(m_p - M) and their sum
  float wsum = 0.f;
  for (int p = tid; p < np; p += kReduceThreads) {
    const float l = pl[p];
    const float w = (!zero && l > 0.f) ? l * exp2f((pm[p] - M) * kLog2e) : 0.f;
    wts[p] = w;
    wsum += w;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) wsum += __shfl_xor_sync(0xffffffffu, wsum, o);
  if (lane == 0) red_w[warp] = wsum;
  __syncthreads();
  float W = 0.f;
  for (int w = 0; w < kReduceThreads / 32; ++w) W += red_w[w];

  // 3. sum_p w_p o_p: group g takes partitions g, g + G, ...; a thread one
  //    16-byte column of head_dim
  const int cols = head_dim / 4;
  const int groups = kReduceThreads / cols;
  const int g = tid / cols, c = tid % cols;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  if (g < groups && !zero) {
    const float4 *po = reinterpret_cast<const float4 *>(part_out + bh * max_partitions * head_dim);
    int p = g;
    // four partitions per step: their loads are in flight together
    for (; p + 3 * groups < np; p += 4 * groups) {
      float4 o[4];
      float w[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        o[u] = __ldg(po + (int64_t)(p + u * groups) * cols + c);
        w[u] = wts[p + u * groups];
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        acc.x += w[u] * o[u].x;
        acc.y += w[u] * o[u].y;
        acc.z += w[u] * o[u].z;
        acc.w += w[u] * o[u].w;
      }
    }
    for (; p < np; p += groups) {
      const float4 o = __ldg(po + (int64_t)p * cols + c);
      const float w = wts[p];
      acc.x += w * o.x;
      acc.y += w * o.y;
      acc.z += w * o.z;
      acc.w += w * o.w;
    }
  }
  if (g < groups) gsum[g * cols + c] = acc;
  __syncthreads();
  if (tid < cols) {
    float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int q = 0; q < groups; ++q) {
      const float4 v = gsum[q * cols + tid];
      s.x += v.x;
      s.y += v.y;
      s.z += v.z;
      s.w += v.w;
    }
    const float inv = zero ? 0.f : 1.f / W;
    s.x *= inv;
    s.y *= inv;
    s.z *= inv;
    s.w *= inv;
    Elem<TO>::store4(out, bh * head_dim + tid * 4, s);
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
  if (head_dim % 4 != 0 || head_dim / 4 > kReduceThreads) return cudaErrorInvalidValue;
  const int groups = kReduceThreads / (head_dim / 4);
  const size_t smem = (size_t)((max_partitions + 3) & ~3) * sizeof(float) +
                      (size_t)groups * head_dim * sizeof(float);
  if (smem > 227 * 1024) return cudaErrorInvalidValue;
  if (smem > 48 * 1024) {
    const cudaError_t e =
        out_dtype == PA_DTYPE_BF16
            ? cudaFuncSetAttribute(reduce_kernel<__nv_bfloat16>,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)
            : cudaFuncSetAttribute(reduce_kernel<float>,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  if (out_dtype == PA_DTYPE_BF16)
    reduce_kernel<__nv_bfloat16><<<(unsigned)blocks, kReduceThreads, smem, stream>>>(
        out, part_max, part_sum, part_out, context_lens, num_q_heads, head_dim,
        partition_tokens, max_partitions, err_word);
  else
    reduce_kernel<float><<<(unsigned)blocks, kReduceThreads, smem, stream>>>(
        out, part_max, part_sum, part_out, context_lens, num_q_heads, head_dim,
        partition_tokens, max_partitions, err_word);
  return cudaGetLastError();
}

}  // namespace pa
