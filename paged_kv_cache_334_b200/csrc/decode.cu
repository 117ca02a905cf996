// decode.cu -- fused paged decode attention (pa_decode, pa_decode_splitk).
//
// What is computed (page "From correct to faster: the PagedAttention
// optimisation route", sections "The core idea of high-performance
// PagedAttention" and "What the attention kernel really does"): for each
// history token the kernel itself maps token -> logical block -> physical
// block -> offset -> K/V address (page "Implementing teaching PagedAttention:
// reading the historical KV cache from the block table", section "From
// logical token to physical block"), scores it against the query, keeps a
// running maximum and normaliser (online softmax) and accumulates the
// weighted V rows -- one pass, no gathered K/V, no stored score vector.
//
// Work decomposition: one CTA per (partition of part_tokens history tokens,
// KV head, sequence) and a tile of up to GT query heads of that KV head's
// GQA group, so one K/V read serves all of them (page "Operators and
// compilers: inference attention and KV kernels", section 7 on MQA / GQA).
// Inside the CTA each warp takes iterations of TPI consecutive tokens; a
// token row of head_dim elements is read by LPT lanes with 16-byte
// streaming loads (adjacent lanes read adjacent bytes).  Per-(token, head)
// dot products are reduced with a transposed butterfly, the online softmax
// bookkeeping runs on one lane per (token, head), and the warps' (max,
// normaliser, accumulator) states are merged through shared memory.
//
// A sequence with one partition writes `out` directly.  With several
// partitions each CTA writes a partial (max, sum, normalised output); in
// pa_decode the last CTA of the (sequence, KV head, head tile) to finish --
// found with an atomic counter, no waiting -- merges them with the same
// rescaling rule and resets the counter.  pa_decode_splitk stops at the
// partials (merged later by pa_reduce).
//
// Scores are kept in log2 units (q pre-scaled by scale * log2(e)) so the
// exponentials are exp2; partial maxima are stored in natural units.
#include <math.h>

#include "pa_common.cuh"
#include "pa_launch.h"

namespace pa {
namespace {

constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;
constexpr int kMaxPartPages = 1024;

struct KParams {
  const void *q;
  void *out;
  const void *key_cache;
  const void *value_cache;
  const int32_t *block_tables;
  const int32_t *context_lens;
  float *part_max;
  float *part_sum;
  float *part_out;
  int32_t *counters;
  int32_t *err_word;
  const int64_t *slot_mapping;
  int32_t num_blocks, block_size, log2_block_size, num_kv_heads;
  int32_t num_q_heads, group, head_tiles, max_blocks;
  int32_t part_tokens, max_parts;
  float scale_log2;
  int32_t merge;
};

template <typename T, int D, int GT>
struct Cfg {
  static constexpr int EPV = Elem<T>::kPerVec;  // elements per 16-byte vector
  static constexpr int LPT = D / EPV;           // lanes per token row
  static constexpr int TPW = 32 / LPT;          // tokens per warp-wide load
  static constexpr int U = (GT >= 8) ? 2 : 4;   // loads per lane per tensor
  static constexpr int TPI = U * TPW;           // tokens per warp iteration
  static constexpr int N = U * GT;              // partial dots per lane
  static constexpr int NV = (N >= LPT) ? N / LPT : 1;
  static constexpr int E = TPI * GT;            // (token, head) entries
  static constexpr int EPL = (E + 31) / 32;     // entries per lane
  static_assert(LPT >= 1 && LPT <= 32 && (32 % LPT) == 0, "row split");
  static_assert((32 % GT) == 0, "head tile must divide the warp");
  static_assert(NV >= 1 && EPL >= 1, "derived sizes");
};

template <typename T, int D, int GT>
__global__ void __launch_bounds__(kThreads, (GT >= 8) ? 2 : 4)
    decode_kernel(const KParams p) {
  using C = Cfg<T, D, GT>;
  __shared__ int32_t s_pages[kMaxPartPages];
  __shared__ float s_scores[kWarps][C::E];
  __shared__ float s_alpha[kWarps][GT];
  __shared__ float s_m[kWarps][GT];
  __shared__ float s_l[kWarps][GT];
  __shared__ float s_acc[kWarps][GT][D];
  __shared__ int s_last;

  const int part = blockIdx.x;
  const int h = blockIdx.y / p.head_tiles;
  const int tile = blockIdx.y % p.head_tiles;
  const int b = blockIdx.z;
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int hq0 = h * p.group + tile * GT;
  const int nheads = min(GT, p.group - tile * GT);

  const int ctx = p.context_lens[b];
  const bool bad_len =
      ctx < 0 || (int64_t)ctx > (int64_t)p.max_blocks * p.block_size;
  const int nparts = bad_len ? 0 : (ctx + p.part_tokens - 1) / p.part_tokens;

  if (part >= nparts) {
    if (bad_len && part == 0 && blockIdx.y == 0 && tid == 0)
      set_error(p.err_word, PA_DEVERR_CONTEXT_LEN);
    if (p.merge) {
      if (part == 0) {
        for (int x = tid; x < nheads * D; x += kThreads)
          Elem<T>::store1(p.out, ((int64_t)b * p.num_q_heads + hq0) * D + x, 0.f);
      }
    } else {
      for (int x = tid; x < nheads * D; x += kThreads) {
        const int g = x / D, d = x % D;
        const int64_t ix = ((int64_t)b * p.num_q_heads + hq0 + g) * p.max_parts + part;
        if (d == 0) {
          p.part_max[ix] = -INFINITY;
          p.part_sum[ix] = 0.f;
        }
        p.part_out[ix * D + d] = 0.f;
      }
    }
    return;
  }

  const int t_begin = part * p.part_tokens;
  const int t_end = min(t_begin + p.part_tokens, ctx);
  const int ntok = t_end - t_begin;
  const int lb0 = t_begin >> p.log2_block_size;
  const int npages = ((t_end - 1) >> p.log2_block_size) - lb0 + 1;

  // Block-table slice of this partition, validated once.
  int bad_block = 0;
  for (int i = tid; i < npages; i += kThreads) {
    int pb = p.block_tables[(int64_t)b * p.max_blocks + lb0 + i];
    if (pb < 0 || pb >= p.num_blocks) {
      bad_block = 1;
      pb = 0;
    }
    s_pages[i] = pb;
  }
  // Fused write (checked by the write kernel that ran before): the partition
  // holding the new token fails when its slot is not the table's.
  bool bad_slot = false;
  if (p.slot_mapping != nullptr && t_end == ctx) {
    const int64_t slot = p.slot_mapping[b];
    if (slot >= 0) {
      const int pos = ctx - 1;
      const int pbl = p.block_tables[(int64_t)b * p.max_blocks + (pos >> p.log2_block_size)];
      bad_slot = pbl < 0 || pbl >= p.num_blocks ||
                 slot != (int64_t)pbl * p.block_size + (pos & (p.block_size - 1));
    }
  }
  bad_block = __syncthreads_or(bad_block);
  const int bad = bad_block || bad_slot;

  const int tg = lane / C::LPT;  // token slot of this lane in a warp load
  const int j = lane % C::LPT;   // 16-byte chunk of the row this lane reads
  // Lane `lane` keeps the softmax state (m_run, l_run) of head lane % GT.

  float m_run = -INFINITY;
  float l_run = 0.f;
  float acc[GT][C::EPV];
#pragma unroll
  for (int g = 0; g < GT; ++g)
#pragma unroll
    for (int e = 0; e < C::EPV; ++e) acc[g][e] = 0.f;

  if (!bad) {
    float qf[GT][C::EPV];
#pragma unroll
    for (int g = 0; g < GT; ++g) {
      if (g < nheads) {
        const T *qp = static_cast<const T *>(p.q) +
                      ((int64_t)b * p.num_q_heads + hq0 + g) * D + j * C::EPV;
        uint4 raw = *reinterpret_cast<const uint4 *>(qp);
        Elem<T>::widen(raw, qf[g]);
#pragma unroll
        for (int e = 0; e < C::EPV; ++e) qf[g][e] *= p.scale_log2;
      } else {
#pragma unroll
        for (int e = 0; e < C::EPV; ++e) qf[g][e] = 0.f;
      }
    }

    const T *kbase = static_cast<const T *>(p.key_cache);
    const T *vbase = static_cast<const T *>(p.value_cache);
    const int64_t row_elems = (int64_t)p.num_kv_heads * D;
    const int64_t head_off = (int64_t)h * D + j * C::EPV;
    const int n_iter = (ntok + C::TPI - 1) / C::TPI;

    for (int it = warp; it < n_iter; it += kWarps) {
      uint4 kr[C::U], vr[C::U];
#pragma unroll
      for (int u = 0; u < C::U; ++u) {
        const int tl = it * C::TPI + u * C::TPW + tg;
        if (tl < ntok) {
          const int t = t_begin + tl;
          const int pb = s_pages[(t >> p.log2_block_size) - lb0];
          const int off = t & (p.block_size - 1);
          const int64_t e = ((int64_t)pb * p.block_size + off) * row_elems + head_off;
          kr[u] = ld_stream16(kbase + e);
          vr[u] = ld_stream16(vbase + e);
        } else {
          kr[u] = make_uint4(0u, 0u, 0u, 0u);
          vr[u] = make_uint4(0u, 0u, 0u, 0u);
        }
      }

      // Partial dot products of this lane's row chunk, all (token, head).
      float sc[C::N];
#pragma unroll
      for (int u = 0; u < C::U; ++u) {
        float kf[C::EPV];
        Elem<T>::widen(kr[u], kf);
#pragma unroll
        for (int g = 0; g < GT; ++g) {
          float dot = 0.f;
#pragma unroll
          for (int e = 0; e < C::EPV; ++e) dot = fmaf(qf[g][e], kf[e], dot);
          sc[u * GT + g] = dot;
        }
      }
      Butterfly<C::N, C::LPT / 2>::run(sc, lane);

      // Publish the reduced scores, masked past the partition's end.
      if constexpr (C::N >= C::LPT) {
#pragma unroll
        for (int i = 0; i < C::NV; ++i) {
          const int idx = j * C::NV + i;
          const int u = idx / GT, g = idx % GT;
          const int tloc = u * C::TPW + tg;
          const bool valid = it * C::TPI + tloc < ntok;
          s_scores[warp][tloc * GT + g] = valid ? sc[i] : -INFINITY;
        }
      } else {
        constexpr int R = C::LPT / C::N;
        if ((j % R) == 0) {
          const int idx = j / R;
          const int u = idx / GT, g = idx % GT;
          const int tloc = u * C::TPW + tg;
          const bool valid = it * C::TPI + tloc < ntok;
          s_scores[warp][tloc * GT + g] = valid ? sc[0] : -INFINITY;
        }
      }
      __syncwarp();

      // Online softmax: entries e = lane + 32*k all belong to head g_lane.
      float sv[C::EPL];
      float tmax = -INFINITY;
#pragma unroll
      for (int k = 0; k < C::EPL; ++k) {
        const int e = lane + 32 * k;
        sv[k] = (e < C::E) ? s_scores[warp][e] : -INFINITY;
        tmax = fmaxf(tmax, sv[k]);
      }
#pragma unroll
      for (int mask = GT; mask < 32; mask <<= 1)
        tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, mask));
      const float m_new = fmaxf(m_run, tmax);
      const float alpha = exp2f(m_run - m_new);
      m_run = m_new;
      float psum = 0.f;
#pragma unroll
      for (int k = 0; k < C::EPL; ++k) {
        const int e = lane + 32 * k;
        const float pe = exp2f(sv[k] - m_new);
        psum += pe;
        if (e < C::E) s_scores[warp][e] = pe;
      }
      l_run = l_run * alpha + psum;
      if (lane < GT) s_alpha[warp][lane] = alpha;
      __syncwarp();

      // Rescale and accumulate the weighted V rows.
#pragma unroll
      for (int g = 0; g < GT; ++g) {
        const float a = s_alpha[warp][g];
#pragma unroll
        for (int e = 0; e < C::EPV; ++e) acc[g][e] *= a;
      }
#pragma unroll
      for (int u = 0; u < C::U; ++u) {
        const int tloc = u * C::TPW + tg;
        float vf[C::EPV];
        Elem<T>::widen(vr[u], vf);
#pragma unroll
        for (int g = 0; g < GT; ++g) {
          const float pg = s_scores[warp][tloc * GT + g];
#pragma unroll
          for (int e = 0; e < C::EPV; ++e) acc[g][e] = fmaf(pg, vf[e], acc[g][e]);
        }
      }
      __syncwarp();
    }
  }

  // Warp state -> shared memory.
#pragma unroll
  for (int mask = C::LPT; mask < 32; mask <<= 1)
#pragma unroll
    for (int g = 0; g < GT; ++g)
#pragma unroll
      for (int e = 0; e < C::EPV; ++e)
        acc[g][e] += __shfl_xor_sync(0xffffffffu, acc[g][e], mask);
#pragma unroll
  for (int mask = GT; mask < 32; mask <<= 1)
    l_run += __shfl_xor_sync(0xffffffffu, l_run, mask);
  if (lane < GT) {
    s_m[warp][lane] = m_run;
    s_l[warp][lane] = l_run;
  }
  if (tg == 0) {
#pragma unroll
    for (int g = 0; g < GT; ++g)
#pragma unroll
      for (int e = 0; e < C::EPV; ++e) s_acc[warp][g][j * C::EPV + e] = acc[g][e];
  }
  __syncthreads();

  const bool direct = p.merge && nparts == 1;
  for (int x = tid; x < nheads * D; x += kThreads) {
    const int g = x / D, d = x % D;
    const int64_t hrow = (int64_t)b * p.num_q_heads + hq0 + g;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, s_m[w][g]);
    float L = 0.f, O = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const float f = exp2f(s_m[w][g] - M);
      L += s_l[w][g] * f;
      O += s_acc[w][g][d] * f;
    }
    const float o = bad ? 0.f : O / L;
    if (direct) {
      Elem<T>::store1(p.out, hrow * D + d, o);
    } else {
      const int64_t ix = hrow * p.max_parts + part;
      if (d == 0) {
        p.part_max[ix] = bad ? -INFINITY : M * kLn2;
        p.part_sum[ix] = bad ? -1.f : L;
      }
      p.part_out[ix * D + d] = o;
    }
  }
  if (bad_block && tid == 0) set_error(p.err_word, PA_DEVERR_BLOCK_ID);
  if (bad_slot && tid == 0) set_error(p.err_word, PA_DEVERR_SLOT);
  if (!p.merge || direct) return;

  // Last CTA of this (sequence, KV head, head tile) merges the partials.
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    int32_t *cnt = p.counters + ((int64_t)b * p.num_kv_heads + h) * p.head_tiles + tile;
    const int prev = atomicAdd(cnt, 1);
    s_last = (prev == nparts - 1);
    if (s_last) atomicExch(cnt, 0);
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  for (int x = tid; x < nheads * D; x += kThreads) {
    const int g = x / D, d = x % D;
    const int64_t hrow = (int64_t)b * p.num_q_heads + hq0 + g;
    const int64_t base = hrow * p.max_parts;
    float M = -INFINITY;
    bool any_bad = false;
    for (int pp = 0; pp < nparts; ++pp) {
      const float l = __ldcg(p.part_sum + base + pp);
      if (l < 0.f) any_bad = true;
      M = fmaxf(M, __ldcg(p.part_max + base + pp));
    }
    float o = 0.f;
    if (!any_bad) {
      float W = 0.f, O = 0.f;
      for (int pp = 0; pp < nparts; ++pp) {
        const float w = __ldcg(p.part_sum + base + pp) *
                        exp2f((__ldcg(p.part_max + base + pp) - M) * kLog2e);
        W += w;
        O += w * __ldcg(p.part_out + (base + pp) * D + d);
      }
      o = O / W;
    }
    Elem<T>::store1(p.out, hrow * D + d, o);
  }
}

template <typename T, int D>
cudaError_t launch_dtype_dim(const KParams &kp, int gt, dim3 grid, cudaStream_t s) {
  switch (gt) {
    case 1: decode_kernel<T, D, 1><<<grid, kThreads, 0, s>>>(kp); break;
    case 2: decode_kernel<T, D, 2><<<grid, kThreads, 0, s>>>(kp); break;
    case 4: decode_kernel<T, D, 4><<<grid, kThreads, 0, s>>>(kp); break;
    case 8: decode_kernel<T, D, 8><<<grid, kThreads, 0, s>>>(kp); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace

int decode_head_tile(int group) {
  if (group <= 1) return 1;
  if (group == 2) return 2;
  if (group <= 4) return 4;
  return 8;
}

cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t stream) {
  KParams kp;
  kp.q = a.q;
  kp.out = a.out;
  kp.key_cache = a.key_cache;
  kp.value_cache = a.value_cache;
  kp.block_tables = a.block_tables;
  kp.context_lens = a.context_lens;
  kp.part_max = a.part_max;
  kp.part_sum = a.part_sum;
  kp.part_out = a.part_out;
  kp.counters = a.counters;
  kp.err_word = a.err_word;
  kp.slot_mapping = a.slot_mapping;
  kp.num_blocks = a.num_blocks;
  kp.block_size = a.block_size;
  int lg = 0;
  while ((1 << lg) < a.block_size) ++lg;
  kp.log2_block_size = lg;
  kp.num_kv_heads = a.num_kv_heads;
  kp.num_q_heads = a.num_q_heads;
  kp.group = a.num_q_heads / a.num_kv_heads;
  const int gt = decode_head_tile(kp.group);
  kp.head_tiles = (kp.group + gt - 1) / gt;
  kp.max_blocks = a.max_blocks;
  kp.part_tokens = a.part_tokens;
  kp.max_parts = a.max_parts;
  kp.scale_log2 = a.scale * kLog2e;
  kp.merge = a.merge ? 1 : 0;
  if (a.batch == 0 || a.max_parts == 0) return cudaSuccess;
  dim3 grid((unsigned)a.max_parts, (unsigned)(a.num_kv_heads * kp.head_tiles),
            (unsigned)a.batch);
  if (a.dtype != PA_DTYPE_BF16 && a.dtype != PA_DTYPE_F32) return cudaErrorInvalidValue;
  const bool bf16 = a.dtype == PA_DTYPE_BF16;
  if (a.head_dim == 64)
    return bf16 ? launch_dtype_dim<__nv_bfloat16, 64>(kp, gt, grid, stream)
                : launch_dtype_dim<float, 64>(kp, gt, grid, stream);
  if (a.head_dim == 128)
    return bf16 ? launch_dtype_dim<__nv_bfloat16, 128>(kp, gt, grid, stream)
                : launch_dtype_dim<float, 128>(kp, gt, grid, stream);
  return cudaErrorInvalidValue;
}

}  // namespace pa
