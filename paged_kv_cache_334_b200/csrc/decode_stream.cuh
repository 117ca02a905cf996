// decode_stream.cuh -- persistent, pipelined paged decode kernel (pa_decode).
//
// Same computation as decode.cu (page "From correct to faster: the
// PagedAttention optimisation route", sections "The core idea of
// high-performance PagedAttention" and "What the attention kernel really
// does"; address mapping from page "Implementing teaching PagedAttention:
// reading the historical KV cache from the block table", section "From logical
// token to physical block"), organised for B200's memory system:
//
// * Work: the visible pages of all sequences form one stream (sequence 0's
//   pages, then sequence 1's, ...).  Pages are cut into "virtual pages" of at
//   most 32 KB (a run of whole token rows of one physical page, all KV heads --
//   contiguous in the [num_blocks, block_size, Hkv, D] layout).  The grid is one
//   CTA per SM; CTA c takes the contiguous range [c*T/G, (c+1)*T/G) of the T
//   virtual pages, so every CTA moves the same number of bytes (+-1 page)
//   whatever the mix of context lengths.
// * Producer warp: walks its range (block-table entries fetched 32 at a time
//   into registers, context lengths likewise), validates each physical block
//   id, and issues 1-D bulk copies (cp.async.bulk, no multicast) of the valid
//   token rows of K and V -- plus the sequence's query rows when a sequence
//   segment starts -- into a ring of shared-memory stages guarded by mbarriers.
//   For the tensor-core consumers each token row lands at a pitch of
//   row_bytes + 16 so that eight consecutive tokens fall in eight different
//   shared-memory bank groups (conflict-free ldmatrix).
// * Consumer warps keep the online-softmax state (running max, normaliser,
//   fp32 accumulator) of up to 8 query heads of one KV head for the current
//   sequence segment.
//     - bf16: the per-page work is a small-M contraction (the GQA group is the
//       N = 8 side, tokens are M): S^T = K Q^T and O^T += V^T P^T run on the
//       tensor cores (mma.sync m16n8k16, fp32 accumulation), P is rounded to
//       bf16 and turned into the B operand with movmatrix.
//     - fp32: CUDA-core FMAs, per-(token, head) dot products reduced with a
//       transposed butterfly (the 1e-5 tolerance rules out bf16/tf32 MMA).
// * A sequence split across CTAs leaves one partial per CTA in the workspace;
//   the last warp to finish (per sequence and query-head slice, found with an
//   atomic counter -- nobody waits) merges them and resets the counter.
//
// Every mbarrier wait is bounded; on expiry the kernel sets PA_DEVERR_TIMEOUT,
// drains its own copies (bounded) and returns.
#pragma once

#include <math.h>

#include <type_traits>

#include "pa_common.cuh"
#include "pa_launch.h"

namespace pa {
namespace stream {

constexpr uint64_t kWaitLimitNs = 1000000000ull;  // 1 s: far beyond any legitimate wait
constexpr int kFirst = 1, kLast = 2, kBad = 4;

struct alignas(16) PageDesc {
  int32_t seq, ntok, flags, n_contrib;
  int32_t c_first, slot_bits, pb, toff;
};

// ---------------------------------------------------------------------------
// PTX wrappers: mbarrier, 1-D bulk copy (no multicast), warp-level MMA.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; "
      "selp.u32 %0, 1, 0, p; }"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
// Bounded wait; false when kWaitLimitNs passes or the CTA's abort flag is set.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity,
                                          volatile int32_t *abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 15) == 0) {
      if (*abort_flag) return false;
      if (global_ns() - t0 > kWaitLimitNs) return false;
    }
  }
}
__device__ __forceinline__ void bulk_g2s(void *smem_dst, const void *gsrc, uint32_t bytes,
                                         uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(smem_dst)),
      "l"(gsrc), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}
// Tiled tensor copy of one box (coordinates innermost first), no multicast.
__device__ __forceinline__ void tma_load_3d(void *smem_dst, const CUtensorMap *map, int x, int y,
                                            int z, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], "
      "[%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_trans(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
// D += A (16x16, row) * B (16x8, col), bf16 inputs, fp32 accumulation.
__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                          uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// Two fp32 -> packed bf16x2 (round to nearest even); `lo` in the low half.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

__device__ __forceinline__ int32_t vpages_of(int32_t ctx, const Params &p) {
  if (ctx <= 0 || (int64_t)ctx > (int64_t)p.max_blocks * p.block_size) return 0;
  return (ctx + p.vbs - 1) >> p.log2_vbs;
}

// Largest CTA index whose range starts at or before page `pg` (ranges
// [c*T/G, (c+1)*T/G) with T >= G, so every range is non-empty).
__device__ __forceinline__ int32_t owner_of(int64_t pg, int64_t T, int32_t G) {
  return (int32_t)(((pg + 1) * G - 1) / T);
}

// Block-wide sum of int64 values (all threads call; result to all).
__device__ __forceinline__ int64_t block_sum(int64_t v, int64_t *s_red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nw = (blockDim.x + 31) >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  __syncthreads();
  if (lane == 0) s_red[warp] = v;
  __syncthreads();
  int64_t t = 0;
  for (int w = 0; w < nw; ++w) t += s_red[w];
  __syncthreads();
  return t;
}

// Block-wide exclusive scan of int64 values; returns the prefix, sets *total.
__device__ __forceinline__ int64_t block_exclusive_scan(int64_t v, int64_t *s_red,
                                                        int64_t *total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nw = (blockDim.x + 31) >> 5;
  int64_t inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int64_t n = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += n;
  }
  __syncthreads();
  if (lane == 31) s_red[warp] = inc;
  __syncthreads();
  int64_t base = 0, tot = 0;
  for (int w = 0; w < nw; ++w) {
    if (w < warp) base += s_red[w];
    tot += s_red[w];
  }
  __syncthreads();
  *total = tot;
  return base + inc - v;
}

struct alignas(16) Shared {
  uint64_t full[kMaxStages];
  uint64_t empty[kMaxStages];
  int64_t red[32];
  int64_t P_begin;
  int32_t s_begin, vlb_begin, abort_flag, pad;
};

// ===========================================================================
// bf16 consumer: tensor-core tiles of 16 tokens x 8 query heads.
// Lane (g = lane / 4, t = lane % 4) holds, for each 16-token tile, the scores
// of tokens g and g + 8 for query heads 2t and 2t + 1, and for each 16-wide
// d tile the output accumulator of d = 16 dt + g (+8) for the same two heads.
// ===========================================================================
template <int D>
struct MmaConsumer {
  static constexpr int KS = D / 16;  // k steps of QK, d tiles of PV
  uint32_t qb[KS][2];                // Q^T as B operand (d x head), one pair per k step
  float o[KS][4];                    // O^T accumulators
  float m0, m1, l0, l1;              // running max / partial normaliser, heads 2t, 2t+1
  float scale_log2_;
  bool seg_bad;

  __device__ __forceinline__ void reset() {
#pragma unroll
    for (int k = 0; k < KS; ++k)
#pragma unroll
      for (int e = 0; e < 4; ++e) o[k][e] = 0.f;
    m0 = m1 = -INFINITY;
    l0 = l1 = 0.f;
    seg_bad = false;
  }

  // Query rows of this warp's heads (bf16 in shared memory, [Hq][D]).
  __device__ __forceinline__ void load_q(const __nv_bfloat16 *qs, int hq0, int nh, int lane) {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int k = 0; k < KS; ++k) {
      if (g < nh) {
        const uint32_t *row = reinterpret_cast<const uint32_t *>(qs + (size_t)(hq0 + g) * D);
        qb[k][0] = row[(k * 16 + t * 2) >> 1];
        qb[k][1] = row[(k * 16 + t * 2 + 8) >> 1];
      } else {
        qb[k][0] = qb[k][1] = 0u;
      }
    }
  }

  // One staged virtual page of `ntok` tokens.  Layouts:
  //  tile  : per 64-wide d half a box of [KV head][vbs tokens][128 B] rows with
  //          the 16-byte chunk index XORed with (row % 8) (128-byte swizzle);
  //  padded: token rows `pitch` bytes apart, this head's slice at col_bytes.
  // Either way eight consecutive tokens at one chunk hit eight bank groups.
  __device__ __forceinline__ void page(const unsigned char *kp, const unsigned char *vp,
                                       int ntok, const Params &p, int h, int col_bytes,
                                       int lane) {
    const int g = lane >> 2, t = lane & 3;
    const bool tile = p.tile != 0;
    for (int m0t = 0; m0t < ntok; m0t += 16) {
      // S^T (16 tokens x 8 heads) = K (16 x D) Q^T (D x 8)
      float s[4] = {0.f, 0.f, 0.f, 0.f};
      const int tk = m0t + (lane & 15), hk = lane >> 4;
      const int rowk = tile ? (h * p.vbs + tk) * 128 : tk * p.row_pitch + col_bytes;
#pragma unroll
      for (int k = 0; k < KS; ++k) {
        const int cg = k * 2 + hk;  // 16-byte chunk of the row (8 elements)
        const int off = tile ? (cg >> 3) * p.box_bytes + rowk + (((cg & 7) ^ (tk & 7)) << 4)
                             : rowk + cg * 16;
        uint32_t a[4];
        ldsm_x4(a, smem_u32(kp + off));
        mma_16816(s, a, qb[k][0], qb[k][1]);
      }
      const bool v0 = m0t + g < ntok, v1 = m0t + g + 8 < ntok;
      s[0] = v0 ? s[0] * scale_log2_ : -INFINITY;
      s[1] = v0 ? s[1] * scale_log2_ : -INFINITY;
      s[2] = v1 ? s[2] * scale_log2_ : -INFINITY;
      s[3] = v1 ? s[3] * scale_log2_ : -INFINITY;
      float x0 = fmaxf(s[0], s[2]), x1 = fmaxf(s[1], s[3]);
#pragma unroll
      for (int mask = 4; mask < 32; mask <<= 1) {
        x0 = fmaxf(x0, __shfl_xor_sync(0xffffffffu, x0, mask));
        x1 = fmaxf(x1, __shfl_xor_sync(0xffffffffu, x1, mask));
      }
      const float n0 = fmaxf(m0, x0), n1 = fmaxf(m1, x1);
      const float a0 = exp2f(m0 - n0), a1 = exp2f(m1 - n1);
      m0 = n0;
      m1 = n1;
      const float p0 = exp2f(s[0] - n0), p1 = exp2f(s[1] - n1);
      const float p2 = exp2f(s[2] - n0), p3 = exp2f(s[3] - n1);
      l0 = l0 * a0 + p0 + p2;
      l1 = l1 * a1 + p1 + p3;
      if (!__all_sync(0xffffffffu, a0 == 1.f && a1 == 1.f)) {
#pragma unroll
        for (int k = 0; k < KS; ++k) {
          o[k][0] *= a0;
          o[k][1] *= a1;
          o[k][2] *= a0;
          o[k][3] *= a1;
        }
      }
      // P^T (16 tokens x 8 heads) as the B operand: transpose the two 8x8 tiles.
      const uint32_t b0 = movmatrix_trans(pack_bf16x2(p0, p1));
      const uint32_t b1 = movmatrix_trans(pack_bf16x2(p2, p3));
      // V rows past ntok may hold anything (other tokens, never-written
      // shared memory): their P is 0, and their V elements are zeroed below
      // so that 0 * NaN cannot occur.
      const bool partial = m0t + 16 > ntok;
      uint32_t mlo = 0xffffffffu, mhi = 0xffffffffu;
      if (partial) {
        mlo = (m0t + 2 * t < ntok ? 0x0000ffffu : 0u) | (m0t + 2 * t + 1 < ntok ? 0xffff0000u : 0u);
        mhi = (m0t + 2 * t + 8 < ntok ? 0x0000ffffu : 0u) |
              (m0t + 2 * t + 9 < ntok ? 0xffff0000u : 0u);
      }
      const int mi = lane >> 3, rr = lane & 7;
      const int tv = m0t + rr + ((mi >> 1) << 3), hv = mi & 1;
      const int rowv = tile ? (h * p.vbs + tv) * 128 : tv * p.row_pitch + col_bytes;
#pragma unroll
      for (int k = 0; k < KS; ++k) {
        const int cg = k * 2 + hv;
        const int off = tile ? (cg >> 3) * p.box_bytes + rowv + (((cg & 7) ^ (tv & 7)) << 4)
                             : rowv + cg * 16;
        uint32_t a[4];
        ldsm_x4_trans(a, smem_u32(vp + off));
        a[0] &= mlo;
        a[1] &= mlo;
        a[2] &= mhi;
        a[3] &= mhi;
        mma_16816(o[k], a, b0, b1);
      }
    }
  }

  // End of a segment: write out[...] directly or a partial + merge.
  template <typename Tout>
  __device__ __forceinline__ void flush(const Params &p, const PageDesc &d, int hq0, int nh,
                                        int c, int lane, int32_t *counter) {
    const int g = lane >> 2, t = lane & 3;
    float L0 = l0, L1 = l1;
#pragma unroll
    for (int mask = 4; mask < 32; mask <<= 1) {
      L0 += __shfl_xor_sync(0xffffffffu, L0, mask);
      L1 += __shfl_xor_sync(0xffffffffu, L1, mask);
    }
    const int h0 = 2 * t, h1 = 2 * t + 1;
    const int64_t orow = (int64_t)d.seq * p.num_q_heads + hq0;
    if (d.n_contrib == 1) {
      const float i0 = 1.f / L0, i1 = 1.f / L1;
#pragma unroll
      for (int k = 0; k < KS; ++k) {
        const int dd = k * 16 + g;
        if (h0 < nh) {
          Elem<Tout>::store1(p.out, (orow + h0) * D + dd, seg_bad ? 0.f : o[k][0] * i0);
          Elem<Tout>::store1(p.out, (orow + h0) * D + dd + 8, seg_bad ? 0.f : o[k][2] * i0);
        }
        if (h1 < nh) {
          Elem<Tout>::store1(p.out, (orow + h1) * D + dd, seg_bad ? 0.f : o[k][1] * i1);
          Elem<Tout>::store1(p.out, (orow + h1) * D + dd + 8, seg_bad ? 0.f : o[k][3] * i1);
        }
      }
      return;
    }
    const int64_t prow = ((int64_t)c * 2 + (d.slot_bits & 1)) * p.num_q_heads + hq0;
    if (g == 0) {
      if (h0 < nh) {
        p.part_ml[(prow + h0) * 2 + 0] = m0;
        p.part_ml[(prow + h0) * 2 + 1] = seg_bad ? -1.f : L0;
      }
      if (h1 < nh) {
        p.part_ml[(prow + h1) * 2 + 0] = m1;
        p.part_ml[(prow + h1) * 2 + 1] = seg_bad ? -1.f : L1;
      }
    }
    {
      const float i0 = 1.f / L0, i1 = 1.f / L1;
#pragma unroll
      for (int k = 0; k < KS; ++k) {
        const int dd = k * 16 + g;
        if (h0 < nh) {
          p.part_o[(prow + h0) * D + dd] = seg_bad ? 0.f : o[k][0] * i0;
          p.part_o[(prow + h0) * D + dd + 8] = seg_bad ? 0.f : o[k][2] * i0;
        }
        if (h1 < nh) {
          p.part_o[(prow + h1) * D + dd] = seg_bad ? 0.f : o[k][1] * i1;
          p.part_o[(prow + h1) * D + dd + 8] = seg_bad ? 0.f : o[k][3] * i1;
        }
      }
    }
    __threadfence();
    __syncwarp();
    int32_t old = 0;
    if (lane == 0) old = atomicAdd(counter, 1);
    old = __shfl_sync(0xffffffffu, old, 0);
    if (old != d.n_contrib - 1) return;
    // Last contributor: merge every CTA's partial of this sequence / slice.
    __threadfence();
    const int first_slot = (d.slot_bits >> 1) & 1;
    float M0 = -INFINITY, M1 = -INFINITY, W0 = 0.f, W1 = 0.f;
    bool any_bad = false;
    for (int x = 0; x < d.n_contrib; ++x) {
      const int64_t r =
          ((int64_t)(d.c_first + x) * 2 + (x == 0 ? first_slot : 0)) * p.num_q_heads + hq0;
      if (h0 < nh) {
        any_bad |= __ldcg(p.part_ml + (r + h0) * 2 + 1) < 0.f;
        M0 = fmaxf(M0, __ldcg(p.part_ml + (r + h0) * 2 + 0));
      }
      if (h1 < nh) {
        any_bad |= __ldcg(p.part_ml + (r + h1) * 2 + 1) < 0.f;
        M1 = fmaxf(M1, __ldcg(p.part_ml + (r + h1) * 2 + 0));
      }
    }
    float acc[KS][4];
#pragma unroll
    for (int k = 0; k < KS; ++k)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[k][e] = 0.f;
    for (int x = 0; x < d.n_contrib; ++x) {
      const int64_t r =
          ((int64_t)(d.c_first + x) * 2 + (x == 0 ? first_slot : 0)) * p.num_q_heads + hq0;
      float w0 = 0.f, w1 = 0.f;
      if (h0 < nh)
        w0 = __ldcg(p.part_ml + (r + h0) * 2 + 1) *
             exp2f(__ldcg(p.part_ml + (r + h0) * 2 + 0) - M0);
      if (h1 < nh)
        w1 = __ldcg(p.part_ml + (r + h1) * 2 + 1) *
             exp2f(__ldcg(p.part_ml + (r + h1) * 2 + 0) - M1);
      W0 += w0;
      W1 += w1;
#pragma unroll
      for (int k = 0; k < KS; ++k) {
        const int dd = k * 16 + g;
        if (h0 < nh) {
          acc[k][0] += w0 * __ldcg(p.part_o + (r + h0) * D + dd);
          acc[k][2] += w0 * __ldcg(p.part_o + (r + h0) * D + dd + 8);
        }
        if (h1 < nh) {
          acc[k][1] += w1 * __ldcg(p.part_o + (r + h1) * D + dd);
          acc[k][3] += w1 * __ldcg(p.part_o + (r + h1) * D + dd + 8);
        }
      }
    }
    const float i0 = 1.f / W0, i1 = 1.f / W1;
#pragma unroll
    for (int k = 0; k < KS; ++k) {
      const int dd = k * 16 + g;
      if (h0 < nh) {
        Elem<Tout>::store1(p.out, (orow + h0) * D + dd, any_bad ? 0.f : acc[k][0] * i0);
        Elem<Tout>::store1(p.out, (orow + h0) * D + dd + 8, any_bad ? 0.f : acc[k][2] * i0);
      }
      if (h1 < nh) {
        Elem<Tout>::store1(p.out, (orow + h1) * D + dd, any_bad ? 0.f : acc[k][1] * i1);
        Elem<Tout>::store1(p.out, (orow + h1) * D + dd + 8, any_bad ? 0.f : acc[k][3] * i1);
      }
    }
    if (lane == 0) atomicExch(counter, 0);
  }
};

// ===========================================================================
// fp32 consumer: CUDA-core FMAs for G query heads of one KV head.
// ===========================================================================
template <typename T, int D, int G>
struct FmaConsumer {
  static constexpr int EPV = Elem<T>::kPerVec;
  static constexpr int LPT = D / EPV;
  static constexpr int TPW = 32 / LPT;
  static constexpr int UMAX = (G >= 8) ? 4 : 8;
  static constexpr int U = (16 / TPW < UMAX) ? 16 / TPW : UMAX;
  static constexpr int TPI = U * TPW;
  static constexpr int N = U * G;
  static constexpr int NV = (N >= LPT) ? N / LPT : 1;
  static constexpr int E = TPI * G;
  static constexpr int EPL = (E + 31) / 32;
  static_assert(U >= 1 && (32 % G) == 0 && (32 % LPT) == 0, "shape");

  float m_run, l_run;
  float acc[G][EPV];
  float qf[G][EPV];
  bool seg_bad;

  __device__ __forceinline__ void reset() {
    m_run = -INFINITY;
    l_run = 0.f;
    seg_bad = false;
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
      for (int e = 0; e < EPV; ++e) acc[g][e] = 0.f;
  }

  __device__ __forceinline__ void load_q(const T *qs, int hq0, int lane, float scale_log2) {
    const int j = lane % LPT;
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const uint4 raw = *reinterpret_cast<const uint4 *>(qs + (size_t)(hq0 + g) * D + j * EPV);
      Elem<T>::widen(raw, qf[g]);
#pragma unroll
      for (int e = 0; e < EPV; ++e) qf[g][e] *= scale_log2;
    }
  }

  __device__ __forceinline__ void page(const unsigned char *kp, const unsigned char *vp,
                                       int ntok, int pitch, int col_bytes, float *sc_buf,
                                       int lane) {
    const int tg = lane / LPT, j = lane % LPT;
    for (int t0 = 0; t0 < ntok; t0 += TPI) {
      uint4 raw[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int t = t0 + u * TPW + tg;
        raw[u] = (t < ntok) ? *reinterpret_cast<const uint4 *>(kp + (size_t)t * pitch + col_bytes +
                                                               j * 16)
                            : make_uint4(0u, 0u, 0u, 0u);
      }
      float sc[N];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        float kf[EPV];
        Elem<T>::widen(raw[u], kf);
#pragma unroll
        for (int g = 0; g < G; ++g) {
          float dot = 0.f;
#pragma unroll
          for (int e = 0; e < EPV; ++e) dot = fmaf(qf[g][e], kf[e], dot);
          sc[u * G + g] = dot;
        }
      }
      Butterfly<N, LPT / 2>::run(sc, lane);
      if constexpr (N >= LPT) {
#pragma unroll
        for (int x = 0; x < NV; ++x) {
          const int idx = j * NV + x;
          const int u = idx / G, g = idx % G;
          const int tl = u * TPW + tg;
          sc_buf[tl * G + g] = (t0 + tl < ntok) ? sc[x] : -INFINITY;
        }
      } else {
        constexpr int R = LPT / N;
        if ((j % R) == 0) {
          const int idx = j / R;
          const int u = idx / G, g = idx % G;
          const int tl = u * TPW + tg;
          sc_buf[tl * G + g] = (t0 + tl < ntok) ? sc[0] : -INFINITY;
        }
      }
      __syncwarp();
      float sv[EPL];
      float tmax = -INFINITY;
#pragma unroll
      for (int x = 0; x < EPL; ++x) {
        const int e = lane + 32 * x;
        sv[x] = (e < E) ? sc_buf[e] : -INFINITY;
        tmax = fmaxf(tmax, sv[x]);
      }
#pragma unroll
      for (int mask = G; mask < 32; mask <<= 1)
        tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, mask));
      const float m_new = fmaxf(m_run, tmax);
      const float alpha = exp2f(m_run - m_new);
      m_run = m_new;
      float psum = 0.f;
#pragma unroll
      for (int x = 0; x < EPL; ++x) {
        const int e = lane + 32 * x;
        const float pe = exp2f(sv[x] - m_new);
        psum += pe;
        if (e < E) sc_buf[e] = pe;
      }
      l_run = l_run * alpha + psum;
      if (!__all_sync(0xffffffffu, alpha == 1.f)) {
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const float a = __shfl_sync(0xffffffffu, alpha, g);
#pragma unroll
          for (int e = 0; e < EPV; ++e) acc[g][e] *= a;
        }
      }
      __syncwarp();
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int t = t0 + u * TPW + tg;
        raw[u] = (t < ntok) ? *reinterpret_cast<const uint4 *>(vp + (size_t)t * pitch + col_bytes +
                                                               j * 16)
                            : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int tl = u * TPW + tg;
        float vf[EPV];
        Elem<T>::widen(raw[u], vf);
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const float pg = sc_buf[tl * G + g];
#pragma unroll
          for (int e = 0; e < EPV; ++e) acc[g][e] = fmaf(pg, vf[e], acc[g][e]);
        }
      }
      __syncwarp();
    }
  }

  __device__ __forceinline__ void flush(const Params &p, const PageDesc &d, int hq0, int c,
                                        int lane, int32_t *counter) {
    const int tg = lane / LPT, j = lane % LPT;
    float ac[G][EPV];
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
      for (int e = 0; e < EPV; ++e) {
        float v = acc[g][e];
#pragma unroll
        for (int mask = LPT; mask < 32; mask <<= 1) v += __shfl_xor_sync(0xffffffffu, v, mask);
        ac[g][e] = v;
      }
    float lsum = l_run;
#pragma unroll
    for (int mask = G; mask < 32; mask <<= 1) lsum += __shfl_xor_sync(0xffffffffu, lsum, mask);
    float lg[G];
#pragma unroll
    for (int g = 0; g < G; ++g) lg[g] = __shfl_sync(0xffffffffu, lsum, g);
    const int64_t orow = (int64_t)d.seq * p.num_q_heads + hq0;
    if (d.n_contrib == 1) {
      if (tg == 0) {
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
          for (int e = 0; e < EPV; ++e)
            Elem<T>::store1(p.out, (orow + g) * D + j * EPV + e,
                            seg_bad ? 0.f : ac[g][e] / lg[g]);
      }
      return;
    }
    const int64_t prow = ((int64_t)c * 2 + (d.slot_bits & 1)) * p.num_q_heads + hq0;
    if (lane < G) {
      p.part_ml[(prow + lane) * 2 + 0] = m_run;
      p.part_ml[(prow + lane) * 2 + 1] = seg_bad ? -1.f : lsum;
    }
    if (tg == 0) {
#pragma unroll
      for (int g = 0; g < G; ++g)
#pragma unroll
        for (int e = 0; e < EPV; ++e)
          p.part_o[(prow + g) * D + j * EPV + e] = seg_bad ? 0.f : ac[g][e] / lg[g];
    }
    __threadfence();
    __syncwarp();
    int32_t old = 0;
    if (lane == 0) old = atomicAdd(counter, 1);
    old = __shfl_sync(0xffffffffu, old, 0);
    if (old != d.n_contrib - 1) return;
    __threadfence();
    const int first_slot = (d.slot_bits >> 1) & 1;
    float M[G], W[G];
    bool any_bad = false;
#pragma unroll
    for (int g = 0; g < G; ++g) {
      M[g] = -INFINITY;
      W[g] = 0.f;
    }
    for (int x = 0; x < d.n_contrib; ++x) {
      const int64_t r =
          ((int64_t)(d.c_first + x) * 2 + (x == 0 ? first_slot : 0)) * p.num_q_heads + hq0;
#pragma unroll
      for (int g = 0; g < G; ++g) {
        any_bad |= __ldcg(p.part_ml + (r + g) * 2 + 1) < 0.f;
        M[g] = fmaxf(M[g], __ldcg(p.part_ml + (r + g) * 2 + 0));
      }
    }
    float O[G][EPV];
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
      for (int e = 0; e < EPV; ++e) O[g][e] = 0.f;
    for (int x = 0; x < d.n_contrib; ++x) {
      const int64_t r =
          ((int64_t)(d.c_first + x) * 2 + (x == 0 ? first_slot : 0)) * p.num_q_heads + hq0;
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float w = __ldcg(p.part_ml + (r + g) * 2 + 1) *
                        exp2f(__ldcg(p.part_ml + (r + g) * 2 + 0) - M[g]);
        W[g] += w;
        if (tg == 0) {
#pragma unroll
          for (int e = 0; e < EPV; ++e)
            O[g][e] += w * __ldcg(p.part_o + (r + g) * D + j * EPV + e);
        }
      }
    }
    if (tg == 0) {
#pragma unroll
      for (int g = 0; g < G; ++g)
#pragma unroll
        for (int e = 0; e < EPV; ++e)
          Elem<T>::store1(p.out, (orow + g) * D + j * EPV + e, any_bad ? 0.f : O[g][e] / W[g]);
    }
    if (lane == 0) atomicExch(counter, 0);
  }
};

// ===========================================================================
// The kernel.  T = element type; D = head_dim; G = query heads per KV head
// for the fp32 consumer (unused, 0, for bf16); NCW = consumer warps.
// ===========================================================================
template <typename T, int D, int G, int NCW>
__global__ void __launch_bounds__((NCW + 1) * 32, 1)
    decode_stream_kernel(const __grid_constant__ Params p) {
  constexpr bool kMma = std::is_same<T, __nv_bfloat16>::value;
  constexpr int kScoreFloats = kMma ? 1 : FmaConsumer<T, D, (G > 0 ? G : 1)>::E;
  static_assert(sizeof(Shared) + sizeof(PageDesc) * kMaxStages * kMaxPPS +
                        sizeof(float) * NCW * kScoreFloats <= kHdrBytes,
                "header region");
  static_assert(sizeof(Shared) % 16 == 0 && sizeof(PageDesc) % 16 == 0,
                "descriptors and score buffers need 16-byte alignment");
  using Cons = typename std::conditional<kMma, MmaConsumer<D>,
                                         FmaConsumer<T, D, (G > 0 ? G : 1)>>::type;
  extern __shared__ __align__(128) unsigned char smem_raw[];
  Shared &sh = *reinterpret_cast<Shared *>(smem_raw);
  PageDesc *descs = reinterpret_cast<PageDesc *>(smem_raw + sizeof(Shared));
  float *s_scores = reinterpret_cast<float *>(smem_raw + sizeof(Shared) +
                                              sizeof(PageDesc) * kMaxStages * kMaxPPS);
  // stages start 1024-byte aligned (the 128-byte swizzle repeats every 1 KB)
  unsigned char *stages =
      smem_raw + (((smem_u32(smem_raw) + p.hdr_bytes + 1023u) & ~1023u) - smem_u32(smem_raw));

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int c = blockIdx.x;

  if (tid == 0) {
    for (int i = 0; i < p.stages; ++i) {
      mbar_init(&sh.full[i], 1);
      mbar_init(&sh.empty[i], NCW);
    }
    sh.abort_flag = 0;
    // make the initialised barriers visible to the bulk-copy (async) proxy
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }

  // ---- Prologue: total virtual pages T, this CTA's range and first page.
  int64_t T_loc = 0;
  for (int base = 0; base < p.batch; base += blockDim.x) {
    const int s = base + tid;
    const int64_t v = (s < p.batch) ? vpages_of(p.context_lens[s], p) : 0;
    T_loc += block_sum(v, sh.red);
  }
  const int64_t Tp = T_loc;
  const int32_t g_eff = (int32_t)((Tp < p.grid) ? Tp : p.grid);
  const bool active = c < g_eff;
  int64_t start = 0, end = 0;
  if (active) {
    start = (int64_t)c * Tp / g_eff;
    end = (int64_t)(c + 1) * Tp / g_eff;
    int64_t run = 0;
    for (int base = 0; base < p.batch; base += blockDim.x) {
      const int s = base + tid;
      const int64_t v = (s < p.batch) ? vpages_of(p.context_lens[s], p) : 0;
      int64_t tot;
      const int64_t P = run + block_exclusive_scan(v, sh.red, &tot);
      if (v > 0 && P <= start && start < P + v) {
        sh.s_begin = s;
        sh.vlb_begin = (int32_t)(start - P);
        sh.P_begin = P;
      }
      run += tot;
      if (run > start) break;  // uniform: every thread sees the same `run`
    }
  }
  __syncthreads();

  const bool per_row = p.row_pitch != p.row_bytes;
  if (active) {
    const int n_stages = (int)((end - start + p.pps - 1) / p.pps);
    if (warp == 0) {
      // ===================== producer =====================
      int32_t s = sh.s_begin;
      int32_t vlb = sh.vlb_begin;
      int64_t P_s = sh.P_begin;
      // context-length window: lane l holds sequence cw + l
      int32_t cw = s;
      int32_t cw_ctx = (cw + lane < p.batch) ? p.context_lens[cw + lane] : 0;
      int32_t ctx_s = __shfl_sync(0xffffffffu, cw_ctx, 0);
      int32_t pages_s = vpages_of(ctx_s, p);
      // block-table window: lane l holds entry tw_lb + l of sequence tw_seq
      int32_t tw_seq = -1, tw_lb = 0, tw_val = -1;
      int64_t cursor = start;
      bool ok = true;
      int issued = 0;
      for (int i = 0; i < n_stages && ok; ++i) {
        const int slot = i % p.stages;
        if (i >= p.stages) {
          ok = __all_sync(0xffffffffu,
                          mbar_wait(&sh.empty[slot], ((i / p.stages) - 1) & 1, &sh.abort_flag));
          if (!ok) break;
        }
        const int npg = (int)min((int64_t)p.pps, end - cursor);
        uint32_t bytes = 0;
        for (int k = 0; k < npg; ++k) {
          const int32_t lb = vlb >> p.log2_vpp;
          if (s != tw_seq || lb >= tw_lb + 32) {
            tw_seq = s;
            tw_lb = lb;
            const int32_t e = lb + lane;
            tw_val = (e < p.max_blocks) ? p.block_tables[(int64_t)s * p.max_blocks + e] : -1;
          }
          const int32_t pb = __shfl_sync(0xffffffffu, tw_val, lb - tw_lb);
          const int32_t ntok = min(p.vbs, ctx_s - vlb * p.vbs);
          const bool first = (vlb == 0) || (cursor == start);
          const bool last = (vlb == pages_s - 1) || (cursor == end - 1);
          const bool bad = pb < 0 || pb >= p.num_blocks;
          if (lane == 0) {
            PageDesc d;
            d.seq = s;
            d.ntok = ntok;
            d.flags = (first ? kFirst : 0) | (last ? kLast : 0) | (bad ? kBad : 0);
            d.pb = pb;
            d.toff = (vlb & ((1 << p.log2_vpp) - 1)) * p.vbs;
            d.n_contrib = 1;
            d.c_first = c;
            d.slot_bits = 0;
            if (last) {
              const int32_t c_first = owner_of(P_s, Tp, g_eff);
              const int32_t c_last = owner_of(P_s + pages_s - 1, Tp, g_eff);
              d.n_contrib = c_last - c_first + 1;
              d.c_first = c_first;
              const int64_t st_first = (int64_t)c_first * Tp / g_eff;
              d.slot_bits = ((start < P_s) ? 1 : 0) | ((st_first < P_s) ? 2 : 0);
            }
            descs[slot * kMaxPPS + k] = d;
          }
          if (!bad)
            bytes += p.tile ? 2u * (uint32_t)p.n_dhalf * (uint32_t)p.box_bytes
                            : 2u * (uint32_t)ntok * (uint32_t)p.row_bytes;
          if (first) bytes += (uint32_t)p.q_bytes;
          // advance the cursor
          ++cursor;
          ++vlb;
          if (vlb == pages_s && cursor < end) {
            // next sequence with at least one page
            int32_t nxt = s + 1;
            for (;;) {
              if (nxt >= cw + 32) {
                cw = nxt;
                cw_ctx = (cw + lane < p.batch) ? p.context_lens[cw + lane] : 0;
              }
              const bool has = (cw + lane >= nxt) && (cw + lane < p.batch) &&
                               vpages_of(cw_ctx, p) > 0;
              const uint32_t m = __ballot_sync(0xffffffffu, has);
              if (m) {
                const int l = __ffs(m) - 1;
                nxt = cw + l;
                ctx_s = __shfl_sync(0xffffffffu, cw_ctx, l);
                break;
              }
              nxt = cw + 32;
            }
            P_s += pages_s;
            s = nxt;
            vlb = 0;
            pages_s = vpages_of(ctx_s, p);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive_expect_tx(&sh.full[slot], bytes);
        __syncwarp();
        unsigned char *st = stages + (size_t)slot * p.stage_bytes;
        unsigned char *kst = st;
        unsigned char *vst = st + (size_t)p.pps * p.vpage_stride;
        unsigned char *qst = st + (size_t)2 * p.pps * p.vpage_stride;
        for (int k = 0; k < npg; ++k) {
          const PageDesc d = descs[slot * kMaxPPS + k];
          if (!(d.flags & kBad) && p.tile) {
            // one box per (tensor, 64-wide d half), one lane each
            if (lane < 2 * p.n_dhalf) {
              const int dh = lane % p.n_dhalf;
              const bool isv = lane >= p.n_dhalf;
              tma_load_3d((isv ? vst : kst) + (size_t)k * p.vpage_stride + (size_t)dh * p.box_bytes,
                          isv ? &p.tmap_v : &p.tmap_k, dh * 64, d.pb * p.block_size + d.toff, 0,
                          &sh.full[slot]);
            }
          } else if (!(d.flags & kBad)) {
            const int64_t off = ((int64_t)d.pb * p.block_size + d.toff) * (int64_t)p.row_bytes;
            const unsigned char *ksrc = static_cast<const unsigned char *>(p.key_cache) + off;
            const unsigned char *vsrc = static_cast<const unsigned char *>(p.value_cache) + off;
            if (per_row) {
              // one row per lane: rows land at the padded pitch
              for (int t = lane; t < d.ntok; t += 32) {
                bulk_g2s(kst + (size_t)k * p.vpage_stride + (size_t)t * p.row_pitch,
                         ksrc + (size_t)t * p.row_bytes, (uint32_t)p.row_bytes, &sh.full[slot]);
                bulk_g2s(vst + (size_t)k * p.vpage_stride + (size_t)t * p.row_pitch,
                         vsrc + (size_t)t * p.row_bytes, (uint32_t)p.row_bytes, &sh.full[slot]);
              }
            } else if (lane == 0) {
              const uint32_t nb = (uint32_t)d.ntok * (uint32_t)p.row_bytes;
              bulk_g2s(kst + (size_t)k * p.vpage_stride, ksrc, nb, &sh.full[slot]);
              bulk_g2s(vst + (size_t)k * p.vpage_stride, vsrc, nb, &sh.full[slot]);
            }
          }
          if ((d.flags & kFirst) && lane == 0) {
            bulk_g2s(qst + (size_t)k * p.q_bytes,
                     static_cast<const unsigned char *>(p.q) + (int64_t)d.seq * p.q_bytes,
                     (uint32_t)p.q_bytes, &sh.full[slot]);
          }
        }
        __syncwarp();
        issued = i + 1;
      }
      if (!ok && lane == 0) {
        sh.abort_flag = 1;
        set_error(p.err_word, PA_DEVERR_TIMEOUT);
      }
      // Drain: every issued stage's copies must land before the CTA exits.
      if (lane == 0) {
        volatile int32_t dummy = 0;
        for (int i = (issued > p.stages ? issued - p.stages : 0); i < issued; ++i)
          mbar_wait(&sh.full[i % p.stages], (i / p.stages) & 1, &dummy);
      }
    } else if (warp <= NCW) {
      // ===================== consumers =====================
      const int cw_idx = warp - 1;
      const int h = cw_idx / p.warps_per_kv;  // KV head
      const int hq0 = h * p.group + (cw_idx % p.warps_per_kv) * p.heads_per_warp;
      const int col_bytes = h * D * (int)sizeof(T);
      Cons cs;
      cs.reset();
      if constexpr (kMma) cs.scale_log2_ = p.scale_log2;
      float *sc_buf = s_scores + (size_t)cw_idx * kScoreFloats;
      int64_t cursor = start;
      for (int i = 0; i < n_stages; ++i) {
        const int slot = i % p.stages;
        if (!__all_sync(0xffffffffu, mbar_wait(&sh.full[slot], (i / p.stages) & 1,
                                               &sh.abort_flag))) {
          if (lane == 0) {
            sh.abort_flag = 1;
            set_error(p.err_word, PA_DEVERR_TIMEOUT);
          }
          break;
        }
        const unsigned char *st = stages + (size_t)slot * p.stage_bytes;
        const unsigned char *kst = st;
        const unsigned char *vst = st + (size_t)p.pps * p.vpage_stride;
        const unsigned char *qst = st + (size_t)2 * p.pps * p.vpage_stride;
        const int npg = (int)min((int64_t)p.pps, end - cursor);
        cursor += npg;
        for (int k = 0; k < npg; ++k) {
          const PageDesc d = descs[slot * kMaxPPS + k];
          if (d.flags & kFirst) {
            cs.reset();
            const T *qs = reinterpret_cast<const T *>(qst + (size_t)k * p.q_bytes);
            if constexpr (kMma) {
              cs.load_q(qs, hq0, p.heads_per_warp, lane);
            } else {
              cs.load_q(qs, hq0, lane, p.scale_log2);
            }
          }
          if (d.flags & kBad) {
            cs.seg_bad = true;
          } else {
            const unsigned char *kp = kst + (size_t)k * p.vpage_stride;
            const unsigned char *vp = vst + (size_t)k * p.vpage_stride;
            if constexpr (kMma) {
              cs.page(kp, vp, d.ntok, p, h, col_bytes, lane);
            } else {
              cs.page(kp, vp, d.ntok, p.row_pitch, col_bytes, sc_buf, lane);
            }
          }
          if (d.flags & kLast) {
            // one counter per (sequence, query-head slice of one warp)
            const int slices = p.num_q_heads / p.heads_per_warp;
            int32_t *counter =
                p.counters + (int64_t)d.seq * slices + hq0 / p.heads_per_warp;
            if constexpr (kMma) {
              cs.template flush<T>(p, d, hq0, p.heads_per_warp, c, lane, counter);
            } else {
              cs.flush(p, d, hq0, c, lane, counter);
            }
            if (cs.seg_bad && lane == 0) set_error(p.err_word, PA_DEVERR_BLOCK_ID);
            cs.reset();
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh.empty[slot]);
      }
    }
  }

  // ---- Sequences with no visible page: zero output (and flag bad lengths).
  __syncthreads();
  for (int s = c; s < p.batch; s += p.grid) {
    const int32_t ctx = p.context_lens[s];
    if (vpages_of(ctx, p) > 0) continue;
    if ((ctx < 0 || (int64_t)ctx > (int64_t)p.max_blocks * p.block_size) && tid == 0)
      set_error(p.err_word, PA_DEVERR_CONTEXT_LEN);
    const int64_t n = (int64_t)p.num_q_heads * D;
    for (int64_t x = tid; x < n; x += blockDim.x) Elem<T>::store1(p.out, (int64_t)s * n + x, 0.f);
  }
}

// ---------------------------------------------------------------------------
// Host side: launch one instantiation.  Explicitly instantiated per dtype in
// its own translation unit.
// ---------------------------------------------------------------------------
template <typename T, int D, int G, int NCW>
cudaError_t launch_one(const Params &p, size_t smem, cudaStream_t stream) {
  auto kern = decode_stream_kernel<T, D, G, NCW>;
  static size_t configured[64] = {};  // per device: largest dynamic smem already allowed
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (smem > configured[dev]) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    configured[dev] = smem;
  }
  kern<<<p.grid, (NCW + 1) * 32, smem, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace stream
}  // namespace pa
