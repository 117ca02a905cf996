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
//   contiguous in the [num_blocks, block_size, Hkv, D] layout); blocks below
//   one page's worth (8-token bf16 blocks, 16-token FP8 blocks) are joined two
//   to a virtual page (two table entries per page).  The grid is one
//   CTA per SM; CTA c takes the contiguous range [c*T/G, (c+1)*T/G) of the T
//   virtual pages, so every CTA moves the same number of bytes (+-1 page)
//   whatever the mix of context lengths.
// * Producer warp: walks its range (block-table entries fetched 32 at a time
//   into registers, context lengths likewise), validates each physical block
//   id, and fills a ring of shared-memory stages guarded by mbarriers (no
//   multicast anywhere):
//     - bf16 with >= 16 tokens per virtual page: tiled tensor copies
//       (cp.async.bulk.tensor.3d) of boxes [64 d][vbs tokens][Hkv heads] of
//       K and V with the 128-byte swizzle, one box per 64-wide half of D, so
//       a whole virtual page takes 2 * D/64 copies and ldmatrix reads it
//       without bank conflicts (two-block pages: one box per block, the
//       second after the first); FP8 pages one box of 128 codes per row;
//       the copies carry an evict-first L2 policy (pages are read once);
//     - otherwise: 1-D bulk copies (cp.async.bulk) of the valid token rows,
//       landing at a pitch of row_bytes + 16 for the tensor-core consumers
//       (eight consecutive tokens in eight different bank groups);
//   plus the sequence's query rows when a sequence segment starts.  With a
//   slot mapping (pa_forward_decode) the producer that reaches a sequence's
//   last page first stores the new token's K/V rows into that page (plain
//   stores + an async-proxy fence) and then copies the page in.
// * Consumer warps keep the online-softmax state (running max, normaliser,
//   fp32 accumulator) of up to 8 query heads of one KV head for the current
//   sequence segment.
//     - bf16: the per-page work is a small-M contraction (the GQA group is the
//       N = 8 side, tokens are M): S^T = K Q^T and O^T += V^T P^T run on the
//       tensor cores (mma.sync m16n8k16, fp32 accumulation), P is rounded to
//       bf16 and turned into the B operand with movmatrix.
//     - FP8: the same tiles in fp16, the fragments built in registers from
//       the staged codes (exact conversion), two 16-token tiles of a 32-token
//       page per pass.
//     - fp32: CUDA-core FMAs, per-(token, head) dot products reduced with a
//       transposed butterfly (the 1e-5 tolerance rules out bf16/tf32 MMA).
// * A sequence split across CTAs leaves one partial per CTA in the workspace,
//   and the CTA that owns its last page records where they are; a small merge
//   kernel (launched right behind, programmatically) folds them together with
//   the running-max rescaling once the stream of pages is done.
// * Split-K mode (pa_decode_splitk): the units are (sequence, partition)
//   pairs of partition_tokens tokens; CTA ranges are snapped to unit
//   boundaries (a unit goes to the CTA whose share of the stream holds its
//   midpoint), so no unit is cut and each CTA writes its units' (max, sum,
//   normalised output) straight into the caller's partial arrays.
//
// Every mbarrier wait is bounded; on expiry the kernel sets PA_DEVERR_TIMEOUT,
// drains its own copies (bounded) and returns.
#pragma once

#include <math.h>

#include <type_traits>

#include "pa_common.cuh"
#include "pa_launch.h"
#include "sm100_ptx.cuh"


namespace pa {
namespace stream {

// Page descriptor flags: first page of a sequence in this CTA (reset, load
// q), last page of a unit (a sequence, or a split-K partition) in this CTA
// (flush, then reset), a bad block id, the sequence is cut between CTAs
// (flush a partial), the partial goes to this CTA's second slot.
constexpr int kFirst = 1, kLast = 2, kBad = 4, kCut = 8, kSlot1 = 16;
// Block tables up to this size are prefetched into L2 at kernel start.
constexpr uint64_t kTablePrefetchMax = 16ull << 20;
constexpr int kSeqCache = 256;

// Element-type tag of FP8 (E4M3) pages: q and out are bf16, the pages hold
// codes standing for code * scale.
struct Fp8E4M3 {};

// One staged page: its sequence, visible tokens, flags, split-K partition;
// its physical block and first token in it; pad0 is the second block of a
// two-block page (-1: the page ends in its first block).
struct alignas(16) PageDesc {
  int32_t seq, ntok, flags, unit;  // unit: split-K partition index
  int32_t pb, toff, pad0, pad1;
};

// Tokens of sequence s this call attends to (all of them, or the suffix
// past the shared prefix in suffix mode).
__device__ __forceinline__ int32_t visible_len(const Params &p, int s) {
  return p.context_lens[s] - p.tok_offset;
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

// Start of the first unit whose midpoint lies at or after stream page x,
// where [P, P + v) are the pages of the sequence holding x and pp the pages
// of a full partition (split-K mode).
__device__ __forceinline__ int64_t unit_bound(int64_t x, int64_t P, int64_t v, int64_t pp) {
  const int64_t u = (x - P) / pp;
  const int64_t us = P + u * pp;
  const int64_t ue = P + ((u + 1) * pp < v ? (u + 1) * pp : v);
  return (us + ue >= 2 * x) ? us : ue;
}

struct alignas(16) Shared {
  uint64_t full[kMaxStages];
  uint64_t empty[kMaxStages];
  int64_t red[32];
  int64_t P_begin;
  int64_t range[2];  // split-K: this CTA's pages [range[0], range[1]) of the stream
  int32_t s_begin, vlb_begin, abort_flag, pad;
  // pa_decode mode, when the CTA's first sequence began in an earlier CTA:
  // the CTA holding its first page and that CTA's partial slot for it
  // (worked out in the prologue, so the producer divides nothing)
  int32_t first_cfirst, first_fslot, pad3[2];
  // Batches of up to kSeqCache sequences: context lengths and new-token
  // slots read once by the prologue, so that the producer never waits on a
  // global load of them behind its own bulk copies.
  int64_t slot_c[kSeqCache];
  int32_t ctx_c[kSeqCache];
};

// Four E4M3 codes (bytes 0..3 of x) to two fp16 pairs, exactly (every E4M3
// value, subnormals included, is an fp16 value): codes 0, 1 in lo, 2, 3 in hi,
// the lower-addressed code in the lower half.
__device__ __forceinline__ void e4m3x4_to_f16x4(uint32_t x, uint32_t &lo, uint32_t &hi) {
  asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %2;\n\t"
      "cvt.rn.f16x2.e4m3x2 %0, l;\n\tcvt.rn.f16x2.e4m3x2 %1, h;\n\t}"
      : "=r"(lo), "=r"(hi)
      : "r"(x));
}

// ===========================================================================
// bf16 consumer: tensor-core tiles of 16 tokens x 8 query heads.
// Lane (g = lane / 4, t = lane % 4) holds, for each 16-token tile, the scores
// of tokens g and g + 8 for query heads 2t and 2t + 1, and for each 16-wide
// d tile the output accumulator of d = 16 dt + g (+8) for the same two heads.
// ===========================================================================
// F16: FP8 pages.  The tensor-core fragments are built in registers from the
// staged codes (their exact fp16 values, see e4m3x4_to_f16x4), with q and P
// in fp16.  Inside the products head_dim is taken in another order, so
// that each lane reads whole 16-byte chunks of codes: in S = q K^T quad lane t
// owns d = 32t .. 32t + 31 (k step ks: d = 32t + 4ks + 0..3, q taken in the
// same order); in O^T the rows g and g + 8 of d tile k are d = 16g + 2k and
// 16g + 2k + 1.  The flush stores natural order.  Else bf16 tiles.
// PAIR: a page is two 8-token blocks, each landed as one box of [KV head][8
// tokens] rows per d half, the second box after the first.
template <int D, bool F16 = false, bool PAIR = false>
struct MmaConsumer {
  static constexpr int KS = D / 16;  // k steps of QK, d tiles of PV
  __device__ __forceinline__ static void mma(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                             uint32_t b1) {
    if constexpr (F16)
      mma_16816_f16(d, a, b0, b1);
    else
      mma_16816(d, a, b0, b1);
  }
  __device__ __forceinline__ static uint32_t pack(float lo, float hi) {
    return F16 ? pack_f16x2(lo, hi) : pack_bf16x2(lo, hi);
  }
  // bf16 pair -> the tile type (fp16 conversion of exact fp32 widening)
  __device__ __forceinline__ static uint32_t q_pair(uint32_t w) {
    if constexpr (F16)
      return pack_f16x2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
    else
      return w;
  }
  uint32_t qb[KS][2];                // Q^T as B operand (d x head), one pair per k step
  float o[KS][4];                    // O^T accumulators
  float m0_, m1_, l0, l1;            // running max / partial normaliser, heads 2t, 2t+1
  float scale_log2_;
  bool seg_bad;

  __device__ __forceinline__ void reset() {
#pragma unroll
    for (int k = 0; k < KS; ++k)
#pragma unroll
      for (int e = 0; e < 4; ++e) o[k][e] = 0.f;
    m0_ = m1_ = -INFINITY;
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
        if constexpr (F16) {
          qb[k][0] = q_pair(row[(t * (D / 4) + 4 * k) >> 1]);
          qb[k][1] = q_pair(row[(t * (D / 4) + 4 * k + 2) >> 1]);
        } else {
          qb[k][0] = q_pair(row[(k * 16 + t * 2) >> 1]);
          qb[k][1] = q_pair(row[(k * 16 + t * 2 + 8) >> 1]);
        }
      } else {
        qb[k][0] = qb[k][1] = 0u;
      }
    }
  }

  // One staged virtual page of `ntok` tokens.  Layouts:
  //  TL (tile): per 64-wide d half a box of [KV head][vbs tokens][128 B] rows
  //          with the 16-byte chunk index XORed with (row % 8) (128-byte
  //          swizzle); a tile's first row is a multiple of 16, so a lane's
  //          XOR term depends only on its own lane bits;
  //  padded: token rows `pitch` bytes apart, this head's slice at col_bytes.
  // Either way eight consecutive tokens at one chunk hit eight bank groups.
  // Tokens go in groups of NT (1 or 2) 16-token tiles that share one max
  // reduction and one rescale; each tile's QK runs as two independent MMA
  // chains, so the dependent-latency path per token is short.
  // Row of KV head h's token tk in a staged tile page (one d half).
  __device__ __forceinline__ static int tile_row(int h, int tk, const Params &p) {
    if constexpr (PAIR)
      return ((tk >> 3) * p.num_kv_heads + h) * 8 + (tk & 7);
    else
      return h * p.vbs + tk;
  }

  template <int NT, bool TL>
  __device__ __forceinline__ void tiles(const unsigned char *kp, const unsigned char *vp, int m0,
                                        int ntok, const Params &p, int h, int col_bytes,
                                        int lane) {
    const int g = lane >> 2, t = lane & 3;
    // K operand rows: token m0 + 16u + (lane & 15), chunk 2k + (lane >> 4)
    const int xk = ((lane >> 4) ^ (lane & 7)) << 4;   // TL: XOR term of chunk 2k
    const int ck = (lane >> 4) << 4;                  // padded: chunk offset
    // V operand rows (transposed load): token base + (lane & 7) + 8 * (lane >> 4),
    // chunk 2k + ((lane >> 3) & 1)
    const int mi = lane >> 3;
    const int xv = ((mi & 1) ^ (lane & 7)) << 4;
    const int cv = (mi & 1) << 4;
    float s[NT][4];
#pragma unroll
    for (int u = 0; u < NT; ++u) {
      const int tk = m0 + 16 * u + (lane & 15);
      const unsigned char *kr =
          TL ? kp + tile_row(h, tk, p) * 128 : kp + tk * p.row_pitch + col_bytes + ck;
      float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int k = 0; k < KS; k += 2) {
        uint32_t a[4], b[4];
        if (TL) {
          ldsm_x4(a, smem_u32(kr + (k >> 2) * p.box_bytes + ((((2 * k) & 7) << 4) ^ xk)));
          ldsm_x4(b, smem_u32(kr + ((k + 1) >> 2) * p.box_bytes +
                              ((((2 * k + 2) & 7) << 4) ^ xk)));
        } else {
          ldsm_x4(a, smem_u32(kr + k * 32));
          ldsm_x4(b, smem_u32(kr + (k + 1) * 32));
        }
        mma(sa, a, qb[k][0], qb[k][1]);
        mma(sb, b, qb[k + 1][0], qb[k + 1][1]);
      }
      const int r0 = m0 + 16 * u + g;
      const bool v0 = r0 < ntok, v1 = r0 + 8 < ntok;
      s[u][0] = v0 ? (sa[0] + sb[0]) * scale_log2_ : -INFINITY;
      s[u][1] = v0 ? (sa[1] + sb[1]) * scale_log2_ : -INFINITY;
      s[u][2] = v1 ? (sa[2] + sb[2]) * scale_log2_ : -INFINITY;
      s[u][3] = v1 ? (sa[3] + sb[3]) * scale_log2_ : -INFINITY;
    }
    float x0 = -INFINITY, x1 = -INFINITY;
#pragma unroll
    for (int u = 0; u < NT; ++u) {
      x0 = fmaxf(x0, fmaxf(s[u][0], s[u][2]));
      x1 = fmaxf(x1, fmaxf(s[u][1], s[u][3]));
    }
#pragma unroll
    for (int mask = 4; mask < 32; mask <<= 1) {
      x0 = fmaxf(x0, __shfl_xor_sync(0xffffffffu, x0, mask));
      x1 = fmaxf(x1, __shfl_xor_sync(0xffffffffu, x1, mask));
    }
    const float n0 = fmaxf(m0_, x0), n1 = fmaxf(m1_, x1);
    const float a0 = ex2(m0_ - n0), a1 = ex2(m1_ - n1);
    m0_ = n0;
    m1_ = n1;
    uint32_t pb[NT][2];
    float add0 = 0.f, add1 = 0.f;
#pragma unroll
    for (int u = 0; u < NT; ++u) {
      const float p0 = ex2(s[u][0] - n0), p1 = ex2(s[u][1] - n1);
      const float p2 = ex2(s[u][2] - n0), p3 = ex2(s[u][3] - n1);
      add0 += p0 + p2;
      add1 += p1 + p3;
      // P^T (16 tokens x 8 heads) as the B operand: transpose the two 8x8 tiles
      pb[u][0] = movmatrix_trans(pack(p0, p1));
      pb[u][1] = movmatrix_trans(pack(p2, p3));
    }
    l0 = l0 * a0 + add0;
    l1 = l1 * a1 + add1;
    if (!__all_sync(0xffffffffu, a0 == 1.f && a1 == 1.f)) {
#pragma unroll
      for (int k = 0; k < KS; ++k) {
        o[k][0] *= a0;
        o[k][1] *= a1;
        o[k][2] *= a0;
        o[k][3] *= a1;
      }
    }
#pragma unroll
    for (int u = 0; u < NT; ++u) {
      // V rows past ntok may hold anything (other tokens, never-written
      // shared memory): their P is 0 and their V elements are zeroed here so
      // that 0 * NaN cannot occur.
      const int base = m0 + 16 * u;
      uint32_t mlo = 0xffffffffu, mhi = 0xffffffffu;
      if (base + 16 > ntok) {
        mlo = (base + 2 * t < ntok ? 0x0000ffffu : 0u) | (base + 2 * t + 1 < ntok ? 0xffff0000u : 0u);
        mhi = (base + 2 * t + 8 < ntok ? 0x0000ffffu : 0u) |
              (base + 2 * t + 9 < ntok ? 0xffff0000u : 0u);
      }
      const int tv = base + (lane & 7) + ((mi >> 1) << 3);
      const unsigned char *vr =
          TL ? vp + tile_row(h, tv, p) * 128 : vp + tv * p.row_pitch + col_bytes + cv;
#pragma unroll
      for (int k = 0; k < KS; ++k) {
        uint32_t a[4];
        if (TL)
          ldsm_x4_trans(a, smem_u32(vr + (k >> 2) * p.box_bytes + ((((2 * k) & 7) << 4) ^ xv)));
        else
          ldsm_x4_trans(a, smem_u32(vr + k * 32));
        a[0] &= mlo;
        a[1] &= mlo;
        a[2] &= mhi;
        a[3] &= mhi;
        mma(o[k], a, pb[u][0], pb[u][1]);
      }
    }
  }

  template <bool TL>
  __device__ __forceinline__ void page_t(const unsigned char *kp, const unsigned char *vp,
                                         int ntok, const Params &p, int h, int col_bytes,
                                         int lane) {
    int m0 = 0;
    for (; m0 + 16 < ntok; m0 += 32) tiles<2, TL>(kp, vp, m0, ntok, p, h, col_bytes, lane);
    if (m0 < ntok) tiles<1, TL>(kp, vp, m0, ntok, p, h, col_bytes, lane);
  }

  __device__ __forceinline__ void page(const unsigned char *kp, const unsigned char *vp,
                                       int ntok, const Params &p, int h, int col_bytes,
                                       int lane) {
    if (p.tile)
      page_t<true>(kp, vp, ntok, p, h, col_bytes, lane);
    else
      page_t<false>(kp, vp, ntok, p, h, col_bytes, lane);
  }

  // FP8 pages (F16, head_dim 128): a page of up to 32 tokens of E4M3 codes,
  // in 16-token tiles; tile u of KV head h starts at row code_row(h, u) of
  // its tensor's staged rows (128 codes each, 16-byte chunk c of row r at
  // chunk c ^ (r % 8)): one box of [KV head][32 tokens], or (PAIR: two
  // 16-token blocks per page) one box of [KV head][16 tokens] per block.
  // The fragments come straight from the codes: for S a lane reads d chunks
  // 2t, 2t + 1 of tokens g and g + 8; for O^T d chunk g of tokens 2t, 2t + 1,
  // 2t + 8, 2t + 9, pairing the two tokens of each fragment register with a
  // byte permute.  The tiles of a page share one max and one rescale.
  __device__ __forceinline__ static int code_row(int h, int u, const Params &p) {
    if constexpr (PAIR)
      return (u * p.num_kv_heads + h) * 16;
    else
      return h * 32 + 16 * u;
  }

  __device__ __forceinline__ void page_codes(const unsigned char *kp, const unsigned char *vp,
                                             int ntok, const Params &p, int h, int lane) {
    if (ntok > 16)
      page_codes_t<2>(kp, vp, ntok, p, h, lane);
    else
      page_codes_t<1>(kp, vp, ntok, p, h, lane);
  }

  template <int NT>
  __device__ __forceinline__ void page_codes_t(const unsigned char *kp, const unsigned char *vp,
                                               int ntok, const Params &p, int h, int lane) {
    static_assert(D == 128, "FP8 pages: head_dim 128");
    const int g = lane >> 2, t = lane & 3;
    const int c0 = ((2 * t) ^ g) << 4, c1 = ((2 * t + 1) ^ g) << 4;
    float s[NT][4];
#pragma unroll
    for (int u = 0; u < NT; ++u) {
      const unsigned char *kr = kp + (code_row(h, u, p) + g) * 128;  // token g; g + 8 is 1 KB on
      const uint4 ka0 = *reinterpret_cast<const uint4 *>(kr + c0);
      const uint4 ka1 = *reinterpret_cast<const uint4 *>(kr + c1);
      const uint4 kb0 = *reinterpret_cast<const uint4 *>(kr + 1024 + c0);
      const uint4 kb1 = *reinterpret_cast<const uint4 *>(kr + 1024 + c1);
      const uint32_t wa[8] = {ka0.x, ka0.y, ka0.z, ka0.w, ka1.x, ka1.y, ka1.z, ka1.w};
      const uint32_t wb[8] = {kb0.x, kb0.y, kb0.z, kb0.w, kb1.x, kb1.y, kb1.z, kb1.w};
      float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int k = 0; k < KS; ++k) {
        uint32_t a[4];
        e4m3x4_to_f16x4(wa[k], a[0], a[2]);
        e4m3x4_to_f16x4(wb[k], a[1], a[3]);
        mma((k & 1) ? sb : sa, a, qb[k][0], qb[k][1]);
      }
      const int r0 = 16 * u + g;
      const bool v0 = r0 < ntok, v1 = r0 + 8 < ntok;
      s[u][0] = v0 ? (sa[0] + sb[0]) * scale_log2_ : -INFINITY;
      s[u][1] = v0 ? (sa[1] + sb[1]) * scale_log2_ : -INFINITY;
      s[u][2] = v1 ? (sa[2] + sb[2]) * scale_log2_ : -INFINITY;
      s[u][3] = v1 ? (sa[3] + sb[3]) * scale_log2_ : -INFINITY;
    }
    float x0 = -INFINITY, x1 = -INFINITY;
#pragma unroll
    for (int u = 0; u < NT; ++u) {
      x0 = fmaxf(x0, fmaxf(s[u][0], s[u][2]));
      x1 = fmaxf(x1, fmaxf(s[u][1], s[u][3]));
    }
#pragma unroll
    for (int mask = 4; mask < 32; mask <<= 1) {
      x0 = fmaxf(x0, __shfl_xor_sync(0xffffffffu, x0, mask));
      x1 = fmaxf(x1, __shfl_xor_sync(0xffffffffu, x1, mask));
    }
    const float n0 = fmaxf(m0_, x0), n1 = fmaxf(m1_, x1);
    const float a0 = ex2(m0_ - n0), a1 = ex2(m1_ - n1);
    m0_ = n0;
    m1_ = n1;
    uint32_t pb[NT][2];
    float add0 = 0.f, add1 = 0.f;
#pragma unroll
    for (int u = 0; u < NT; ++u) {
      const float p0 = ex2(s[u][0] - n0), p1 = ex2(s[u][1] - n1);
      const float p2 = ex2(s[u][2] - n0), p3 = ex2(s[u][3] - n1);
      add0 += p0 + p2;
      add1 += p1 + p3;
      // P^T (16 tokens x 8 heads) as the B operand
      pb[u][0] = movmatrix_trans(pack(p0, p1));
      pb[u][1] = movmatrix_trans(pack(p2, p3));
    }
    l0 = l0 * a0 + add0;
    l1 = l1 * a1 + add1;
    if (!__all_sync(0xffffffffu, a0 == 1.f && a1 == 1.f)) {
#pragma unroll
      for (int k = 0; k < KS; ++k) {
        o[k][0] *= a0;
        o[k][1] *= a1;
        o[k][2] *= a0;
        o[k][3] *= a1;
      }
    }
#pragma unroll
    for (int u = 0; u < NT; ++u) {
      // tokens past ntok may hold anything: their V codes are zeroed (P is 0)
      const int base = 16 * u;
      uint32_t mlo = 0xffffffffu, mhi = 0xffffffffu;
      if (base + 16 > ntok) {
        mlo = (base + 2 * t < ntok ? 0x0000ffffu : 0u) |
              (base + 2 * t + 1 < ntok ? 0xffff0000u : 0u);
        mhi = (base + 2 * t + 8 < ntok ? 0x0000ffffu : 0u) |
              (base + 2 * t + 9 < ntok ? 0xffff0000u : 0u);
      }
      const unsigned char *vr = vp + (code_row(h, u, p) + 2 * t) * 128;
      const int e0 = (g ^ (2 * t)) << 4, e1 = (g ^ (2 * t + 1)) << 4;
      const uint4 vx = *reinterpret_cast<const uint4 *>(vr + e0);         // token 2t
      const uint4 vy = *reinterpret_cast<const uint4 *>(vr + 128 + e1);   // 2t + 1
      const uint4 vz = *reinterpret_cast<const uint4 *>(vr + 1024 + e0);  // 2t + 8
      const uint4 vw = *reinterpret_cast<const uint4 *>(vr + 1152 + e1);  // 2t + 9
      const uint32_t xs[4] = {vx.x, vx.y, vx.z, vx.w}, ys[4] = {vy.x, vy.y, vy.z, vy.w};
      const uint32_t zs[4] = {vz.x, vz.y, vz.z, vz.w}, ws[4] = {vw.x, vw.y, vw.z, vw.w};
#pragma unroll
      for (int k = 0; k < KS; ++k) {
        // codes 2k, 2k + 1 of the chunk (d = 16g + 2k, + 1) of two tokens
        const uint32_t sel = (k & 1) ? 0x7362u : 0x5140u;
        uint32_t a[4];
        e4m3x4_to_f16x4(__byte_perm(xs[k >> 1], ys[k >> 1], sel), a[0], a[1]);
        e4m3x4_to_f16x4(__byte_perm(zs[k >> 1], ws[k >> 1], sel), a[2], a[3]);
        a[0] &= mlo;
        a[1] &= mlo;
        a[2] &= mhi;
        a[3] &= mhi;
        mma(o[k], a, pb[u][0], pb[u][1]);
      }
    }
  }

  // End of a segment: write out[...] directly (n_contrib == 1) or this CTA's
  // normalised partial for the merge kernel.  Two rounds of lane swaps turn
  // the MMA layout into four consecutive d per lane, so that every store
  // moves 16 bytes (fp32) or 8 bytes (bf16): with q = g % 4, an even-g lane
  // ends with head 2t and an odd-g lane with head 2t + 1, at d = 16k +
  // (g - q) + (q < 2 ? 0 : 8) .. + 3.
  template <typename Tout>
  __device__ __forceinline__ void flush(const Params &p, const PageDesc &d, int hq0, int nh,
                                        int c, int lane) {
    const int g = lane >> 2, t = lane & 3;
    float L0 = l0, L1 = l1;
#pragma unroll
    for (int mask = 4; mask < 32; mask <<= 1) {
      L0 += __shfl_xor_sync(0xffffffffu, L0, mask);
      L1 += __shfl_xor_sync(0xffffffffu, L1, mask);
    }
    const bool odd = g & 1;
    const int q = g & 3;
    const int hh = 2 * t + (odd ? 1 : 0);  // head of this lane's values
    // out_scale: 1, or V's scale for FP8 pages (the products saw the codes)
    const float inv = seg_bad ? 0.f : p.out_scale / (odd ? L1 : L0);
    // this lane's float4 k holds d = dcol + k * dstep .. + 3
    int dcol, dstep;
    float4 v[KS];
    if constexpr (F16) {
      // O^T row pairs: lane g holds d = 16g + 2k, + 1 of heads 2t, 2t + 1;
      // one exchange (lanes g, g ^ 1) leaves an even-g lane head 2t and an
      // odd-g lane head 2t + 1, each for d = 16 (g & ~1) .. + 31
      dcol = 16 * (g & ~1);
      dstep = 4;
      float lo[KS][2], hi[KS][2];
#pragma unroll
      for (int k = 0; k < KS; ++k) {
        const float s0 = __shfl_xor_sync(0xffffffffu, odd ? o[k][0] : o[k][1], 4);
        const float s2 = __shfl_xor_sync(0xffffffffu, odd ? o[k][2] : o[k][3], 4);
        lo[k][0] = odd ? s0 : o[k][0];
        lo[k][1] = odd ? s2 : o[k][2];
        hi[k][0] = odd ? o[k][1] : s0;
        hi[k][1] = odd ? o[k][3] : s2;
      }
#pragma unroll
      for (int j = 0; j < KS / 2; ++j) {
        v[j] = make_float4(lo[2 * j][0] * inv, lo[2 * j][1] * inv, lo[2 * j + 1][0] * inv,
                           lo[2 * j + 1][1] * inv);
        v[KS / 2 + j] = make_float4(hi[2 * j][0] * inv, hi[2 * j][1] * inv,
                                    hi[2 * j + 1][0] * inv, hi[2 * j + 1][1] * inv);
      }
    } else {
      dcol = (g - q) + (q < 2 ? 0 : 8);
      dstep = 16;
#pragma unroll
      for (int k = 0; k < KS; ++k) {
        // first exchange (lanes g, g ^ 1): pairs (d, d + 1) of one head, at +0 and +8
        const float s0 = __shfl_xor_sync(0xffffffffu, odd ? o[k][0] : o[k][1], 4);
        const float s2 = __shfl_xor_sync(0xffffffffu, odd ? o[k][2] : o[k][3], 4);
        const float lo0 = odd ? s0 : o[k][0], lo1 = odd ? o[k][1] : s0;
        const float hi0 = odd ? s2 : o[k][2], hi1 = odd ? o[k][3] : s2;
        // second exchange (lanes g, g ^ 2): q < 2 keeps the +0 pairs, q >= 2 the +8 pairs
        const float r0 = __shfl_xor_sync(0xffffffffu, q < 2 ? hi0 : lo0, 8);
        const float r1 = __shfl_xor_sync(0xffffffffu, q < 2 ? hi1 : lo1, 8);
        v[k] = q < 2 ? make_float4(lo0 * inv, lo1 * inv, r0 * inv, r1 * inv)
                     : make_float4(r0 * inv, r1 * inv, hi0 * inv, hi1 * inv);
      }
    }
    if (p.sk_o != nullptr) {
      // split-K: this partition's (max, normaliser, normalised output), the
      // max back in natural units
      const int64_t row = ((int64_t)d.seq * p.num_q_heads + hq0) * p.max_parts + d.unit;
      const int64_t mp = p.max_parts;
      if (g == 0) {
        if (2 * t < nh) {
          p.sk_max[row + 2 * t * mp] = m0_ * kLn2;
          p.sk_sum[row + 2 * t * mp] = seg_bad ? -1.f : L0;
        }
        if (2 * t + 1 < nh) {
          p.sk_max[row + (2 * t + 1) * mp] = m1_ * kLn2;
          p.sk_sum[row + (2 * t + 1) * mp] = seg_bad ? -1.f : L1;
        }
      }
      if (hh < nh) {
#pragma unroll
        for (int k = 0; k < KS; ++k)
          *reinterpret_cast<float4 *>(p.sk_o + (row + hh * mp) * D + k * dstep + dcol) = v[k];
      }
      return;
    }
    if (!(d.flags & kCut)) {
      if (p.seq_o != nullptr) {
        // suffix mode: the sequence's result as a partial for the prefix pass
        const int64_t row = (int64_t)d.seq * p.num_q_heads + hq0;
        if (g == 0) {
          if (2 * t < nh)
            reinterpret_cast<float2 *>(p.seq_ml)[row + 2 * t] = make_float2(m0_, seg_bad ? -1.f : L0);
          if (2 * t + 1 < nh)
            reinterpret_cast<float2 *>(p.seq_ml)[row + 2 * t + 1] =
                make_float2(m1_, seg_bad ? -1.f : L1);
        }
        if (hh < nh) {
#pragma unroll
          for (int k = 0; k < KS; ++k)
            *reinterpret_cast<float4 *>(p.seq_o + (row + hh) * D + k * dstep + dcol) = v[k];
        }
        return;
      }
      if (hh < nh) {
        const int64_t row = ((int64_t)d.seq * p.num_q_heads + hq0 + hh) * D;
#pragma unroll
        for (int k = 0; k < KS; ++k) Elem<Tout>::store4(p.out, row + k * dstep + dcol, v[k]);
      }
      return;
    }
    const int64_t prow = ((int64_t)c * 2 + ((d.flags & kSlot1) ? 1 : 0)) * p.num_q_heads + hq0;
    if (g == 0) {
      if (2 * t < nh)
        *reinterpret_cast<float2 *>(p.part_ml + (prow + 2 * t) * 2) =
            make_float2(m0_, seg_bad ? -1.f : L0);
      if (2 * t + 1 < nh)
        *reinterpret_cast<float2 *>(p.part_ml + (prow + 2 * t + 1) * 2) =
            make_float2(m1_, seg_bad ? -1.f : L1);
    }
    if (hh < nh) {
      float *row = p.part_o + (prow + hh) * D;
#pragma unroll
      for (int k = 0; k < KS; ++k) *reinterpret_cast<float4 *>(row + k * dstep + dcol) = v[k];
    }
    // merged by the last contributing CTA at its end
  }
};

// ===========================================================================
// bf16 consumer for large GQA / MQA groups (a multiple of 16 query heads per
// KV head): the warp's 16 query heads are the M side of the tensor-core
// tiles, so Q stays in registers as the A operand of S = Q K^T, the scores
// of one head sit in one lane quad (row statistics need two shuffles), and P
// is already the A operand of O += P V.  Lane (r = lane / 4, c = lane % 4)
// holds rows r and r + 8 (heads hq0 + r, hq0 + r + 8); score column
// (token) 8n + 2c (+1) of n tile n; output column d = 8j + 2c (+1) of d tile j.
// ===========================================================================
template <int D>
struct HeadRowConsumer {
  static constexpr int KS = D / 16;  // k steps of QK
  static constexpr int NJ = D / 8;   // d tiles of PV
  uint32_t qa[KS][4];                // Q (16 heads x D) as A fragments
  float o[NJ][4];                    // O (16 heads x D) accumulators
  float m0_, m1_, l0, l1;            // rows r, r + 8: running max, this lane's partial sum
  float scale_log2_;
  bool seg_bad;

  __device__ __forceinline__ void reset() {
#pragma unroll
    for (int j = 0; j < NJ; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) o[j][e] = 0.f;
    m0_ = m1_ = -INFINITY;
    l0 = l1 = 0.f;
    seg_bad = false;
  }

  __device__ __forceinline__ void load_q(const __nv_bfloat16 *qs, int hq0, int nh, int lane) {
    (void)nh;  // always 16
    const int r = lane >> 2, c = lane & 3;
    const uint32_t *row0 = reinterpret_cast<const uint32_t *>(qs + (size_t)(hq0 + r) * D);
    const uint32_t *row1 = reinterpret_cast<const uint32_t *>(qs + (size_t)(hq0 + r + 8) * D);
#pragma unroll
    for (int k = 0; k < KS; ++k) {
      qa[k][0] = row0[(k * 16 + 2 * c) >> 1];
      qa[k][1] = row1[(k * 16 + 2 * c) >> 1];
      qa[k][2] = row0[(k * 16 + 2 * c + 8) >> 1];
      qa[k][3] = row1[(k * 16 + 2 * c + 8) >> 1];
    }
  }

  // Shared-memory address of 16 bytes of token row `tok`, d chunk `ch`
  // (8 elements): TL = swizzled boxes [d half][KV head][vbs tokens][128 B],
  // else rows `row_pitch` apart with this head's slice at col_bytes.
  template <bool TL>
  __device__ __forceinline__ uint32_t row_addr(const unsigned char *base, int tok, int ch,
                                               const Params &p, int h, int col_bytes) const {
    if (TL)
      return smem_u32(base + (ch >> 3) * p.box_bytes + (h * p.vbs + tok) * 128 +
                      (((ch & 7) ^ (tok & 7)) << 4));
    return smem_u32(base + tok * p.row_pitch + col_bytes + ch * 16);
  }

  // Tokens [m0, m0 + 16 * NH) of a staged page (NH = 1 or 2 groups of 16),
  // ntok valid tokens in the page.
  template <int NH, bool TL>
  __device__ __forceinline__ void chunk(const unsigned char *kp, const unsigned char *vp, int m0,
                                        int ntok, const Params &p, int h, int col_bytes,
                                        int lane) {
    constexpr int NN = 2 * NH;  // n tiles of 8 tokens
    const int c = lane & 3;
    float s[NN][4];
#pragma unroll
    for (int n = 0; n < NN; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) s[n][e] = 0.f;
    // K rows as B operands: one ldmatrix.x4 gives two n tiles x one k step
    const int kt = (lane & 7) + ((lane >> 4) << 3);
    const int kc = (lane >> 3) & 1;
#pragma unroll
    for (int k = 0; k < KS; ++k) {
#pragma unroll
      for (int u = 0; u < NH; ++u) {
        uint32_t b[4];
        ldsm_x4(b, row_addr<TL>(kp, m0 + 16 * u + kt, 2 * k + kc, p, h, col_bytes));
        mma_16816(s[2 * u], qa[k], b[0], b[1]);
        mma_16816(s[2 * u + 1], qa[k], b[2], b[3]);
      }
    }
    // scale to log2 units, mask tokens past the page, row maxima
    float x0 = -INFINITY, x1 = -INFINITY;
#pragma unroll
    for (int n = 0; n < NN; ++n) {
      const int t0 = m0 + 8 * n + 2 * c;
      s[n][0] = t0 < ntok ? s[n][0] * scale_log2_ : -INFINITY;
      s[n][1] = t0 + 1 < ntok ? s[n][1] * scale_log2_ : -INFINITY;
      s[n][2] = t0 < ntok ? s[n][2] * scale_log2_ : -INFINITY;
      s[n][3] = t0 + 1 < ntok ? s[n][3] * scale_log2_ : -INFINITY;
      x0 = fmaxf(x0, fmaxf(s[n][0], s[n][1]));
      x1 = fmaxf(x1, fmaxf(s[n][2], s[n][3]));
    }
#pragma unroll
    for (int mask = 1; mask < 4; mask <<= 1) {
      x0 = fmaxf(x0, __shfl_xor_sync(0xffffffffu, x0, mask));
      x1 = fmaxf(x1, __shfl_xor_sync(0xffffffffu, x1, mask));
    }
    const float n0 = fmaxf(m0_, x0), n1 = fmaxf(m1_, x1);
    const float a0 = ex2(m0_ - n0), a1 = ex2(m1_ - n1);
    m0_ = n0;
    m1_ = n1;
    uint32_t pa[NH][4];
    float add0 = 0.f, add1 = 0.f;
#pragma unroll
    for (int n = 0; n < NN; ++n) {
      const float p0 = ex2(s[n][0] - n0), p1 = ex2(s[n][1] - n0);
      const float p2 = ex2(s[n][2] - n1), p3 = ex2(s[n][3] - n1);
      add0 += p0 + p1;
      add1 += p2 + p3;
      pa[n >> 1][(n & 1) * 2 + 0] = pack_bf16x2(p0, p1);
      pa[n >> 1][(n & 1) * 2 + 1] = pack_bf16x2(p2, p3);
    }
    l0 = l0 * a0 + add0;
    l1 = l1 * a1 + add1;
    if (!__all_sync(0xffffffffu, a0 == 1.f && a1 == 1.f)) {
#pragma unroll
      for (int j = 0; j < NJ; ++j) {
        o[j][0] *= a0;
        o[j][1] *= a0;
        o[j][2] *= a1;
        o[j][3] *= a1;
      }
    }
    // V rows as B operands (transposed): one ldmatrix.x4 gives two d tiles
    // x one 16-token k step.  V rows past ntok may hold anything; their P is
    // 0 and their values are zeroed here so that 0 * NaN cannot occur.
    const int vt = (lane & 7) + (((lane >> 3) & 1) << 3);
    const int vc = lane >> 4;
#pragma unroll
    for (int u = 0; u < NH; ++u) {
      const int base = m0 + 16 * u;
      uint32_t mk0 = 0xffffffffu, mk1 = 0xffffffffu;
      if (base + 16 > ntok) {
        mk0 = (base + 2 * c < ntok ? 0x0000ffffu : 0u) | (base + 2 * c + 1 < ntok ? 0xffff0000u : 0u);
        mk1 = (base + 2 * c + 8 < ntok ? 0x0000ffffu : 0u) |
              (base + 2 * c + 9 < ntok ? 0xffff0000u : 0u);
      }
#pragma unroll
      for (int jj = 0; jj < NJ / 2; ++jj) {
        uint32_t b[4];
        ldsm_x4_trans(b, row_addr<TL>(vp, base + vt, 2 * jj + vc, p, h, col_bytes));
        b[0] &= mk0;
        b[1] &= mk1;
        b[2] &= mk0;
        b[3] &= mk1;
        mma_16816(o[2 * jj], pa[u], b[0], b[1]);
        mma_16816(o[2 * jj + 1], pa[u], b[2], b[3]);
      }
    }
  }

  template <bool TL>
  __device__ __forceinline__ void page_t(const unsigned char *kp, const unsigned char *vp,
                                         int ntok, const Params &p, int h, int col_bytes,
                                         int lane) {
    int m0 = 0;
    for (; m0 + 16 < ntok; m0 += 32) chunk<2, TL>(kp, vp, m0, ntok, p, h, col_bytes, lane);
    if (m0 < ntok) chunk<1, TL>(kp, vp, m0, ntok, p, h, col_bytes, lane);
  }

  __device__ __forceinline__ void page(const unsigned char *kp, const unsigned char *vp,
                                       int ntok, const Params &p, int h, int col_bytes,
                                       int lane) {
    if (p.tile)
      page_t<true>(kp, vp, ntok, p, h, col_bytes, lane);
    else
      page_t<false>(kp, vp, ntok, p, h, col_bytes, lane);
  }

  // End of a segment: out[...] directly (n_contrib == 1) or this CTA's
  // normalised partial for the merge kernel.
  template <typename Tout>
  __device__ __forceinline__ void flush(const Params &p, const PageDesc &d, int hq0, int nh,
                                        int c_idx, int lane) {
    (void)nh;
    const int r = lane >> 2, c = lane & 3;
    float L0 = l0, L1 = l1;
#pragma unroll
    for (int mask = 1; mask < 4; mask <<= 1) {
      L0 += __shfl_xor_sync(0xffffffffu, L0, mask);
      L1 += __shfl_xor_sync(0xffffffffu, L1, mask);
    }
    const float i0 = seg_bad ? 0.f : p.out_scale / L0, i1 = seg_bad ? 0.f : p.out_scale / L1;
    if (p.sk_o != nullptr) {
      // split-K: this partition's (max, normaliser, normalised output)
      const int64_t mp = p.max_parts;
      const int64_t ix0 = ((int64_t)d.seq * p.num_q_heads + hq0 + r) * mp + d.unit;
      const int64_t ix1 = ix0 + 8 * mp;
      if (c == 0) {
        p.sk_max[ix0] = m0_ * kLn2;
        p.sk_sum[ix0] = seg_bad ? -1.f : L0;
        p.sk_max[ix1] = m1_ * kLn2;
        p.sk_sum[ix1] = seg_bad ? -1.f : L1;
      }
#pragma unroll
      for (int j = 0; j < NJ; ++j) {
        *reinterpret_cast<float2 *>(p.sk_o + ix0 * D + 8 * j + 2 * c) =
            make_float2(o[j][0] * i0, o[j][1] * i0);
        *reinterpret_cast<float2 *>(p.sk_o + ix1 * D + 8 * j + 2 * c) =
            make_float2(o[j][2] * i1, o[j][3] * i1);
      }
      return;
    }
    if (!(d.flags & kCut) && p.seq_o != nullptr) {
      // suffix mode: the sequence's result as a partial for the prefix pass
      const int64_t row = (int64_t)d.seq * p.num_q_heads + hq0 + r;
      if (c == 0) {
        reinterpret_cast<float2 *>(p.seq_ml)[row] = make_float2(m0_, seg_bad ? -1.f : L0);
        reinterpret_cast<float2 *>(p.seq_ml)[row + 8] = make_float2(m1_, seg_bad ? -1.f : L1);
      }
#pragma unroll
      for (int j = 0; j < NJ; ++j) {
        *reinterpret_cast<float2 *>(p.seq_o + row * D + 8 * j + 2 * c) =
            make_float2(o[j][0] * i0, o[j][1] * i0);
        *reinterpret_cast<float2 *>(p.seq_o + (row + 8) * D + 8 * j + 2 * c) =
            make_float2(o[j][2] * i1, o[j][3] * i1);
      }
      return;
    }
    if (!(d.flags & kCut)) {
      const int64_t row0 = ((int64_t)d.seq * p.num_q_heads + hq0 + r) * D;
      const int64_t row1 = row0 + 8 * D;
#pragma unroll
      for (int j = 0; j < NJ; ++j) {
        Elem<Tout>::store2(p.out, row0 + 8 * j + 2 * c, o[j][0] * i0, o[j][1] * i0);
        Elem<Tout>::store2(p.out, row1 + 8 * j + 2 * c, o[j][2] * i1, o[j][3] * i1);
      }
      return;
    }
    const int64_t prow =
        ((int64_t)c_idx * 2 + ((d.flags & kSlot1) ? 1 : 0)) * p.num_q_heads + hq0;
    if (c == 0) {
      *reinterpret_cast<float2 *>(p.part_ml + (prow + r) * 2) =
          make_float2(m0_, seg_bad ? -1.f : L0);
      *reinterpret_cast<float2 *>(p.part_ml + (prow + r + 8) * 2) =
          make_float2(m1_, seg_bad ? -1.f : L1);
    }
    float *orow0 = p.part_o + (prow + r) * D;
    float *orow1 = p.part_o + (prow + r + 8) * D;
#pragma unroll
    for (int j = 0; j < NJ; ++j) {
      *reinterpret_cast<float2 *>(orow0 + 8 * j + 2 * c) = make_float2(o[j][0] * i0, o[j][1] * i0);
      *reinterpret_cast<float2 *>(orow1 + 8 * j + 2 * c) = make_float2(o[j][2] * i1, o[j][3] * i1);
    }
    // merged by the last contributing CTA at its end
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
                                        int lane) {
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
    if (p.sk_o != nullptr) {
      // split-K: this partition's (max, normaliser, normalised output)
      const int64_t mp = p.max_parts;
      if (lane < G) {
        const int64_t ix = (orow + lane) * mp + d.unit;
        p.sk_max[ix] = m_run * kLn2;
        p.sk_sum[ix] = seg_bad ? -1.f : lsum;
      }
      if (tg == 0) {
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
          for (int e = 0; e < EPV; ++e)
            p.sk_o[((orow + g) * mp + d.unit) * D + j * EPV + e] =
                seg_bad ? 0.f : ac[g][e] / lg[g];
      }
      return;
    }
    if (!(d.flags & kCut)) {
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
    const int64_t prow = ((int64_t)c * 2 + ((d.flags & kSlot1) ? 1 : 0)) * p.num_q_heads + hq0;
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
    // merged by the last contributing CTA at its end
  }
};

// ===========================================================================
// Walk over a CTA's virtual pages in stream order (all lanes of the producer
// warp in lock step).  Context lengths and block-table entries are fetched 32
// at a time into lane registers; the current page's values are shuffled out.
// ===========================================================================
struct PageWalker {
  int32_t s, vlb, ctx_s, pages_s;
  int32_t cw, cw_ctx;             // context-length window: lane l holds sequence cw + l
  int32_t tw_seq, tw_lb, tw_val;  // table window: lane l holds entry tw_lb + l of tw_seq
  int64_t cw_slot, slot_s;        // fused write: slot of sequence cw + l; of sequence s
  int32_t tn_seq, tn_lb, tn_val;  // next table window, loading ahead of use
  int64_t P_s, cursor;

  const Shared *shc;  // context lengths / slots cached in shared memory, or NULL

  __device__ __forceinline__ void load_window(const Params &p, int lane) {
    const bool in = cw + lane < p.batch;
    if (shc != nullptr) {
      cw_ctx = in ? shc->ctx_c[cw + lane] : 0;
      cw_slot = in ? shc->slot_c[cw + lane] : -1;
    } else {
      cw_ctx = in ? visible_len(p, cw + lane) : 0;
      cw_slot = (in && p.slot_mapping != nullptr) ? p.slot_mapping[cw + lane] : -1;
    }
  }
  // Fused write: when this CTA owns the sequence's last page, start moving
  // the new token's rows towards L2 now; they are copied at that page.
  __device__ __forceinline__ void prefetch_new_rows(const Params &p, int64_t end, int lane) {
    if (p.slot_mapping != nullptr && lane == 0 && slot_s >= 0 && P_s + pages_s <= end) {
      const int64_t in_row = (p.fp8 ? 2 : 1) * (int64_t)p.row_bytes;  // fp8: bf16 rows
      const int64_t off = (int64_t)s * in_row;
      prefetch_l2(static_cast<const unsigned char *>(p.k_new) + off, (uint32_t)in_row);
      prefetch_l2(static_cast<const unsigned char *>(p.v_new) + off, (uint32_t)in_row);
    }
  }
  __device__ __forceinline__ void init(const Params &p, const Shared *cache, int32_t s0,
                                       int32_t vlb0, int64_t P0, int64_t cur0, int64_t end,
                                       int lane) {
    shc = cache;
    s = s0;
    vlb = vlb0;
    P_s = P0;
    cursor = cur0;
    cw = s0;
    load_window(p, lane);
    ctx_s = __shfl_sync(0xffffffffu, cw_ctx, 0);
    slot_s = __shfl_sync(0xffffffffu, cw_slot, 0);
    pages_s = vpages_of(ctx_s, p);
    tw_seq = -1;
    tw_lb = 0;
    tw_val = -1;
    tn_seq = -1;
    tn_lb = 0;
    tn_val = -1;
    prefetch_new_rows(p, end, lane);
  }
  // Block-table window (32 entries of one sequence from entry lb) into lane
  // registers: the load is only issued here, and waited for at first use.
  __device__ __forceinline__ int32_t load_table(const Params &p, int32_t seq, int32_t lb,
                                                int lane) const {
    const int32_t e = lb + lane;
    return (e < p.max_blocks) ? p.block_tables[(int64_t)seq * p.table_stride + e] : -1;
  }
  // Start loading the window after the current one: the rest of a long
  // sequence, else the next sequence with visible pages, looked up in the
  // cached context lengths (nothing is prefetched without the cache).
  __device__ __forceinline__ void prefetch_next_window(const Params &p, int64_t end,
                                                       int lane) {
    const int32_t blocks = (ctx_s + p.block_size - 1) >> p.log2_bs;
    if (tw_lb + 32 < blocks) {
      tn_seq = s;
      tn_lb = tw_lb + 32;
    } else {
      if (shc == nullptr) return;
      const int64_t next_page = P_s + pages_s;  // stream index of the next sequence's page
      if (next_page >= end) return;             // this CTA's range ends first
      int32_t n = s + 1;
      while (n < p.batch && n < s + 33 && vpages_of(shc->ctx_c[n], p) == 0) ++n;
      if (n >= p.batch || n >= s + 33) return;
      tn_seq = n;
      tn_lb = 0;
    }
    tn_val = load_table(p, tn_seq, tn_lb, lane);
  }
  // Physical block of the current page.
  __device__ __forceinline__ int32_t block(const Params &p, int64_t end, int lane) {
    const int32_t lb = vlb >> p.log2_vpp;
    if (s != tw_seq || lb >= tw_lb + 32) {
      if (s == tn_seq && lb >= tn_lb && lb < tn_lb + 32) {
        tw_val = tn_val;  // prefetched
        tw_lb = tn_lb;
      } else {
        tw_lb = lb;
        tw_val = load_table(p, s, lb, lane);
      }
      tw_seq = s;
      tn_seq = -1;
      prefetch_next_window(p, end, lane);
    }
    return __shfl_sync(0xffffffffu, tw_val, lb - tw_lb);
  }
  // Two-block pages: the physical blocks of the current 16-token page
  // (entries 2 vlb and 2 vlb + 1; windows start at even entries, so both sit
  // in one window).
  __device__ __forceinline__ int32_t block_pair(const Params &p, int64_t end, int lane,
                                                int32_t &pb2) {
    const int32_t lb = vlb << 1;
    if (s != tw_seq || lb >= tw_lb + 32) {
      if (s == tn_seq && lb >= tn_lb && lb < tn_lb + 32) {
        tw_val = tn_val;  // prefetched
        tw_lb = tn_lb;
      } else {
        tw_lb = lb;
        tw_val = load_table(p, s, lb, lane);
      }
      tw_seq = s;
      tn_seq = -1;
      prefetch_next_window(p, end, lane);
    }
    pb2 = __shfl_sync(0xffffffffu, tw_val, lb + 1 - tw_lb);
    return __shfl_sync(0xffffffffu, tw_val, lb - tw_lb);
  }
  __device__ __forceinline__ int32_t ntok(const Params &p) const {
    return min(p.vbs, ctx_s - vlb * p.vbs);
  }
  // Next page of the stream (skips sequences without pages).
  __device__ __forceinline__ void advance(const Params &p, int64_t end, int lane) {
    ++cursor;
    ++vlb;
    if (vlb == pages_s && cursor < end) {
      int32_t nxt = s + 1;
      for (;;) {
        if (nxt >= cw + 32) {
          cw = nxt;
          load_window(p, lane);
        }
        const bool has =
            (cw + lane >= nxt) && (cw + lane < p.batch) && vpages_of(cw_ctx, p) > 0;
        const uint32_t m = __ballot_sync(0xffffffffu, has);
        if (m) {
          const int l = __ffs(m) - 1;
          nxt = cw + l;
          ctx_s = __shfl_sync(0xffffffffu, cw_ctx, l);
          slot_s = __shfl_sync(0xffffffffu, cw_slot, l);
          break;
        }
        nxt = cw + 32;
      }
      P_s += pages_s;
      s = nxt;
      vlb = 0;
      pages_s = vpages_of(ctx_s, p);
      prefetch_new_rows(p, end, lane);
    }
  }
};

// Fused cache write of sequence s's new token to `slot` (all lanes of the
// producer warp): row_bytes of K and of V, 16-byte vectors, loads batched
// ahead of the stores.  Each lane then fences its stores against the tensor
// copy that will read the page back.
__device__ __forceinline__ void write_new_rows(const Params &p, int32_t s, int64_t slot,
                                               int lane) {
  const int n = p.row_bytes >> 4;
  const uint4 *ks = reinterpret_cast<const uint4 *>(static_cast<const unsigned char *>(p.k_new) +
                                                    (int64_t)s * p.row_bytes);
  const uint4 *vs = reinterpret_cast<const uint4 *>(static_cast<const unsigned char *>(p.v_new) +
                                                    (int64_t)s * p.row_bytes);
  uint4 *kd = reinterpret_cast<uint4 *>(static_cast<unsigned char *>(p.key_cache) +
                                        slot * p.row_bytes);
  uint4 *vd = reinterpret_cast<uint4 *>(static_cast<unsigned char *>(p.value_cache) +
                                        slot * p.row_bytes);
  for (int x0 = lane; x0 < n; x0 += 4 * 32) {
    uint4 a[4], b[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int x = x0 + 32 * u;
      if (x < n) {
        a[u] = __ldg(ks + x);
        b[u] = __ldg(vs + x);
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int x = x0 + 32 * u;
      if (x < n) {
        kd[x] = a[u];
        vd[x] = b[u];
      }
    }
  }
  fence_proxy_async_global();
}

// FP8 pages: the new token's bf16 rows (2 * row_bytes bytes each) divided
// by the tensors' scales and quantised to E4M3 codes in its slot (row_bytes
// codes), 16 elements per lane step; then the same fence.
__device__ __forceinline__ void write_new_rows_fp8(const Params &p, int32_t s, int64_t slot,
                                                   int lane) {
  const int groups = p.row_bytes >> 4;
  const uint4 *ks = reinterpret_cast<const uint4 *>(static_cast<const unsigned char *>(p.k_new) +
                                                    (int64_t)s * 2 * p.row_bytes);
  const uint4 *vs = reinterpret_cast<const uint4 *>(static_cast<const unsigned char *>(p.v_new) +
                                                    (int64_t)s * 2 * p.row_bytes);
  uint4 *kd = reinterpret_cast<uint4 *>(static_cast<unsigned char *>(p.key_cache) +
                                        slot * p.row_bytes);
  uint4 *vd = reinterpret_cast<uint4 *>(static_cast<unsigned char *>(p.value_cache) +
                                        slot * p.row_bytes);
  for (int x = lane; x < groups; x += 32) {
    const uint4 k0 = __ldg(ks + 2 * x), k1 = __ldg(ks + 2 * x + 1);
    const uint4 v0 = __ldg(vs + 2 * x), v1 = __ldg(vs + 2 * x + 1);
    kd[x] = bf16x16_to_e4m3(k0, k1, p.k_scale);
    vd[x] = bf16x16_to_e4m3(v0, v1, p.v_scale);
  }
  fence_proxy_async_global();
}

// ===========================================================================
// The kernel.  T = element type; D = head_dim; G = query heads per KV head
// for the fp32 consumer; for bf16, G = 16 selects the head-row consumer (16
// heads per warp) and G = 0 the token-row one (up to 8 heads per warp);
// NCW = consumer warps.
// ===========================================================================
template <typename T, int D, int G, int NCW, bool PAIR = false>
__global__ void __launch_bounds__((NCW + 1) * 32, 1)
    decode_stream_kernel(const __grid_constant__ Params p) {
  // T: __nv_bfloat16, float, or Fp8E4M3 (FP8 pages; q and out bf16)
  constexpr bool kFp8 = std::is_same<T, Fp8E4M3>::value;
  constexpr bool kMma = std::is_same<T, __nv_bfloat16>::value || kFp8;
  using TA = typename std::conditional<kFp8, __nv_bfloat16, T>::type;  // q, out
  constexpr int kFmaG = kMma ? 1 : (G > 0 ? G : 1);  // fp32 consumer's group
  constexpr int kScoreFloats = kMma ? 1 : FmaConsumer<TA, D, kFmaG>::E;
  static_assert(sizeof(Shared) + sizeof(PageDesc) * kMaxStages * kMaxPPS +
                        sizeof(float) * NCW * kScoreFloats <= kHdrBytes,
                "header region");
  static_assert(sizeof(Shared) % 16 == 0 && sizeof(PageDesc) % 16 == 0,
                "descriptors and score buffers need 16-byte alignment");
  using MmaCons =
      typename std::conditional<G == 16, HeadRowConsumer<D>, MmaConsumer<D, kFp8, PAIR>>::type;
  using Cons = typename std::conditional<kMma, MmaCons, FmaConsumer<TA, D, kFmaG>>::type;
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
  // Hints first (they read nothing into registers): the tensor maps, and this
  // CTA's share of the block table into L2, so that the first table lookups
  // after the scan of context lengths hit L2.
  if (tid == 0 && p.tile) {
    prefetch_tensormap(&p.tmap_k);
    prefetch_tensormap(&p.tmap_v);
  }
  if (tid == 32) {
    const uint64_t bytes = (uint64_t)p.batch * (uint64_t)p.max_blocks * 4u;
    if (bytes <= kTablePrefetchMax) {
      const uint64_t base = reinterpret_cast<uint64_t>(p.block_tables);
      const uint64_t chunk = ((bytes + p.grid - 1) / p.grid + 15) & ~15ull;
      uint64_t lo = base + (uint64_t)c * chunk, hi = lo + chunk;
      if (hi > base + bytes) hi = base + bytes;
      lo = (lo + 15) & ~15ull;
      hi &= ~15ull;
      if (hi > lo) prefetch_l2(reinterpret_cast<const void *>(lo), (uint32_t)(hi - lo));
    }
  }
  // Launched with programmatic stream serialisation: this CTA may start
  // while the previous kernel of the stream still runs.  Nothing it reads or
  // writes is touched before that kernel has finished and flushed.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  // the merge kernel that follows may be scheduled now; it waits for this grid
  asm volatile("griddepcontrol.launch_dependents;");

  if (tid == 0) {
    for (int i = 0; i < p.stages; ++i) {
      mbar_init(&sh.full[i], 1);
      mbar_init(&sh.empty[i], NCW);
    }
    sh.abort_flag = 0;
    sh.range[0] = sh.range[1] = 0;
    // make the initialised barriers visible to the bulk-copy (async) proxy
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }

  // ---- Prologue: pages per sequence, the stream's total T, this CTA's
  // range [start, end) of it and the sequence / page it starts at.
  //   pa_decode: ranges of equal page counts; units (sequences) may be cut.
  //   split-K: unit boundaries nearest to the equal cuts (a unit goes to the
  //   CTA whose share holds its midpoint); no unit is cut.
  const bool splitk = p.sk_o != nullptr;
  const int32_t pp = splitk ? p.part_pages : 0;  // pages per split-K partition
  int64_t Tp, start = 0, end = 0;
  int32_t g_eff;
  const bool cached = p.batch <= kSeqCache;
  if (p.batch <= (int)blockDim.x) {
    // one scan gives both the total and every sequence's first page
    int32_t ctx = 0;
    if (tid < p.batch) {
      ctx = visible_len(p, tid);
      if (cached) {
        sh.ctx_c[tid] = ctx;
        sh.slot_c[tid] = (p.slot_mapping != nullptr) ? p.slot_mapping[tid] : -1;
      }
    }
    const int64_t v = (tid < p.batch) ? vpages_of(ctx, p) : 0;
    const int64_t P = block_exclusive_scan(v, sh.red, &Tp);
    if (splitk) {
      g_eff = p.grid;
      const int64_t x0 = (int64_t)c * Tp / g_eff, x1 = (int64_t)(c + 1) * Tp / g_eff;
      if (v > 0 && P <= x0 && x0 < P + v) sh.range[0] = unit_bound(x0, P, v, pp);
      if (v > 0 && P <= x1 && x1 < P + v) sh.range[1] = unit_bound(x1, P, v, pp);
      if (tid == 0 && x1 >= Tp) sh.range[1] = Tp;
      __syncthreads();
      start = sh.range[0];
      end = sh.range[1];
    } else {
      g_eff = (int32_t)((Tp < p.grid) ? Tp : p.grid);
      if (c < g_eff) {
        start = (int64_t)c * Tp / g_eff;
        end = (int64_t)(c + 1) * Tp / g_eff;
      }
    }
    if (start < end && v > 0 && P <= start && start < P + v) {
      sh.s_begin = tid;
      sh.vlb_begin = (int32_t)(start - P);
      sh.P_begin = P;
      if (!splitk && P < start) {
        const int32_t cf = owner_of(P, Tp, g_eff);
        sh.first_cfirst = cf;
        sh.first_fslot = ((int64_t)cf * Tp / g_eff < P) ? 1 : 0;
      }
    }
  } else {
    int64_t T_loc = 0;
    for (int base = 0; base < p.batch; base += blockDim.x) {
      const int s = base + tid;
      int32_t ctx = 0;
      if (s < p.batch) {
        ctx = visible_len(p, s);
        if (cached) {
          sh.ctx_c[s] = ctx;
          sh.slot_c[s] = (p.slot_mapping != nullptr) ? p.slot_mapping[s] : -1;
        }
      }
      const int64_t v = (s < p.batch) ? vpages_of(ctx, p) : 0;
      T_loc += block_sum(v, sh.red);
    }
    Tp = T_loc;
    if (splitk) {
      g_eff = p.grid;
      const int64_t x0 = (int64_t)c * Tp / g_eff, x1 = (int64_t)(c + 1) * Tp / g_eff;
      int64_t run = 0;
      for (int base = 0; base < p.batch; base += blockDim.x) {
        const int s = base + tid;
        const int64_t v = (s < p.batch) ? vpages_of(visible_len(p, s), p) : 0;
        int64_t tot;
        const int64_t P = run + block_exclusive_scan(v, sh.red, &tot);
        if (v > 0 && P <= x0 && x0 < P + v) sh.range[0] = unit_bound(x0, P, v, pp);
        if (v > 0 && P <= x1 && x1 < P + v) sh.range[1] = unit_bound(x1, P, v, pp);
        run += tot;
        if (run > x1) break;  // uniform: every thread sees the same `run`
      }
      if (tid == 0 && x1 >= Tp) sh.range[1] = Tp;
      __syncthreads();
      start = sh.range[0];
      end = sh.range[1];
    } else {
      g_eff = (int32_t)((Tp < p.grid) ? Tp : p.grid);
      if (c < g_eff) {
        start = (int64_t)c * Tp / g_eff;
        end = (int64_t)(c + 1) * Tp / g_eff;
      }
    }
    if (start < end) {
      int64_t run = 0;
      for (int base = 0; base < p.batch; base += blockDim.x) {
        const int s = base + tid;
        const int64_t v = (s < p.batch) ? vpages_of(visible_len(p, s), p) : 0;
        int64_t tot;
        const int64_t P = run + block_exclusive_scan(v, sh.red, &tot);
        if (v > 0 && P <= start && start < P + v) {
          sh.s_begin = s;
          sh.vlb_begin = (int32_t)(start - P);
          sh.P_begin = P;
          if (!splitk && P < start) {
            const int32_t cf = owner_of(P, Tp, g_eff);
            sh.first_cfirst = cf;
            sh.first_fslot = ((int64_t)cf * Tp / g_eff < P) ? 1 : 0;
          }
        }
        run += tot;
        if (run > start) break;  // uniform: every thread sees the same `run`
      }
    }
  }
  const bool active = start < end;
  __syncthreads();

  const bool per_row = p.row_pitch != p.row_bytes;
  if (active) {
    const int n_stages = (int)((end - start + p.pps - 1) / p.pps);
    if (warp == 0) {
      // ===================== producer =====================
      const int nbox = kFp8 ? 1 : p.n_dhalf;  // tensor copies per page and tensor
      PageWalker wk;
      wk.init(p, cached ? &sh : nullptr, sh.s_begin, sh.vlb_begin, sh.P_begin, start, end,
              lane);
      bool ok = true;
      int issued = 0;
      // pages are read once: they go to L2 with evict-first priority, so that
      // the block tables, the partials and the merge records stay there
      const uint64_t kv_policy = l2_evict_first_policy();
      // split-K: the partition of the current page and the pages left in it
      // (CTA ranges start on partition boundaries), kept without a division
      int32_t u_cur = pp > 0 ? sh.vlb_begin / pp : 0, u_left = pp;
      // stage slot and how many times the ring went round (no divisions)
      int slot = -1, round = 0;
      for (int i = 0; i < n_stages && ok; ++i) {
        if (++slot == p.stages) {
          slot = 0;
          ++round;
        }
        if (round > 0) {
          ok = __all_sync(0xffffffffu,
                          mbar_wait(&sh.empty[slot], (round - 1) & 1, &sh.abort_flag));
          if (!ok) break;
        }
        const int npg = (int)min((int64_t)p.pps, end - wk.cursor);
        uint32_t bytes = 0;
        bool wrote = false;
        for (int k = 0; k < npg; ++k) {
          int32_t pb2 = -1;  // two-block pages: the second block, if the page reaches it
          const int32_t pb = PAIR ? wk.block_pair(p, end, lane, pb2) : wk.block(p, end, lane);
          const int32_t ntok = wk.ntok(p);
          if (PAIR && ntok <= p.block_size) pb2 = -1;
          const bool first = (wk.vlb == 0) || (wk.cursor == start);
          const bool seq_last = wk.vlb == wk.pages_s - 1;
          // split-K: a partition ends every pp pages (ranges end on unit ends)
          const bool last = seq_last || (wk.cursor == end - 1) || u_left == 1;
          const bool bad_block =
              pb < 0 || pb >= p.num_blocks ||
              (PAIR && ntok > p.block_size && (pb2 < 0 || pb2 >= p.num_blocks));
          bool bad = bad_block;
          if (bad_block && lane == 0) set_error(p.err_word, PA_DEVERR_BLOCK_ID);
          if (p.slot_mapping != nullptr && seq_last && wk.slot_s >= 0) {
            // Fused cache write: the new token sits at position ctx - 1, in
            // this page; its slot must be the one the table gives it, else
            // nothing is stored and the sequence's output is zeroed.
            const int32_t pos = wk.ctx_s - 1;
            // the block holding pos
            const int32_t pbw = (PAIR && ((pos >> p.log2_bs) & 1)) ? pb2 : pb;
            const int64_t want = (int64_t)pbw * p.block_size + (pos & (p.block_size - 1));
            if (!bad_block && wk.slot_s == want) {
              if constexpr (kFp8)
                write_new_rows_fp8(p, wk.s, want, lane);
              else
                write_new_rows(p, wk.s, want, lane);
              wrote = true;
            } else {
              bad = true;
              if (lane == 0) set_error(p.err_word, PA_DEVERR_SLOT);
            }
          }
          if (lane == 0) {
            PageDesc d;
            d.seq = wk.s;
            d.ntok = ntok;
            d.unit = u_cur;
            d.pb = pb;
            d.toff = PAIR ? 0 : (wk.vlb & ((1 << p.log2_vpp) - 1)) * p.vbs;
            d.pad0 = pb2;
            d.pad1 = 0;
            int32_t flags = (first ? kFirst : 0) | (last ? kLast : 0) | (bad ? kBad : 0);
            if (last && pp == 0) {
              // is the sequence cut between CTAs (it began before this CTA's
              // range or runs past it)?  Then this CTA leaves a partial in
              // its slot 0 (the sequence holds the CTA's first page) or 1
              // (it starts inside the range and runs past it).
              const bool before = wk.P_s < start;
              if (before || !seq_last) flags |= kCut | ((start < wk.P_s) ? kSlot1 : 0);
              if (seq_last) {
                // the owner of the sequence's last page tells the merge kernel
                // where the partials are (or that there is nothing to merge);
                // only the CTA's first sequence can have begun earlier
                reinterpret_cast<int4 *>(p.seq_merge)[wk.s] =
                    before ? make_int4(sh.first_cfirst, c - sh.first_cfirst + 1, sh.first_fslot, 0)
                           : make_int4(c, 1, 0, 0);
              }
            }
            d.flags = flags;
            descs[slot * kMaxPPS + k] = d;
          }
          if (!bad)
            bytes += PAIR     ? (pb2 >= 0 ? 2u : 1u) * (uint32_t)nbox * (uint32_t)p.box_bytes
                     : p.tile ? 2u * (uint32_t)nbox * (uint32_t)p.box_bytes
                              : 2u * (uint32_t)ntok * (uint32_t)p.row_bytes;
          if (first) bytes += (uint32_t)p.q_bytes;
          const int32_t s_before = wk.s;
          wk.advance(p, end, lane);
          if (pp > 0) {
            if (wk.s != s_before) {
              u_cur = 0;
              u_left = pp;
            } else if (--u_left == 0) {
              ++u_cur;
              u_left = pp;
            }
          }
        }
        __syncwarp();
        // the rows written above are read back by this stage's copies
        if (wrote) fence_proxy_async_global();
        if (lane == 0) mbar_arrive_expect_tx(&sh.full[slot], bytes);
        __syncwarp();
        unsigned char *st = stages + (size_t)slot * p.stage_bytes;
        unsigned char *kst = st;
        unsigned char *vst = st + (size_t)p.pps * p.vpage_stride;
        unsigned char *qst = st + (size_t)2 * p.pps * p.vpage_stride;
        for (int k = 0; k < npg; ++k) {
          const PageDesc d = descs[slot * kMaxPPS + k];
          if constexpr (PAIR) {
            if (!(d.flags & kBad)) {
              // one box of the block's token rows of every KV head per
              // (block, tensor, box of the row); the second block's box lands
              // after the first's
              constexpr int kHalves = kFp8 ? 1 : D / 64;
              const int nblk = d.pad0 >= 0 ? 2 : 1;
              if (lane < nblk * 2 * kHalves) {
                const int dh = lane % kHalves;
                const bool isv = (lane / kHalves) & 1;
                const int blk = lane / (2 * kHalves);
                tma_load_3d_hint((isv ? vst : kst) + (size_t)k * p.vpage_stride +
                                     (size_t)dh * p.box_bytes + (size_t)blk * (p.box_bytes / 2),
                                 isv ? &p.tmap_v : &p.tmap_k, dh * 64,
                                 (blk ? d.pad0 : d.pb) * p.block_size, 0, &sh.full[slot],
                                 kv_policy);
              }
            }
          } else if (!(d.flags & kBad) && p.tile) {
            // one box per (tensor, 64-wide d half), one lane each
            if (lane < 2 * nbox) {
              const int dh = lane % nbox;
              const bool isv = lane >= nbox;
              tma_load_3d_hint((isv ? vst : kst) + (size_t)k * p.vpage_stride +
                                   (size_t)dh * p.box_bytes,
                               isv ? &p.tmap_v : &p.tmap_k, dh * 64, d.pb * p.block_size + d.toff,
                               0, &sh.full[slot], kv_policy);
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
      int slot = -1, round = 0;  // stage slot and ring round, as the producer's
      for (int i = 0; i < n_stages; ++i) {
        if (++slot == p.stages) {
          slot = 0;
          ++round;
        }
        if (!__all_sync(0xffffffffu, mbar_wait(&sh.full[slot], round & 1, &sh.abort_flag))) {
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
        bool released = false;
        for (int k = 0; k < npg; ++k) {
          const PageDesc d = descs[slot * kMaxPPS + k];
          if (d.flags & kFirst) {
            cs.reset();
            const TA *qs = reinterpret_cast<const TA *>(qst + (size_t)k * p.q_bytes);
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
            if constexpr (kFp8) {
              cs.page_codes(kp, vp, d.ntok, p, h, lane);
            } else if constexpr (kMma) {
              cs.page(kp, vp, d.ntok, p, h, col_bytes, lane);
            } else {
              cs.page(kp, vp, d.ntok, p.row_pitch, col_bytes, sc_buf, lane);
            }
          }
          if (d.flags & kLast) {
            // The flush works on registers only: hand the stage back first
            // when this was its last page, so the producer is not held up.
            if (k == npg - 1 && !released) {
              __syncwarp();
              if (lane == 0) mbar_arrive(&sh.empty[slot]);
              released = true;
            }
            if constexpr (kMma) {
              cs.template flush<TA>(p, d, hq0, p.heads_per_warp, c, lane);
            } else {
              cs.flush(p, d, hq0, c, lane);
            }
            cs.reset();
          }
        }
        if (!released) {
          __syncwarp();
          if (lane == 0) mbar_arrive(&sh.empty[slot]);
        }
      }
    }
  }

  __syncthreads();

  // ---- Sequences with no visible page: zero output, or empty partials
  // (split-K: also every partition past a sequence's context); flag bad
  // lengths.
  for (int s = c; s < p.batch; s += p.grid) {
    const int32_t vis = cached ? sh.ctx_c[s] : visible_len(p, s);
    const bool has = vpages_of(vis, p) > 0;
    const int32_t ctx = vis + p.tok_offset;
    if (!has && tid == 0) {
      if (!splitk) reinterpret_cast<int4 *>(p.seq_merge)[s] = make_int4(0, 0, 0, 0);
      if (ctx < 0 || (int64_t)ctx > (int64_t)p.table_stride * p.block_size)
        set_error(p.err_word, PA_DEVERR_CONTEXT_LEN);
      // fused write: no visible position for the new token
      if (p.slot_mapping != nullptr && (cached ? sh.slot_c[s] : p.slot_mapping[s]) >= 0)
        set_error(p.err_word, PA_DEVERR_SLOT);
    }
    if (splitk) {
      const int32_t pt = (int32_t)pp << p.log2_vbs;  // tokens per partition
      const int32_t used = has ? (vis + pt - 1) / pt : 0;
      const int32_t left = p.max_parts - used;
      if (left <= 0) continue;
      const int64_t n4 = (int64_t)p.num_q_heads * left * (D / 4);
      for (int64_t x = tid; x < n4; x += blockDim.x) {
        const int32_t r = (int32_t)(x / (D / 4)), dq = (int32_t)(x % (D / 4));
        const int64_t ix = ((int64_t)s * p.num_q_heads + r / left) * p.max_parts + used + r % left;
        *reinterpret_cast<float4 *>(p.sk_o + ix * D + dq * 4) = make_float4(0.f, 0.f, 0.f, 0.f);
        if (dq == 0) {
          p.sk_max[ix] = -INFINITY;
          p.sk_sum[ix] = 0.f;
        }
      }
      continue;
    }
    if (has) continue;
    const int64_t n = (int64_t)p.num_q_heads * D;
    if (p.seq_o != nullptr) {
      // empty suffix: a partial that weighs nothing
      for (int64_t x = tid; x < n; x += blockDim.x) p.seq_o[(int64_t)s * n + x] = 0.f;
      for (int x = tid; x < p.num_q_heads; x += blockDim.x)
        reinterpret_cast<float2 *>(p.seq_ml)[(int64_t)s * p.num_q_heads + x] =
            make_float2(-INFINITY, 0.f);
    } else {
      for (int64_t x = tid; x < n; x += blockDim.x)
        Elem<TA>::store1(p.out, (int64_t)s * n + x, 0.f);
    }
  }
}

// ---------------------------------------------------------------------------
// Host side: launch one instantiation.  Explicitly instantiated per dtype in
// its own translation unit.
// ---------------------------------------------------------------------------
template <typename T, int D, int G, int NCW, bool PAIR = false>
cudaError_t launch_one(const Params &p, size_t smem, cudaStream_t stream) {
  auto kern = decode_stream_kernel<T, D, G, NCW, PAIR>;
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
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)p.grid);
  cfg.blockDim = dim3((NCW + 1) * 32);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, p);
}

// ---------------------------------------------------------------------------
// Merge kernel: one warp per (sequence, query-head slice of a consumer warp).
// Runs after the decode kernel (programmatic launch: it may be scheduled
// early and waits for the decode grid), when the memory system is quiet.
// ---------------------------------------------------------------------------
template <typename Tout, int D>
__global__ void __launch_bounds__(128) merge_kernel(const __grid_constant__ Params p) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  // a following kernel launched programmatically (the shared-prefix pass)
  // may start; it waits for this grid before reading what it writes
  asm volatile("griddepcontrol.launch_dependents;");
  const int slices = p.num_q_heads / p.heads_per_warp;
  const int seq = blockIdx.x / slices;
  const int hq0 = (blockIdx.x % slices) * p.heads_per_warp;
  const int4 md = __ldcg(reinterpret_cast<const int4 *>(p.seq_merge) + seq);
  const int n = md.y;
  if (n <= 1) return;  // empty, or written directly by its only CTA
  const int first_slot = md.z;
  const int64_t orow = (int64_t)seq * p.num_q_heads + hq0;
  // thread -> 4 consecutive outputs (head, d .. d+3) of this slice
  for (int f = threadIdx.x * 4; f < p.heads_per_warp * D; f += blockDim.x * 4) {
    const int h = f / D, d0 = f % D;
    float M = -INFINITY, W = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    bool bad = false;
    // contributors in batches of 8: all loads of a batch are in flight together
    for (int x0 = 0; x0 < n; x0 += 8) {
      float2 ml[8];
      float4 o4[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int x = x0 + j;
        if (x < n) {
          const int64_t r = ((int64_t)(md.x + x) * 2 + (x == 0 ? first_slot : 0)) *
                                p.num_q_heads + hq0 + h;
          ml[j] = __ldcg(reinterpret_cast<const float2 *>(p.part_ml) + r);
          o4[j] = __ldcg(reinterpret_cast<const float4 *>(p.part_o + r * D + d0));
        } else {
          ml[j] = make_float2(-INFINITY, 0.f);
          o4[j] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
      float mb = M;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        bad |= ml[j].y < 0.f;
        if (ml[j].y > 0.f) mb = fmaxf(mb, ml[j].x);
      }
      const float keep = (M == -INFINITY) ? 0.f : ex2(M - mb);
      W *= keep;
      acc.x *= keep;
      acc.y *= keep;
      acc.z *= keep;
      acc.w *= keep;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float w = (ml[j].y > 0.f) ? ml[j].y * ex2(ml[j].x - mb) : 0.f;
        W += w;
        acc.x += w * o4[j].x;
        acc.y += w * o4[j].y;
        acc.z += w * o4[j].z;
        acc.w += w * o4[j].w;
      }
      M = mb;
    }
    const float inv = 1.f / W;
    const int64_t e = (orow + h) * D + d0;
    if (p.seq_o != nullptr) {
      // suffix mode: the merged result as a partial for the prefix pass
      *reinterpret_cast<float4 *>(p.seq_o + e) =
          bad ? make_float4(0.f, 0.f, 0.f, 0.f)
              : make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
      if (d0 == 0)
        reinterpret_cast<float2 *>(p.seq_ml)[orow + h] = make_float2(M, bad ? -1.f : W);
      continue;
    }
    Elem<Tout>::store4(p.out, e,
                       bad ? make_float4(0.f, 0.f, 0.f, 0.f)
                           : make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv));
  }
}

template <typename Tout, int D>
cudaError_t launch_merge_one(const Params &p, cudaStream_t stream) {
  const int64_t blocks = (int64_t)p.batch * (p.num_q_heads / p.heads_per_warp);
  if (blocks == 0) return cudaSuccess;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)blocks);
  cfg.blockDim = dim3(128);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, merge_kernel<Tout, D>, p);
}

}  // namespace stream
}  // namespace pa
