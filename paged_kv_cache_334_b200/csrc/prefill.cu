// prefill.cu -- paged (chunked) prefill attention with the causal mask, on
// the 5th-generation tensor cores (tcgen05), for pa_prefill.
//
// [teaching] page "Implementing teaching PagedAttention: reading the
// historical KV cache from the block table", section "Where is the attention
// mask": in prefill a prompt token sees itself and the tokens before it,
// nothing later.  [route] page "From correct to faster: the PagedAttention
// optimisation route", section "decode attention and prefill attention are
// different": prefill handles a whole prompt, or a chunk of one, at once, so
// many query tokens read the same pages and the work is a dense contraction.
// Sequence b brings n_b new tokens (rows query_start[b] .. query_start[b+1]-1
// of q) whose K/V already sit in the cache at their slots; its history holds
// context_lens[b] tokens including them, so new token j has position
// p_j = context_lens[b] - n_b + j and attends to positions 0 .. p_j, read
// through row b of the block table.
//
// One CTA per (tile of 128 rows, KV head, sequence).  A tile's rows are
// 128 / G query tokens x the G query heads of the KV head (row = token * G +
// head), so one K/V read serves the whole GQA group.  It walks the sequence's
// 128-token K/V tiles up to its last row's position, as a FlashAttention
// forward pass (online softmax, no score matrix in memory); tiles past a
// row's position are masked per row, and the last tile's products stop at
// the 16-token step that holds the tile's last position.  The later tiles of a sequence do the
// most work and are launched first.
//
//   warp 0     tiled copies (no multicast): the Q tile once, then K and V of
//              each 128-token tile page by page into separate rings (3 K
//              stages, 2 V stages);
//   warp 1     issues tcgen05.mma: S_b = Q K^T (M 128, N 128, K = D), then
//              O += P_{b'} V for the previous tile (A = P in tensor memory);
//   warps 2-9  softmax, two warps per tensor-memory subpartition: warp w
//              owns row 32 (w % 4) + lane and half of each tile's columns
//              (and of O's); the pair exchanges row maxima and, at the end,
//              the normaliser through shared memory; then the epilogue.
// Tensor memory (512 columns): O [0, D), S_b [D + 128 b, +128), P_b (bf16
// pairs) [D + 256 + 64 b, +64).  The running maximum is raised only when a
// score exceeds it by more than 8 (log2 units), so P < 2^8 and O is rescaled
// rarely; O and the normaliser share the maximum, so the result is exact.
// Every wait is bounded (PA_DEVERR_TIMEOUT on expiry).
//
// The whole sequence's table slice (ceil(context_len / block_size) entries)
// is read into shared memory and checked before the first copy, so that a
// bad block id anywhere in the sequence zeroes all its rows, in every CTA.
#include <cuda_bf16.h>
#include <math.h>

#include "pa_common.cuh"
#include "pa_launch.h"
#include "sm100_ptx.cuh"

namespace pa {
namespace prefill {

using namespace pa::stream;

constexpr int kRows = 128;       // M: (query token, query head) rows of one tile
constexpr int kTok = 128;        // N of S: KV tokens per tile
constexpr int kThreads = 320;    // 10 warps
constexpr uint32_t kTmemCols = 512;
constexpr float kSlack = 8.f;    // lazy rescaling threshold (log2 units)
constexpr int kBox = kRows * 128;  // bytes of one 64-element-wide half of a 128-row tile
constexpr int kKStages = 3, kVStages = 2;

struct alignas(16) Shared {
  uint64_t qfull, kfull[kKStages], kempty[kKStages], vfull[kVStages], vempty[kVStages];
  uint64_t sfull[2], sfree[2], pfull[2], pfree[2], mma_done;
  uint64_t xbar[4][2], xend[4];  // softmax pair handshakes (per subpartition)
  uint32_t tmem_base;
  int32_t abort_flag, bad, pad;
  float xm[2][2][kRows];  // [tile parity][column half][row] partial row maxima
  float xl[2][kRows];     // [column half][row] partial normalisers
  int32_t ids[kMaxPrefillBlocks];  // the sequence's physical blocks
};
// header, alignment slack, Q tile and the K / V rings at head_dim 128
static_assert(sizeof(Shared) + 1024 + 2 * kBox * (1 + kKStages + kVStages) <= kSmemLimit,
              "prefill tiles exceed the shared memory of one CTA");

// Warp-uniform bounded wait: one inline test, the rest out of line.
static __device__ __noinline__ bool wait_all_slow(uint64_t *bar, uint32_t parity, Shared &sh,
                                                  int32_t *err_word, int lane) {
  const bool ok = __all_sync(0xffffffffu, mbar_wait_slow(bar, parity, &sh.abort_flag));
  if (!ok && lane == 0) {
    sh.abort_flag = 1;
    set_error(err_word, PA_DEVERR_TIMEOUT);
  }
  return ok;
}
__device__ __forceinline__ bool wait_all(uint64_t *bar, uint32_t parity, Shared &sh,
                                         const PrefillParams &p, int lane) {
  if (__all_sync(0xffffffffu, mbar_try_wait(bar, parity))) return true;
  return wait_all_slow(bar, parity, sh, p.err_word, lane);
}

template <int D>
struct Cols {
  static constexpr uint32_t O = 0, S = D, P = D + 2 * kTok;
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_attention_kernel(const __grid_constant__ PrefillParams p) {
  constexpr int NH = D / 64;  // 64-element halves of head_dim
  extern __shared__ __align__(128) unsigned char smem_raw[];
  Shared &sh = *reinterpret_cast<Shared *>(smem_raw);
  unsigned char *tiles =
      smem_raw + (((smem_u32(smem_raw) + sizeof(Shared) + 1023u) & ~1023u) - smem_u32(smem_raw));
  unsigned char *qt = tiles;                            // NH x [128 rows][128 B]
  unsigned char *kring = tiles + NH * kBox;             // K stage s: NH x kBox
  unsigned char *vring = kring + kKStages * NH * kBox;  // V stage s: NH x kBox
  auto k_stage = [&](int s) { return kring + (size_t)s * NH * kBox; };
  auto v_stage = [&](int s) { return vring + (size_t)s * NH * kBox; };

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tile = p.tiles_per_seq - 1 - (int)blockIdx.x;  // late (long) tiles first
  const int h = blockIdx.y;                                // KV head
  const int b = blockIdx.z;                                // sequence
  const int tpt = kRows / p.group;                         // query tokens per tile
  const int j0 = tile * tpt;                               // first new token of the tile

  // The sequence's rows and length; every thread reads the same words and
  // takes the same decisions.
  const int32_t q0 = p.query_start[b], q1 = p.query_start[b + 1];
  const int32_t ctx = p.context_lens[b];
  const bool range_ok = q0 >= 0 && q1 >= q0 && q1 <= p.num_tokens;
  if (!range_ok) {
    // rows that cannot be located: nothing is written
    if (tid == 0 && h == 0 && blockIdx.x == 0) set_error(p.err_word, PA_DEVERR_CONTEXT_LEN);
    return;
  }
  const int n = q1 - q0;
  // a chunk longer than the grid covers, more new tokens than the history
  // holds, or a history longer than the table: the rows are zeroed
  const bool len_bad = (int64_t)n > (int64_t)p.tiles_per_seq * tpt || n > ctx ||
                       (int64_t)ctx > (int64_t)p.table_stride * p.block_size;
  if (len_bad && tid == 0 && h == 0 && blockIdx.x == 0) set_error(p.err_word, PA_DEVERR_CONTEXT_LEN);
  if (j0 >= n) return;  // the grid covers the longest chunk; this tile is empty
  const int j_end = min(j0 + tpt, n);  // one past the tile's last new token
  const int pos_max = ctx - n + j_end - 1;  // position of the tile's last row

  if (tid == 0) {
    prefetch_tensormap(&p.tmap_q);
    prefetch_tensormap(&p.tmap_k);
    prefetch_tensormap(&p.tmap_v);
    mbar_init(&sh.qfull, 1);
    for (int i = 0; i < kKStages; ++i) {
      mbar_init(&sh.kfull[i], 1);
      mbar_init(&sh.kempty[i], 1);
    }
    for (int i = 0; i < kVStages; ++i) {
      mbar_init(&sh.vfull[i], 1);
      mbar_init(&sh.vempty[i], 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&sh.sfull[x], 1);
      mbar_init(&sh.sfree[x], 8);
      mbar_init(&sh.pfull[x], 8);
      mbar_init(&sh.pfree[x], 1);
    }
    mbar_init(&sh.mma_done, 1);
    for (int q = 0; q < 4; ++q) {
      mbar_init(&sh.xbar[q][0], 64);
      mbar_init(&sh.xbar[q][1], 64);
      mbar_init(&sh.xend[q], 64);
    }
    sh.abort_flag = 0;
    sh.bad = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    if (!len_bad) {
      // the Q tile does not depend on the table: its copy overlaps the
      // table check below
      mbar_arrive_expect_tx(&sh.qfull, (uint32_t)(NH * kBox));
      for (int dh = 0; dh < NH; ++dh)
        tma_load_3d(qt + dh * kBox, &p.tmap_q, dh * 64, h * p.group, q0 + j0, &sh.qfull);
    }
  }
  // tensor memory is allocated while the table is read
  if (warp == 1 && !len_bad) {
    tc_alloc(&sh.tmem_base, kTmemCols);
    tc_relinquish();
  }
  __syncthreads();
  if (len_bad) {
    if (tid == 0) sh.bad = 1;
  } else {
    // the sequence's whole table slice, checked
    const int n_ids = (ctx + p.block_size - 1) / p.block_size;
    const int32_t *trow = p.block_tables + (int64_t)b * p.table_stride;
    for (int i = tid; i < n_ids; i += kThreads) {
      int32_t pb = trow[i];
      if (pb < 0 || pb >= p.num_blocks) {
        sh.bad = 1;
        if (h == 0) set_error(p.err_word, PA_DEVERR_BLOCK_ID);
        pb = 0;
      }
      sh.ids[i] = pb;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (sh.bad) {
    if (!len_bad) {
      // the Q copy lands before the CTA's shared memory is released, and
      // the tensor memory goes back
      if (tid == 0) {
        volatile int32_t never = 0;
        if (!mbar_wait(&sh.qfull, 0, &never)) set_error(p.err_word, PA_DEVERR_TIMEOUT);
      }
      if (warp == 1) tc_dealloc(sh.tmem_base, kTmemCols);
    }
    // zero the tile's rows: tokens [j0, j_end) x the group's heads
    const int64_t row_elems = (int64_t)p.group * D;  // one token's heads of this KV head
    const int64_t per_tok = (int64_t)p.num_q_heads * D;
    const int64_t units = (int64_t)(j_end - j0) * row_elems / 8;  // 8 bf16 per store
    for (int64_t u = tid; u < units; u += kThreads) {
      const int64_t e = u * 8, tok = e / row_elems, w = e - tok * row_elems;
      const int64_t at = ((int64_t)q0 + j0 + tok) * per_tok + (int64_t)h * p.group * D + w;
      *reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(p.out) + at) =
          make_uint4(0u, 0u, 0u, 0u);
    }
    return;
  }

  const uint32_t tm = sh.tmem_base;

  const int ppt = kTok / p.block_size;        // pages per K/V tile
  const int n_tiles = pos_max / kTok + 1;     // K/V tiles the tile's rows reach
  const int last_page = pos_max / p.block_size;
  // tokens of K/V tile t at positions <= pos_max (all 128 but in the last)
  auto tile_tokens = [&](int t) { return min(kTok, pos_max + 1 - t * kTok); };

  if (warp == 0) {
    // ===================== tiled copies (Q was issued above) =====================
    const uint32_t page_bytes = (uint32_t)p.block_size * 128u;
    // one K or V tile: its pages' boxes back to back per d half
    auto load = [&](const CUtensorMap *map, unsigned char *dst, uint64_t *bar, int t) {
      const int npg = min(ppt, last_page + 1 - t * ppt);
      if (lane == 0) {
        mbar_arrive_expect_tx(bar, (uint32_t)NH * (uint32_t)npg * page_bytes);
        for (int i = 0; i < npg; ++i) {
          const int pb = sh.ids[t * ppt + i];
          for (int dh = 0; dh < NH; ++dh)
            tma_load_3d(dst + dh * kBox + i * page_bytes, map, dh * 64, pb * p.block_size, h, bar);
        }
      }
      __syncwarp();
    };
    // K runs one tile ahead of V: V(t) is needed only after the softmax of t
    for (int t = 0; t <= n_tiles; ++t) {
      if (t < n_tiles) {
        const int ks = t % kKStages;
        if (t >= kKStages &&
            !wait_all(&sh.kempty[ks], ((t / kKStages) - 1) & 1, sh, p, lane))
          break;
        load(&p.tmap_k, k_stage(ks), &sh.kfull[ks], t);
      }
      if (t >= 1) {
        const int u = t - 1, vs = u % kVStages;
        if (u >= kVStages &&
            !wait_all(&sh.vempty[vs], ((u / kVStages) - 1) & 1, sh, p, lane))
          break;
        load(&p.tmap_v, v_stage(vs), &sh.vfull[vs], u);
      }
    }
  } else if (warp == 1) {
    // ===================== tensor-core issue =====================
    const uint32_t id_s = idesc_bf16(kRows, kTok, false);
    const uint32_t id_o = idesc_bf16(kRows, D, true);
    bool ok = wait_all(&sh.qfull, 0, sh, p, lane);
    auto issue_pv = [&](int u) -> bool {
      const int x = u & 1, vst = u % kVStages;
      if (!wait_all(&sh.vfull[vst], (u / kVStages) & 1, sh, p, lane)) return false;
      if (!wait_all(&sh.pfull[x], (u >> 1) & 1, sh, p, lane)) return false;
      const int ntok = tile_tokens(u);
      // K steps of 16 tokens that hold a position <= pos_max; the later ones
      // (all masked) are skipped
      const int nks = (ntok + 15) >> 4;
      if (ntok < 16 * nks) {
        // V rows past the last position inside the last K step: later slots
        // of the last page (which may hold anything) or stage memory no page
        // was copied to; their probabilities are 0, but 0 x NaN is not
        unsigned char *vs = v_stage(vst);
        const int units = (16 * nks - ntok) * 8;
        for (int i = lane; i < units * NH; i += 32) {
          const int dh = i / units, rem = i - dh * units;
          *reinterpret_cast<uint4 *>(vs + dh * kBox + (ntok + (rem >> 3)) * 128 + (rem & 7) * 16) =
              make_uint4(0u, 0u, 0u, 0u);
        }
        fence_proxy_async_smem();
      }
      __syncwarp();
      tc_fence_after();
      if (lane == 0) {
        const uint32_t va = smem_u32(v_stage(vst));
        for (int ks = 0; ks < nks; ++ks)
          tc_mma_ts(tm + Cols<D>::O, tm + Cols<D>::P + 64 * x + 8 * ks,
                    sw128_desc(va + 2048 * ks, (uint32_t)kBox, 1024), id_o,
                    (u == 0 && ks == 0) ? 0u : 1u);
        tc_commit(&sh.pfree[x]);
        tc_commit(&sh.vempty[vst]);
      }
      __syncwarp();
      return true;
    };
    for (int t = 0; t < n_tiles && ok; ++t) {
      const int x = t & 1, kst = t % kKStages;
      if (!wait_all(&sh.kfull[kst], (t / kKStages) & 1, sh, p, lane)) {
        ok = false;
        break;
      }
      if (t >= 2 && !wait_all(&sh.sfree[x], ((t >> 1) - 1) & 1, sh, p, lane)) {
        ok = false;
        break;
      }
      tc_fence_after();
      if (lane == 0) {
        const uint32_t qa = smem_u32(qt), ka = smem_u32(k_stage(kst));
        // the last tile: only its first columns (16 at a time) hold positions
        // <= pos_max; the rest of S is left as it was and masked by the softmax
        const int ntok = tile_tokens(t);
        const uint32_t id_t =
            ntok < kTok ? idesc_bf16(kRows, (ntok + 15) & ~15, false) : id_s;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (uint32_t)(kk >> 2) * kBox + (uint32_t)(kk & 3) * 32;
          tc_mma_ss(tm + Cols<D>::S + kTok * x, sw128_desc(qa + off, 16, 1024),
                    sw128_desc(ka + off, 16, 1024), id_t, kk > 0 ? 1u : 0u);
        }
        tc_commit(&sh.sfull[x]);
        tc_commit(&sh.kempty[kst]);  // K stage free once S is computed
      }
      __syncwarp();
      if (t >= 1 && !issue_pv(t - 1)) ok = false;
    }
    if (ok) issue_pv(n_tiles - 1);
  } else {
    // ===================== softmax and epilogue =====================
    const int sp = warp & 3;               // tensor-memory subpartition
    const int half = (warp - 2) >> 2;      // which 64 of a tile's 128 columns
    const uint32_t lane_base = (uint32_t)(32 * sp) << 16;
    const int r = 32 * sp + lane;          // this thread's row
    const int j = j0 + r / p.group;        // its new token
    const bool valid = j < n;
    // its position (rows past the chunk borrow the last row's: never written)
    const int pos = ctx - n + min(j, n - 1);
    constexpr int HC = kTok / 2;           // score columns per thread
    constexpr int HD = D / 2;              // output columns per thread
    auto pair_sync = [&](uint64_t *bar, uint32_t parity) -> bool {
      mbar_arrive(bar);
      return wait_all(bar, parity, sh, p, lane);
    };
    const float sl = p.scale_log2;
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    for (int t = 0; t < n_tiles && ok; ++t) {
      const int x = t & 1;
      // columns c < limit of this tile are at positions <= pos
      const int limit = pos + 1 - t * kTok;
      if (!wait_all(&sh.sfull[x], (t >> 1) & 1, sh, p, lane)) {
        ok = false;
        break;
      }
      tc_fence_after();
      float sc[HC];
#pragma unroll
      for (int c = 0; c < HC / 16; ++c) {
        uint32_t raw[16];
        tc_ld16(tm + lane_base + Cols<D>::S + kTok * x + HC * half + 16 * c, raw);
#pragma unroll
        for (int i = 0; i < 16; ++i) sc[16 * c + i] = __uint_as_float(raw[i]);
      }
      tc_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh.sfree[x]);
      // unmasked tiles keep raw scores (with scale > 0 the maximum of the
      // scaled scores is the scaled maximum); masked ones are scaled here and
      // the columns past the row's position become -inf, whatever K held
      const bool scaled = limit < kTok || sl < 0.f;
      if (scaled) {
#pragma unroll
        for (int i = 0; i < HC; ++i) sc[i] = (HC * half + i < limit) ? sc[i] * sl : -INFINITY;
      }
      float mx = -INFINITY;
#pragma unroll
      for (int i = 0; i < HC; ++i) mx = fmaxf(mx, sc[i]);
      sh.xm[x][half][r] = scaled ? mx : mx * sl;
      if (!pair_sync(&sh.xbar[sp][x], (t >> 1) & 1)) {
        ok = false;
        break;
      }
      // position 0 is in every row's first tile, so m_new is finite from then on
      const float m_new = fmaxf(m_used, fmaxf(sh.xm[x][0][r], sh.xm[x][1][r]));
      const bool need = m_new > m_used + kSlack;
      if (__any_sync(0xffffffffu, need)) {
        const float f = need ? ex2(m_used - m_new) : 1.f;
        if (t >= 1) {
          // O holds the earlier tiles: wait for the last product, rescale
          // this warp's half of the columns
          if (!wait_all(&sh.pfree[(t - 1) & 1], ((t - 1) >> 1) & 1, sh, p, lane)) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll 1
          for (int c = 0; c < HD / 16; ++c) {
            uint32_t o16[16];
            tc_ld16(tm + lane_base + Cols<D>::O + HD * half + 16 * c, o16);
            tc_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; ++i) o16[i] = __float_as_uint(__uint_as_float(o16[i]) * f);
            tc_st16(tm + lane_base + Cols<D>::O + HD * half + 16 * c, o16);
          }
          tc_wait_st();
        }
        if (need) {
          l *= f;
          m_used = m_new;
        }
      }
      uint32_t pk[HC / 2];
      float add = 0.f;
      const float mul = scaled ? 1.f : sl;
#pragma unroll
      for (int i = 0; i < HC / 2; ++i) {
        const float p0 = ex2(fmaf(sc[2 * i], mul, -m_used));
        const float p1 = ex2(fmaf(sc[2 * i + 1], mul, -m_used));
        add += p0 + p1;
        pk[i] = pack_bf16x2(p0, p1);
      }
      l += add;
      if (t >= 2 && !wait_all(&sh.pfree[x], ((t >> 1) - 1) & 1, sh, p, lane)) {
        ok = false;
        break;
      }
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < HC / 32; ++c) {
        uint32_t w16[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) w16[i] = pk[16 * c + i];
        tc_st16(tm + lane_base + Cols<D>::P + (kTok / 2) * x + (HC / 2) * half + 16 * c, w16);
      }
      tc_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh.pfull[x]);
    }
    if (ok && wait_all(&sh.pfree[(n_tiles - 1) & 1], ((n_tiles - 1) >> 1) & 1, sh, p, lane)) {
      // the pair's normalisers add up to the row's
      sh.xl[half][r] = l;
      if (pair_sync(&sh.xend[sp], 0)) {
        const float inv = 1.f / (sh.xl[0][r] + sh.xl[1][r]);
        tc_fence_after();
        const int64_t orow =
            ((int64_t)q0 + j) * p.num_q_heads + (int64_t)h * p.group + r % p.group;
#pragma unroll 1
        for (int c = 0; c < HD / 16; ++c) {
          const int col = HD * half + 16 * c;
          uint32_t o16[16];
          tc_ld16(tm + lane_base + Cols<D>::O + col, o16);
          tc_wait_ld();
          if (valid) {
            const int64_t e = orow * D + col;
#pragma unroll
            for (int i = 0; i < 16; i += 4)
              Elem<__nv_bfloat16>::store4(
                  p.out, e + i,
                  make_float4(__uint_as_float(o16[i]) * inv, __uint_as_float(o16[i + 1]) * inv,
                              __uint_as_float(o16[i + 2]) * inv,
                              __uint_as_float(o16[i + 3]) * inv));
          }
        }
      }
    }
  }

  // every tensor-core operation has finished before the memory is released
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    if (lane == 0) tc_commit(&sh.mma_done);
    __syncwarp();
    volatile int32_t never = 0;
    if (!__all_sync(0xffffffffu, mbar_wait(&sh.mma_done, 0, &never)) && lane == 0)
      set_error(p.err_word, PA_DEVERR_TIMEOUT);
    tc_dealloc(tm, kTmemCols);
  }
}

template <int D>
cudaError_t launch_d(const PrefillParams &p, cudaStream_t stream) {
  auto kern = prefill_attention_kernel<D>;
  const size_t smem = prefill_smem_bytes(D);
  static size_t configured[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (smem > configured[dev]) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    configured[dev] = smem;
  }
  const dim3 grid((unsigned)p.tiles_per_seq, (unsigned)p.num_kv_heads, (unsigned)p.batch);
  kern<<<grid, kThreads, smem, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace prefill

size_t prefill_smem_bytes(int head_dim) {
  const size_t nh = (size_t)head_dim / 64;
  // header (with the table slice), 1 KB alignment slack, the Q tile, the K
  // and V rings; at least 120 KB, so that no other CTA holding tensor memory
  // shares the SM
  const size_t need = sizeof(prefill::Shared) + 1024 +
                      nh * prefill::kBox * (1 + prefill::kKStages + prefill::kVStages);
  return need < 120 * 1024 ? 120 * 1024 : need;
}

cudaError_t launch_prefill(const PrefillParams &p, int head_dim, cudaStream_t stream) {
  if (head_dim == 64) return prefill::launch_d<64>(p, stream);
  if (head_dim == 128) return prefill::launch_d<128>(p, stream);
  return cudaErrorInvalidValue;
}

}  // namespace pa
