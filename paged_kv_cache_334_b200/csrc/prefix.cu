// prefix.cu -- attention over a KV prefix shared by every sequence of the
// batch, on the 5th-generation tensor cores (tcgen05), for
// pa_decode_shared_prefix.
//
// Page "Operators and compilers: inference attention and KV kernels", section
// 6 (prefix caching: requests that share a prompt prefix share its KV pages)
// and section 4.1: once many queries read the same pages, the work is a
// dense contraction, not a stream.  Every (sequence, query head) row of a KV
// head attends to the same prefix tokens, so 128 such rows form the M side of
// S = Q K^T and O += P V, tile after tile of 128 prefix tokens, as in a
// FlashAttention forward pass ([route] page "From correct to faster: the
// PagedAttention optimisation route", section "The core idea of
// high-performance PagedAttention": online softmax, no score matrix in
// memory).  The suffix past the prefix is decoded first: for groups of 64 or
// 128 query heads by the tensor-core suffix kernel (suffix.cu), which leaves
// one (max, sum, normalised output) per row or, for a (sequence, KV head)
// pair cut between its CTAs, one such partial per CTA with a record of where
// they are; for other groups by the persistent page-stream kernel in suffix
// mode and its merge kernel, one partial per row.  This kernel's epilogue
// folds the parts in with the running-max rescaling and writes the output.
//
// One CTA per (tile of 128 rows, KV head), 6 warps:
//   warp 0     tiled copies (no multicast): the Q tile once, then K and V of
//              each 128-token prefix tile into separate rings (3 K stages, 2
//              V stages), so that a K stage comes back as soon as its S
//              product is done;
//   warp 1     issues tcgen05.mma: S_b = Q K^T (M 128, N 128, K = D), then
//              O += P_{b'} V for the previous tile (A = P in tensor memory);
//   warps 2-9  softmax, two warps per tensor-memory subpartition: warp w
//              owns row 32 (w % 4) + lane and half of each tile's 128
//              columns (and of O's); the pair exchanges row maxima (and at
//              the end the normaliser) through shared memory with a bounded
//              mbarrier handshake; then the epilogue.
// Tensor memory (512 columns): O [0, D), S_b [D + 128 b, +128), P_b (bf16
// pairs) [D + 256 + 64 b, +64).  The running max is raised only when a score
// exceeds it by more than 8 (log2 units), so P < 2^8 and O is rescaled
// rarely; O and the normaliser share the maximum, so the result is exact.
// Every wait is bounded (PA_DEVERR_TIMEOUT on expiry).
#include <cuda_bf16.h>
#include <math.h>

#include "pa_common.cuh"
#include "pa_launch.h"
#include "sm100_ptx.cuh"

namespace pa {
namespace prefix {

using namespace pa::stream;

constexpr int kRows = 128;       // M: (sequence, query head) rows of one tile
constexpr int kTok = 128;        // N of S: prefix tokens per tile
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
  int32_t abort_flag, bad_prefix, pad;
  float xm[2][2][kRows];  // [tile parity][column half][row] partial row maxima
  float xl[2][kRows];     // [column half][row] partial normalisers
  int32_t ids[kMaxPrefixBlocks];  // the shared prefix's physical blocks
};

// Warp-uniform bounded wait: one inline test, the rest out of line (see
// mbar_wait_slow).
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
                                         const PrefixParams &p, int lane) {
  if (__all_sync(0xffffffffu, mbar_try_wait(bar, parity))) return true;
  return wait_all_slow(bar, parity, sh, p.err_word, lane);
}

template <int D>
struct Cols {
  static constexpr uint32_t O = 0, S = D, P = D + 2 * kTok;
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    prefix_attention_kernel(const __grid_constant__ PrefixParams p) {
  constexpr int NH = D / 64;  // 64-element halves of head_dim
  extern __shared__ __align__(128) unsigned char smem_raw[];
  Shared &sh = *reinterpret_cast<Shared *>(smem_raw);
  unsigned char *tiles =
      smem_raw + (((smem_u32(smem_raw) + sizeof(Shared) + 1023u) & ~1023u) - smem_u32(smem_raw));
  unsigned char *qt = tiles;                          // NH x [128 rows][128 B]
  unsigned char *kring = tiles + NH * kBox;           // K stage s: NH x kBox
  unsigned char *vring = kring + kKStages * NH * kBox;  // V stage s: NH x kBox
  auto k_stage = [&](int s) { return kring + (size_t)s * NH * kBox; };
  auto v_stage = [&](int s) { return vring + (size_t)s * NH * kBox; };

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = blockIdx.y;                  // KV head
  const int row0 = blockIdx.x * kRows;       // first (sequence, group head) row
  const int s0 = row0 / p.group;             // its sequence
  const int ppt = kTok / p.block_size;       // pages per prefix tile
  const int n_tiles = (p.prefix_blocks + ppt - 1) / ppt;

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
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sh.sfull[b], 1);
      mbar_init(&sh.sfree[b], 8);
      mbar_init(&sh.pfull[b], 8);
      mbar_init(&sh.pfree[b], 1);
    }
    mbar_init(&sh.mma_done, 1);
    for (int q = 0; q < 4; ++q) {
      mbar_init(&sh.xbar[q][0], 64);
      mbar_init(&sh.xbar[q][1], 64);
      mbar_init(&sh.xend[q], 64);
    }
    sh.abort_flag = 0;
    sh.bad_prefix = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  // the shared prefix: the first prefix_blocks entries of sequence 0's table
  for (int i = tid; i < p.prefix_blocks; i += kThreads) {
    int32_t pb = p.block_tables[i];
    if (pb < 0 || pb >= p.num_blocks) {
      sh.bad_prefix = 1;
      set_error(p.err_word, PA_DEVERR_BLOCK_ID);
      pb = 0;  // any valid page: the outputs are zeroed
    }
    sh.ids[i] = pb;
  }
  if (warp == 1) {
    tc_alloc(&sh.tmem_base, kTmemCols);
    tc_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = sh.tmem_base;

  if (warp == 0) {
    // ===================== tiled copies =====================
    if (lane == 0) {
      mbar_arrive_expect_tx(&sh.qfull, (uint32_t)(NH * kBox));
      for (int dh = 0; dh < NH; ++dh)
        tma_load_3d(qt + dh * kBox, &p.tmap_q, dh * 64, h * p.group, s0, &sh.qfull);
    }
    const uint32_t page_bytes = (uint32_t)p.block_size * 128u;
    // one tile of K or V: its pages' boxes land back to back per d half
    auto load = [&](const CUtensorMap *map, unsigned char *dst, uint64_t *bar, int t) {
      const int npg = min(ppt, p.prefix_blocks - t * ppt);
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
      const int b = u & 1, vst = u % kVStages;
      if (!wait_all(&sh.vfull[vst], (u / kVStages) & 1, sh, p, lane)) return false;
      if (!wait_all(&sh.pfull[b], (u >> 1) & 1, sh, p, lane)) return false;
      const int ntok = min(ppt, p.prefix_blocks - u * ppt) * p.block_size;
      if (ntok < kTok) {
        // rows past the prefix in the last tile may hold anything
        unsigned char *vs = v_stage(vst);
        const int units = (kTok - ntok) * 8;
        for (int x = lane; x < units * NH; x += 32) {
          const int dh = x / units, rem = x - dh * units;
          *reinterpret_cast<uint4 *>(vs + dh * kBox + (ntok + (rem >> 3)) * 128 + (rem & 7) * 16) =
              make_uint4(0u, 0u, 0u, 0u);
        }
        fence_proxy_async_smem();
      }
      __syncwarp();
      tc_fence_after();
      if (lane == 0) {
        const uint32_t va = smem_u32(v_stage(vst));
        for (int ks = 0; ks < kTok / 16; ++ks)
          tc_mma_ts(tm + Cols<D>::O, tm + Cols<D>::P + 64 * b + 8 * ks,
                    sw128_desc(va + 2048 * ks, (uint32_t)kBox, 1024), id_o,
                    (u == 0 && ks == 0) ? 0u : 1u);
        tc_commit(&sh.pfree[b]);
        tc_commit(&sh.vempty[vst]);
      }
      __syncwarp();
      return true;
    };
    for (int t = 0; t < n_tiles && ok; ++t) {
      const int b = t & 1, kst = t % kKStages;
      if (!wait_all(&sh.kfull[kst], (t / kKStages) & 1, sh, p, lane)) {
        ok = false;
        break;
      }
      if (t >= 2 && !wait_all(&sh.sfree[b], ((t >> 1) - 1) & 1, sh, p, lane)) {
        ok = false;
        break;
      }
      tc_fence_after();
      if (lane == 0) {
        const uint32_t qa = smem_u32(qt), ka = smem_u32(k_stage(kst));
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (uint32_t)(kk >> 2) * kBox + (uint32_t)(kk & 3) * 32;
          tc_mma_ss(tm + Cols<D>::S + kTok * b, sw128_desc(qa + off, 16, 1024),
                    sw128_desc(ka + off, 16, 1024), id_s, kk > 0 ? 1u : 0u);
        }
        tc_commit(&sh.sfull[b]);
        tc_commit(&sh.kempty[kst]);  // K stage free once S is computed
      }
      __syncwarp();
      if (t >= 1 && !issue_pv(t - 1)) ok = false;
    }
    if (ok && n_tiles > 0) issue_pv(n_tiles - 1);
  } else {
    // ===================== softmax and epilogue =====================
    const int sp = warp & 3;               // tensor-memory subpartition
    const int half = (warp - 2) >> 2;      // which 64 of a tile's 128 columns
    const uint32_t lane_base = (uint32_t)(32 * sp) << 16;
    const int r = 32 * sp + lane;          // this thread's row
    const int grow = row0 + r;
    const int seq = grow / p.group;
    const int hq = h * p.group + grow % p.group;
    const bool valid = seq < p.batch;
    constexpr int HC = kTok / 2;           // score columns per thread
    constexpr int HD = D / 2;              // output columns per thread
    // The sequence must contain the declared prefix.  Checked before the
    // tiles (independent loads, in flight together) so that the latency
    // hides behind the first copies and products.
    bool mismatch = false;
    if (valid) {
      mismatch = p.context_lens[seq] < p.prefix_blocks * p.block_size;
      const int32_t *trow = p.block_tables + (int64_t)seq * p.table_stride;
      for (int i0 = 0; i0 < p.prefix_blocks; i0 += 16) {
        int32_t e[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) e[j] = (i0 + j < p.prefix_blocks) ? trow[i0 + j] : 0;
#pragma unroll
        for (int j = 0; j < 16; ++j)
          mismatch |= (i0 + j < p.prefix_blocks) && e[j] != sh.ids[i0 + j];
      }
    }
    // partner handshake: both warps of the pair arrive, then wait (bounded)
    auto pair_sync = [&](uint64_t *bar, uint32_t parity) -> bool {
      mbar_arrive(bar);
      return wait_all(bar, parity, sh, p, lane);
    };
    const float sl = p.scale_log2;
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    for (int t = 0; t < n_tiles && ok; ++t) {
      const int b = t & 1;
      const int ntok = min(ppt, p.prefix_blocks - t * ppt) * p.block_size;
      if (!wait_all(&sh.sfull[b], (t >> 1) & 1, sh, p, lane)) {
        ok = false;
        break;
      }
      tc_fence_after();
      float sc[HC];
#pragma unroll
      for (int c = 0; c < HC / 16; ++c) {
        uint32_t raw[16];
        tc_ld16(tm + lane_base + Cols<D>::S + kTok * b + HC * half + 16 * c, raw);
#pragma unroll
        for (int j = 0; j < 16; ++j) sc[16 * c + j] = __uint_as_float(raw[j]);
      }
      tc_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh.sfree[b]);
      // scores stay raw where possible: with scale > 0 the maximum of the
      // scaled scores is the scaled maximum and 2^(s scale - m) is one fused
      // multiply-add and one ex2 per score
      const bool scaled = ntok < kTok || sl < 0.f;
      if (scaled) {
#pragma unroll
        for (int j = 0; j < HC; ++j) sc[j] = (HC * half + j < ntok) ? sc[j] * sl : -INFINITY;
      }
      float mx = -INFINITY;
#pragma unroll
      for (int j = 0; j < HC; ++j) mx = fmaxf(mx, sc[j]);
      sh.xm[b][half][r] = scaled ? mx : mx * sl;
      if (!pair_sync(&sh.xbar[sp][b], (t >> 1) & 1)) {
        ok = false;
        break;
      }
      const float m_new = fmaxf(m_used, fmaxf(sh.xm[b][0][r], sh.xm[b][1][r]));
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
            for (int j = 0; j < 16; ++j) o16[j] = __float_as_uint(__uint_as_float(o16[j]) * f);
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
      for (int j = 0; j < HC / 2; ++j) {
        const float p0 = ex2(fmaf(sc[2 * j], mul, -m_used));
        const float p1 = ex2(fmaf(sc[2 * j + 1], mul, -m_used));
        add += p0 + p1;
        pk[j] = pack_bf16x2(p0, p1);
      }
      l += add;
      if (t >= 2 && !wait_all(&sh.pfree[b], ((t >> 1) - 1) & 1, sh, p, lane)) {
        ok = false;
        break;
      }
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < HC / 32; ++c) {
        uint32_t w16[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) w16[j] = pk[16 * c + j];
        tc_st16(tm + lane_base + Cols<D>::P + (kTok / 2) * b + (HC / 2) * half + 16 * c, w16);
      }
      tc_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh.pfull[b]);
    }
    if (ok && n_tiles > 0 &&
        wait_all(&sh.pfree[(n_tiles - 1) & 1], ((n_tiles - 1) >> 1) & 1, sh, p, lane)) {
      // the pair's normalisers add up to the row's
      sh.xl[half][r] = l;
      if (pair_sync(&sh.xend[sp], 0)) {
        const float l_row = sh.xl[0][r] + sh.xl[1][r];
        tc_fence_after();
        // the suffix partials are written by the kernels before this one
        asm volatile("griddepcontrol.wait;" ::: "memory");
        bool bad = sh.bad_prefix != 0;
        // The suffix as n contributions (max, normaliser, normalised output):
        // one row of seq_ml / seq_o, or (merge records) the partials of the
        // CTAs of the suffix kernel that cut the pair, or none.
        const int64_t row = (int64_t)seq * p.num_q_heads + hq;
        int n = 1, cf = 0, fs = 0;
        if (valid) {
          if (mismatch) {
            bad = true;
            if (half == 0) set_error(p.err_word, PA_DEVERR_PREFIX);
          }
          if (p.merge != nullptr) {
            const int4 md = reinterpret_cast<const int4 *>(p.merge)[(int64_t)seq * p.num_kv_heads + h];
            cf = md.x;
            n = md.y;
            fs = md.z;
            bad |= md.w != 0;  // a length outside the table
          }
        } else {
          n = 0;
        }
        const float2 *mls = reinterpret_cast<const float2 *>(n == 1 ? p.seq_ml : p.part_ml);
        const float *obase = n == 1 ? p.seq_o : p.part_o;
        auto crow = [&](int x) -> int64_t {
          return n == 1 ? row : ((int64_t)(cf + x) * 2 + (x == 0 ? fs : 0)) * p.num_q_heads + hq;
        };
        // running-max merge: M over every part, weights l 2^(m - M)
        float M = m_used;
        for (int x = 0; x < n; ++x) {
          const float2 ml = mls[crow(x)];
          bad |= ml.y < 0.f;  // a bad page in the suffix
          if (ml.y > 0.f) M = fmaxf(M, ml.x);
        }
        const float wp = ex2(m_used - M);
        float W = l_row * wp;
        for (int x = 0; x < n; ++x) {
          const float2 ml = mls[crow(x)];
          if (ml.y > 0.f) W += ml.y * ex2(ml.x - M);
        }
        const float inv = 1.f / W;
#pragma unroll 1
        for (int c = 0; c < HD / 16; ++c) {
          const int col = HD * half + 16 * c;
          uint32_t o16[16];
          tc_ld16(tm + lane_base + Cols<D>::O + col, o16);
          tc_wait_ld();
          if (valid) {
            float y[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) y[j] = __uint_as_float(o16[j]) * wp;
            for (int x = 0; x < n; ++x) {
              const int64_t cr = crow(x);
              const float2 ml = mls[cr];
              if (!(ml.y > 0.f)) continue;
              const float w = ml.y * ex2(ml.x - M);
              const float *os = obase + cr * D + col;
#pragma unroll
              for (int j = 0; j < 16; j += 4) {
                const float4 sv = *reinterpret_cast<const float4 *>(os + j);
                y[j + 0] += w * sv.x;
                y[j + 1] += w * sv.y;
                y[j + 2] += w * sv.z;
                y[j + 3] += w * sv.w;
              }
            }
#pragma unroll
            for (int j = 0; j < 16; ++j) y[j] = bad ? 0.f : y[j] * inv;
            const int64_t e = row * D + col;
#pragma unroll
            for (int j = 0; j < 16; j += 4)
              Elem<__nv_bfloat16>::store4(p.out, e + j,
                                          make_float4(y[j], y[j + 1], y[j + 2], y[j + 3]));
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
cudaError_t launch_d(const PrefixParams &p, cudaStream_t stream) {
  auto kern = prefix_attention_kernel<D>;
  const size_t smem = prefix_smem_bytes(D);
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
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((p.batch * p.group + kRows - 1) / kRows), (unsigned)p.num_kv_heads);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, p);
}

}  // namespace prefix

size_t prefix_smem_bytes(int head_dim) {
  const size_t nh = (size_t)head_dim / 64;
  // header, 1 KB alignment slack, the Q tile, the K and V rings; at least
  // 120 KB, so that no other CTA holding tensor memory shares the SM
  const size_t need = sizeof(prefix::Shared) + 1024 +
                      nh * prefix::kBox * (1 + prefix::kKStages + prefix::kVStages);
  return need < 120 * 1024 ? 120 * 1024 : need;
}

cudaError_t launch_prefix(const PrefixParams &p, int head_dim, cudaStream_t stream) {
  if (head_dim == 64) return prefix::launch_d<64>(p, stream);
  if (head_dim == 128) return prefix::launch_d<128>(p, stream);
  return cudaErrorInvalidValue;
}

}  // namespace pa
