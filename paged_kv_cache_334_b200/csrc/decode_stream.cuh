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
//   id, and issues one 1-D bulk copy (cp.async.bulk, no multicast) per virtual
//   page for K and for V -- only the valid token rows -- plus the sequence's
//   query rows when a sequence segment starts, into a ring of shared-memory
//   stages guarded by mbarriers.
// * Consumer warps: one per KV head.  Each keeps the online-softmax state
//   (running max, normaliser, fp32 accumulator) of the GQA group's query heads
//   for the current sequence segment, reads its head's rows of each staged
//   page with 16-byte shared-memory loads, and reduces per-(token, head) dot
//   products with a transposed butterfly.
// * A sequence split across CTAs leaves one partial per CTA in the workspace;
//   the last warp to finish (per sequence and KV head, found with an atomic
//   counter -- nobody waits) merges them and resets the counter.
//
// Every mbarrier wait is bounded; on expiry the kernel sets PA_DEVERR_TIMEOUT,
// drains its own copies (bounded) and returns.
#pragma once

#include <math.h>

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

template <typename T, int D, int G>
struct Cfg {
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
};

// ---------------------------------------------------------------------------
// PTX wrappers: mbarrier and 1-D bulk copy (no multicast).
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

struct Shared {
  uint64_t full[kMaxStages];
  uint64_t empty[kMaxStages];
  int64_t red[32];
  int64_t T, start, end, P_begin;
  int32_t s_begin, vlb_begin, g_eff, abort_flag;
};

template <typename T, int D, int G, int NCW>
__global__ void __launch_bounds__((NCW + 1) * 32, 1) decode_stream_kernel(const Params p) {
  using C = Cfg<T, D, G>;
  static_assert(sizeof(Shared) + sizeof(PageDesc) * kMaxStages * kMaxPPS +
                        sizeof(float) * NCW * C::E <= kHdrBytes,
                "header region");
  extern __shared__ __align__(128) unsigned char smem_raw[];
  Shared &sh = *reinterpret_cast<Shared *>(smem_raw);
  PageDesc *descs = reinterpret_cast<PageDesc *>(smem_raw + sizeof(Shared));
  float *s_scores = reinterpret_cast<float *>(
      smem_raw + sizeof(Shared) + sizeof(PageDesc) * kMaxStages * kMaxPPS);
  unsigned char *stages = smem_raw + p.hdr_bytes;

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

  if (active) {
    const int n_stages = (int)((end - start + p.pps - 1) / p.pps);
    if (warp == 0) {
      // ===================== producer =====================
      int32_t s = sh.s_begin;
      int32_t vlb = sh.vlb_begin;
      int64_t P_s = sh.P_begin;
      // context-length window: lane l holds seq cw + l
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
          if (!bad) bytes += 2u * (uint32_t)ntok * (uint32_t)p.row_bytes;
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
        if (lane == 0) {
          mbar_arrive_expect_tx(&sh.full[slot], bytes);
          unsigned char *st = stages + (size_t)slot * p.stage_bytes;
          for (int k = 0; k < npg; ++k) {
            const PageDesc d = descs[slot * kMaxPPS + k];
            if (!(d.flags & kBad)) {
              const int64_t off =
                  ((int64_t)d.pb * p.block_size + d.toff) * (int64_t)p.row_bytes;
              const uint32_t nb = (uint32_t)d.ntok * (uint32_t)p.row_bytes;
              bulk_g2s(st + (size_t)k * p.vpage_bytes,
                       static_cast<const unsigned char *>(p.key_cache) + off, nb, &sh.full[slot]);
              bulk_g2s(st + (size_t)(p.pps + k) * p.vpage_bytes,
                       static_cast<const unsigned char *>(p.value_cache) + off, nb,
                       &sh.full[slot]);
            }
            if (d.flags & kFirst) {
              bulk_g2s(st + (size_t)2 * p.pps * p.vpage_bytes + (size_t)k * p.q_bytes,
                       static_cast<const unsigned char *>(p.q) + (int64_t)d.seq * p.q_bytes,
                       (uint32_t)p.q_bytes, &sh.full[slot]);
            }
          }
        }
        __syncwarp();
        issued = i + 1;
      }
      if (!ok) {
        if (lane == 0) {
          sh.abort_flag = 1;
          set_error(p.err_word, PA_DEVERR_TIMEOUT);
        }
      }
      // Drain: every issued stage's copies must land before the CTA exits.
      if (lane == 0) {
        volatile int32_t dummy = 0;
        for (int i = (issued > p.stages ? issued - p.stages : 0); i < issued; ++i)
          mbar_wait(&sh.full[i % p.stages], (i / p.stages) & 1, &dummy);
      }
    } else if (warp <= NCW) {
      // ===================== consumers =====================
      const int h = warp - 1;
      const int tg = lane / C::LPT;
      const int j = lane % C::LPT;
      float *sc_buf = s_scores + (size_t)h * C::E;
      float m_run = -INFINITY, l_run = 0.f;
      float acc[G][C::EPV];
      float qf[G][C::EPV];
      bool seg_bad = false;
#pragma unroll
      for (int g = 0; g < G; ++g)
#pragma unroll
        for (int e = 0; e < C::EPV; ++e) {
          acc[g][e] = 0.f;
          qf[g][e] = 0.f;
        }
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
        const int npg = (int)min((int64_t)p.pps, end - cursor);
        cursor += npg;
        for (int k = 0; k < npg; ++k) {
          const PageDesc d = descs[slot * kMaxPPS + k];
          if (d.flags & kFirst) {
            m_run = -INFINITY;
            l_run = 0.f;
            seg_bad = false;
            const T *qs = reinterpret_cast<const T *>(st + (size_t)2 * p.pps * p.vpage_bytes +
                                                      (size_t)k * p.q_bytes);
#pragma unroll
            for (int g = 0; g < G; ++g) {
              const uint4 raw =
                  *reinterpret_cast<const uint4 *>(qs + (size_t)(h * G + g) * D + j * C::EPV);
              Elem<T>::widen(raw, qf[g]);
#pragma unroll
              for (int e = 0; e < C::EPV; ++e) {
                qf[g][e] *= p.scale_log2;
                acc[g][e] = 0.f;
              }
            }
          }
          if (d.flags & kBad) {
            seg_bad = true;
          } else {
            const unsigned char *kp = st + (size_t)k * p.vpage_bytes;
            const unsigned char *vp = st + (size_t)(p.pps + k) * p.vpage_bytes;
            for (int t0 = 0; t0 < d.ntok; t0 += C::TPI) {
              uint4 raw[C::U];
#pragma unroll
              for (int u = 0; u < C::U; ++u) {
                const int t = t0 + u * C::TPW + tg;
                raw[u] = (t < d.ntok)
                             ? *reinterpret_cast<const uint4 *>(
                                   kp + (size_t)t * p.row_bytes + (size_t)(h * D + j * C::EPV) * sizeof(T))
                             : make_uint4(0u, 0u, 0u, 0u);
              }
              float sc[C::N];
#pragma unroll
              for (int u = 0; u < C::U; ++u) {
                float kf[C::EPV];
                Elem<T>::widen(raw[u], kf);
#pragma unroll
                for (int g = 0; g < G; ++g) {
                  float dot = 0.f;
#pragma unroll
                  for (int e = 0; e < C::EPV; ++e) dot = fmaf(qf[g][e], kf[e], dot);
                  sc[u * G + g] = dot;
                }
              }
              Butterfly<C::N, C::LPT / 2>::run(sc, lane);
              if constexpr (C::N >= C::LPT) {
#pragma unroll
                for (int x = 0; x < C::NV; ++x) {
                  const int idx = j * C::NV + x;
                  const int u = idx / G, g = idx % G;
                  const int tl = u * C::TPW + tg;
                  sc_buf[tl * G + g] = (t0 + tl < d.ntok) ? sc[x] : -INFINITY;
                }
              } else {
                constexpr int R = C::LPT / C::N;
                if ((j % R) == 0) {
                  const int idx = j / R;
                  const int u = idx / G, g = idx % G;
                  const int tl = u * C::TPW + tg;
                  sc_buf[tl * G + g] = (t0 + tl < d.ntok) ? sc[0] : -INFINITY;
                }
              }
              __syncwarp();
              float sv[C::EPL];
              float tmax = -INFINITY;
#pragma unroll
              for (int x = 0; x < C::EPL; ++x) {
                const int e = lane + 32 * x;
                sv[x] = (e < C::E) ? sc_buf[e] : -INFINITY;
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
              for (int x = 0; x < C::EPL; ++x) {
                const int e = lane + 32 * x;
                const float pe = exp2f(sv[x] - m_new);
                psum += pe;
                if (e < C::E) sc_buf[e] = pe;
              }
              l_run = l_run * alpha + psum;
              // rescale only when some head's maximum moved
              if (!__all_sync(0xffffffffu, alpha == 1.f)) {
#pragma unroll
                for (int g = 0; g < G; ++g) {
                  const float a = __shfl_sync(0xffffffffu, alpha, g);
#pragma unroll
                  for (int e = 0; e < C::EPV; ++e) acc[g][e] *= a;
                }
              }
              __syncwarp();
#pragma unroll
              for (int u = 0; u < C::U; ++u) {
                const int t = t0 + u * C::TPW + tg;
                raw[u] = (t < d.ntok)
                             ? *reinterpret_cast<const uint4 *>(
                                   vp + (size_t)t * p.row_bytes + (size_t)(h * D + j * C::EPV) * sizeof(T))
                             : make_uint4(0u, 0u, 0u, 0u);
              }
#pragma unroll
              for (int u = 0; u < C::U; ++u) {
                const int tl = u * C::TPW + tg;
                float vf[C::EPV];
                Elem<T>::widen(raw[u], vf);
#pragma unroll
                for (int g = 0; g < G; ++g) {
                  const float pg = sc_buf[tl * G + g];
#pragma unroll
                  for (int e = 0; e < C::EPV; ++e) acc[g][e] = fmaf(pg, vf[e], acc[g][e]);
                }
              }
              __syncwarp();
            }
          }
          if (d.flags & kLast) {
            // ---- flush the segment of sequence d.seq for KV head h ----
            float ac[G][C::EPV];
#pragma unroll
            for (int g = 0; g < G; ++g)
#pragma unroll
              for (int e = 0; e < C::EPV; ++e) {
                float v = acc[g][e];
#pragma unroll
                for (int mask = C::LPT; mask < 32; mask <<= 1)
                  v += __shfl_xor_sync(0xffffffffu, v, mask);
                ac[g][e] = v;
              }
            float lsum = l_run;
#pragma unroll
            for (int mask = G; mask < 32; mask <<= 1)
              lsum += __shfl_xor_sync(0xffffffffu, lsum, mask);
            const int64_t hrow0 = (int64_t)d.seq * p.num_q_heads + (int64_t)h * G;
            if (d.n_contrib == 1) {
#pragma unroll
              for (int g = 0; g < G; ++g) {
                // every lane takes part in the shuffle; only one token group stores
                const float lg = __shfl_sync(0xffffffffu, lsum, g);
                const float inv = 1.f / lg;
                if (tg == 0) {
#pragma unroll
                  for (int e = 0; e < C::EPV; ++e)
                    Elem<T>::store1(p.out, (hrow0 + g) * D + j * C::EPV + e,
                                    seg_bad ? 0.f : ac[g][e] * inv);
                }
              }
            } else {
              const int my_slot = d.slot_bits & 1;
              const int64_t prow = ((int64_t)c * 2 + my_slot) * p.num_q_heads + (int64_t)h * G;
              if (lane < G) {
                p.part_ml[(prow + lane) * 2 + 0] = m_run;
                p.part_ml[(prow + lane) * 2 + 1] = seg_bad ? -1.f : lsum;
              }
#pragma unroll
              for (int g = 0; g < G; ++g) {
                const float lg = __shfl_sync(0xffffffffu, lsum, g);
                if (tg == 0) {
#pragma unroll
                  for (int e = 0; e < C::EPV; ++e)
                    p.part_o[(prow + g) * D + j * C::EPV + e] = seg_bad ? 0.f : ac[g][e] / lg;
                }
              }
              __threadfence();
              __syncwarp();
              int32_t old = 0;
              int32_t *cnt = p.counters + (int64_t)d.seq * p.num_kv_heads + h;
              if (lane == 0) old = atomicAdd(cnt, 1);
              old = __shfl_sync(0xffffffffu, old, 0);
              if (old == d.n_contrib - 1) {
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
                  const int cc = d.c_first + x;
                  const int sl = (x == 0) ? first_slot : 0;
                  const int64_t r = ((int64_t)cc * 2 + sl) * p.num_q_heads + (int64_t)h * G;
#pragma unroll
                  for (int g = 0; g < G; ++g) {
                    const float l = __ldcg(p.part_ml + (r + g) * 2 + 1);
                    if (l < 0.f) any_bad = true;
                    M[g] = fmaxf(M[g], __ldcg(p.part_ml + (r + g) * 2 + 0));
                  }
                }
                float O[G][C::EPV];
#pragma unroll
                for (int g = 0; g < G; ++g)
#pragma unroll
                  for (int e = 0; e < C::EPV; ++e) O[g][e] = 0.f;
                for (int x = 0; x < d.n_contrib; ++x) {
                  const int cc = d.c_first + x;
                  const int sl = (x == 0) ? first_slot : 0;
                  const int64_t r = ((int64_t)cc * 2 + sl) * p.num_q_heads + (int64_t)h * G;
#pragma unroll
                  for (int g = 0; g < G; ++g) {
                    const float w = __ldcg(p.part_ml + (r + g) * 2 + 1) *
                                    exp2f(__ldcg(p.part_ml + (r + g) * 2 + 0) - M[g]);
                    W[g] += w;
                    if (tg == 0) {
#pragma unroll
                      for (int e = 0; e < C::EPV; ++e)
                        O[g][e] += w * __ldcg(p.part_o + (r + g) * D + j * C::EPV + e);
                    }
                  }
                }
                if (tg == 0) {
#pragma unroll
                  for (int g = 0; g < G; ++g) {
                    const float inv = 1.f / W[g];
#pragma unroll
                    for (int e = 0; e < C::EPV; ++e)
                      Elem<T>::store1(p.out, (hrow0 + g) * D + j * C::EPV + e,
                                      any_bad ? 0.f : O[g][e] * inv);
                  }
                }
                if (lane == 0) atomicExch(cnt, 0);
              }
            }
            if (seg_bad && lane == 0) set_error(p.err_word, PA_DEVERR_BLOCK_ID);
#pragma unroll
            for (int g = 0; g < G; ++g)
#pragma unroll
              for (int e = 0; e < C::EPV; ++e) acc[g][e] = 0.f;
            m_run = -INFINITY;
            l_run = 0.f;
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

// Host side: launch the instantiation for (head_dim, group, Hkv) of dtype T.
// Explicitly instantiated once per dtype in its own translation unit.
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

template <typename T, int D, int G>
cudaError_t launch_hkv(const Params &p, int hkv, size_t smem, cudaStream_t stream) {
  if (hkv == 4) return launch_one<T, D, G, 4>(p, smem, stream);
  if (hkv == 8) return launch_one<T, D, G, 8>(p, smem, stream);
  return cudaErrorInvalidValue;
}

template <typename T, int D>
cudaError_t launch_group(const Params &p, int group, int hkv, size_t smem, cudaStream_t stream) {
  switch (group) {
    case 1: return launch_hkv<T, D, 1>(p, hkv, smem, stream);
    case 2: return launch_hkv<T, D, 2>(p, hkv, smem, stream);
    case 4: return launch_hkv<T, D, 4>(p, hkv, smem, stream);
    case 8: return launch_hkv<T, D, 8>(p, hkv, smem, stream);
    default: return cudaErrorInvalidValue;
  }
}

template <typename T>
cudaError_t launch_stream_dtype(const Params &p, int head_dim, int group, int hkv, size_t smem,
                                cudaStream_t stream) {
  if (head_dim == 64) return launch_group<T, 64>(p, group, hkv, smem, stream);
  if (head_dim == 128) return launch_group<T, 128>(p, group, hkv, smem, stream);
  return cudaErrorInvalidValue;
}

}  // namespace stream
}  // namespace pa
