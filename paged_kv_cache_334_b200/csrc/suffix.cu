// suffix.cu -- decode attention on the 5th-generation tensor cores (tcgen05)
// when one KV head serves 64 or 128 query heads: the private part of every
// sequence for pa_decode_shared_prefix, and with no prefix the whole of
// pa_decode / pa_forward_decode (then finish_kernel merges and writes bf16).
//
// Page "Operators and compilers: inference attention and KV kernels",
// section 4.1: with that many query heads per KV head, decode attention does
// tens of flops per byte of KV and is a dense contraction, not a stream.  The
// G query heads of one (sequence, KV head) pair are the M side (G = 64 or
// 128) of S = Q K^T and O += P V, against tiles of 128 tokens gathered from
// the pair's own pages (one tiled copy per page and 64-wide half of
// head_dim), with the online softmax of the [route] page "From correct to
// faster: the PagedAttention optimisation route", section "The core idea of
// high-performance PagedAttention" (running max, rescaled sum, no score
// matrix in memory).
//
// Work split: the 128-token tiles of all pairs, in (sequence, KV head, tile)
// order, are cut into one contiguous range per CTA (one CTA per SM), so every
// SM gets the same number of tiles whatever the mix of lengths.  A pair that
// lies inside one range leaves (max, normaliser, normalised output) in
// seq_ml / seq_o; a pair cut by range boundaries leaves one partial per CTA
// it touches (slot 1 of the CTA where it starts inside the range, slot 0 of
// the others), and the CTA holding its last tile records (first CTA, number
// of CTAs, slot of the first) for the prefix kernel, which folds the
// partials in with the same running-max rescaling.
//
// 11 warps:
//   warp 0     walks the range: page ids two tiles ahead (4-byte asynchronous
//              copies into shared memory), one descriptor per tile, the Q
//              tile of each pair it starts, K and V tiles into separate rings
//              (tiled copies, no multicast);
//   warp 1     tcgen05.mma: S_b = Q K^T of the next tile and O += P V of the
//              previous one, whichever has its inputs first;
//   warps 2-9  softmax, two warps per tensor-memory subpartition (each owns
//              half of a tile's 128 columns and of O's), and the epilogue of
//              every pair segment;
//   warp 10    (group 64) the epilogue's tiled stores from a staging buffer:
//              issuing a store waits while the SM's copy engine is busy with
//              tile loads, so no other warp issues one.
// Tensor memory (512 columns): O [0, D), S_b [D + 128 b), P_b (bf16 pairs)
// [D + 256 + 64 b).  An M = 64 accumulator keeps row r in lane
// (r % 16) + 32 (r / 16): lanes 0-15 of each softmax warp own rows, lanes
// 16-31 compute on lanes no product reads.  The running max is raised only
// when a score exceeds it by more than 8 (log2 units), so P < 2^8 and O is
// rescaled rarely; O and the normaliser share the maximum, so the result is
// exact.  Every wait is bounded (PA_DEVERR_TIMEOUT on expiry).
#include <cuda_bf16.h>
#include <math.h>

#include "pa_common.cuh"
#include "pa_launch.h"
#include "sm100_ptx.cuh"

namespace pa {
namespace suffix {

using namespace pa::stream;

constexpr int kTok = 128;             // tokens per tile: N of S, K of P V
constexpr int kThreads = 352;         // 11 warps
constexpr uint32_t kTmemCols = 512;
constexpr float kSlack = 8.f;         // lazy rescaling threshold (log2 units)
constexpr int kTileBox = kTok * 128;  // bytes of one 64-wide half of a K or V tile
constexpr int kRing = 8;              // tile descriptors in flight
constexpr int kMaxPPT = 16;           // pages per tile (block_size >= 8)
constexpr int kQStages = 2, kVStages = 2, kMaxKStages = 3;
constexpr int kFirst = 1, kLast = 2, kBad = 4, kDirect = 8, kPairEnd = 16;
// At least this much shared memory per CTA keeps one CTA per SM: tensor
// memory is allocated whole (512 columns) and is not shared.
constexpr size_t kMinSmem = 120 * 1024;

template <int D, int M>
struct Cfg {
  static constexpr int NH = D / 64;                          // 64-wide halves of head_dim
  static constexpr int kQBox = M * 128;                      // one half of a Q tile
  static constexpr int KS = D == 128 ? 2 : 3;                // K stages within 227 KB
  // group 64: a staging buffer for the epilogue's tiled stores (M x D fp32)
  static constexpr int kStage = M == 64 ? M * D * 4 : 0;
  static constexpr uint32_t O = 0, S = D, P = D + 2 * kTok;  // tensor-memory columns
};

struct alignas(16) Desc {
  int32_t s, h, ntok, flags;
  int32_t row;  // first output row: of seq_ml / seq_o (kDirect) or of part_ml / part_o
  int32_t pad[3];
};

struct alignas(16) Shared {
  uint64_t qfull[kQStages], qempty[kQStages], kfull[kMaxKStages], kempty[kMaxKStages];
  uint64_t vfull[kVStages], vempty[kVStages];
  uint64_t sfull[2], sfree[2], pfull[2], pfree[2], ofull, ofree, mma_done;
  uint64_t staged, stfree;  // epilogue staging (group 64): written / read by the store
  uint64_t dfull[kRing], dempty[kRing];
  uint64_t xbar[4][2], xend[4];  // softmax pair handshakes (per subpartition)
  int64_t red[32];
  int64_t P_begin;
  int32_t s_begin, off_begin, abort_flag;
  uint32_t tmem_base;
  Desc desc[kRing];
  int32_t pids[kRing][kMaxPPT];  // page ids of a tile, written by asynchronous copies
  int64_t slots[kRing];          // new-token slot of the pair ending in the tile
  float xm[2][2][128];           // [tile parity][column half][row] partial row maxima
  float xl[2][128];              // [column half][row] partial normalisers
  float2 mlst[128];              // epilogue staging of (max, normaliser) per row
  int32_t st_row, st_direct;     // the staged pair's first output row, and where it goes
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
                                         const SuffixParams &p, int lane) {
  if (__all_sync(0xffffffffu, mbar_try_wait(bar, parity))) return true;
  return wait_all_slow(bar, parity, sh, p.err_word, lane);
}

// Exclusive prefix sum of v over the CTA; *total = the sum of every thread's v.
__device__ __forceinline__ int64_t cta_scan(int64_t v, int64_t *red, int64_t *total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  int64_t inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int64_t y = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += y;
  }
  if (lane == 31) red[warp] = inc;
  __syncthreads();
  int64_t base = 0, tot = 0;
  for (int w = 0; w < nw; ++w) {
    const int64_t x = red[w];
    if (w < warp) base += x;
    tot += x;
  }
  __syncthreads();
  *total = tot;
  return base + inc - v;
}

// Tokens of sequence s past the prefix (0 for a length outside the table).
__device__ __forceinline__ int32_t suffix_len(const SuffixParams &p, int s) {
  const int32_t ctx = p.context_lens[s];
  const int32_t ptok = p.prefix_blocks * p.block_size;
  if (ctx < 0 || (int64_t)ctx > (int64_t)p.table_stride * p.block_size) return 0;
  return ctx > ptok ? ctx - ptok : 0;
}
__device__ __forceinline__ int32_t tiles_of(int32_t len) { return (len + kTok - 1) / kTok; }
// The CTA whose range [c T / g, (c + 1) T / g) holds tile u.
__device__ __forceinline__ int32_t owner(int64_t u, int64_t T, int32_t g) {
  return (int32_t)(((u + 1) * g + T - 1) / T - 1);
}

// The producer's position in its range (all lanes in lock step).
struct Walker {
  int32_t s, h, j, n, len;  // tile j of pair (s, h); the pair's tiles; s's suffix tokens
  int64_t P;                // index of the pair's tile 0
  int32_t cw, cw_len;       // lane l holds suffix_len(cw + l)

  __device__ __forceinline__ void load_window(const SuffixParams &p, int lane) {
    cw_len = (cw + lane < p.batch) ? suffix_len(p, cw + lane) : 0;
  }
  __device__ __forceinline__ void init(const SuffixParams &p, int32_t s0, int32_t off0,
                                       int64_t P0, int lane) {
    s = s0;
    cw = s0;
    load_window(p, lane);
    len = __shfl_sync(0xffffffffu, cw_len, 0);
    n = tiles_of(len);
    h = off0 / n;
    j = off0 - h * n;
    P = P0 + (int64_t)h * n;
  }
  // Next tile; called only while the range has tiles left.
  __device__ __forceinline__ void advance(const SuffixParams &p, int lane) {
    if (++j < n) return;
    j = 0;
    P += n;
    if (++h < p.num_kv_heads) return;
    h = 0;
    int32_t nxt = s + 1;
    for (;;) {
      if (nxt >= p.batch) {  // unreachable inside a range; ends the walk
        s = p.batch;
        len = 0;
        n = 1;
        return;
      }
      if (nxt >= cw + 32) {
        cw = nxt;
        load_window(p, lane);
      }
      const uint32_t m = __ballot_sync(0xffffffffu, cw + lane >= nxt && cw_len > 0);
      if (m) {
        const int l = __ffs(m) - 1;
        s = cw + l;
        len = __shfl_sync(0xffffffffu, cw_len, l);
        n = tiles_of(len);
        return;
      }
      nxt = cw + 32;
    }
  }
};

// A tile as the producer issues it (lane-uniform values).
struct Tile {
  int32_t s, h, ntok, npg, flags, row;
};

template <int D, int M>
__global__ void __launch_bounds__(kThreads, 1)
    suffix_attention_kernel(const __grid_constant__ SuffixParams p) {
  using C = Cfg<D, M>;
  constexpr int NH = C::NH, KS = C::KS;
  extern __shared__ __align__(128) unsigned char smem_raw[];
  Shared &sh = *reinterpret_cast<Shared *>(smem_raw);
  unsigned char *tiles =
      smem_raw + (((smem_u32(smem_raw) + sizeof(Shared) + 1023u) & ~1023u) - smem_u32(smem_raw));
  unsigned char *qring = tiles;                             // Q stage: NH x kQBox
  unsigned char *kring = qring + kQStages * NH * C::kQBox;  // K stage: NH x kTileBox
  unsigned char *vring = kring + KS * NH * kTileBox;        // V stage: NH x kTileBox
  unsigned char *stg = vring + kVStages * NH * kTileBox;    // epilogue staging (group 64)
  auto q_stage = [&](int s) { return qring + (size_t)s * NH * C::kQBox; };
  auto k_stage = [&](int s) { return kring + (size_t)s * NH * kTileBox; };
  auto v_stage = [&](int s) { return vring + (size_t)s * NH * kTileBox; };

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int c = blockIdx.x;
  if (tid == 0) {
    prefetch_tensormap(&p.tmap_q);
    prefetch_tensormap(&p.tmap_k);
    prefetch_tensormap(&p.tmap_v);
  }
  // Launched with programmatic stream serialisation: nothing is read before
  // the previous kernel of the stream has finished.
  asm volatile("griddepcontrol.wait;" ::: "memory");

  if (tid == 0) {
    for (int i = 0; i < kQStages; ++i) {
      mbar_init(&sh.qfull[i], 1);
      mbar_init(&sh.qempty[i], 1);
    }
    for (int i = 0; i < KS; ++i) {
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
    mbar_init(&sh.ofull, 1);
    mbar_init(&sh.ofree, 8);
    mbar_init(&sh.mma_done, 1);
    mbar_init(&sh.staged, 8);
    mbar_init(&sh.stfree, 1);
    for (int i = 0; i < kRing; ++i) {
      mbar_init(&sh.dfull[i], 1);
      mbar_init(&sh.dempty[i], 9);  // the tensor-core warp and the 8 softmax warps
    }
    for (int q = 0; q < 4; ++q) {
      mbar_init(&sh.xbar[q][0], 64);
      mbar_init(&sh.xbar[q][1], 64);
      mbar_init(&sh.xend[q], 64);
    }
    sh.abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }

  // ---- This CTA's range of tiles: T = Hkv * sum of the sequences' tiles.
  int64_t T = 0, start = 0, end = 0;
  int32_t g_eff = 0;
  if (p.batch <= kThreads) {
    const int64_t v = (tid < p.batch) ? (int64_t)p.num_kv_heads * tiles_of(suffix_len(p, tid)) : 0;
    const int64_t P = cta_scan(v, sh.red, &T);
    g_eff = (int32_t)(T < p.grid ? T : p.grid);
    if (c < g_eff) {
      start = (int64_t)c * T / g_eff;
      end = (int64_t)(c + 1) * T / g_eff;
      if (v > 0 && P <= start && start < P + v) {
        sh.s_begin = tid;
        sh.off_begin = (int32_t)(start - P);
        sh.P_begin = P;
      }
    }
  } else {
    for (int base = 0; base < p.batch; base += kThreads) {
      const int s = base + tid;
      const int64_t v = (s < p.batch) ? (int64_t)p.num_kv_heads * tiles_of(suffix_len(p, s)) : 0;
      int64_t tot;
      cta_scan(v, sh.red, &tot);
      T += tot;
    }
    g_eff = (int32_t)(T < p.grid ? T : p.grid);
    if (c < g_eff) {
      start = (int64_t)c * T / g_eff;
      end = (int64_t)(c + 1) * T / g_eff;
      int64_t run = 0;
      for (int base = 0; base < p.batch; base += kThreads) {
        const int s = base + tid;
        const int64_t v = (s < p.batch) ? (int64_t)p.num_kv_heads * tiles_of(suffix_len(p, s)) : 0;
        int64_t tot;
        const int64_t P = run + cta_scan(v, sh.red, &tot);
        if (v > 0 && P <= start && start < P + v) {
          sh.s_begin = s;
          sh.off_begin = (int32_t)(start - P);
          sh.P_begin = P;
        }
        run += tot;
        if (run > start) break;  // uniform: every thread sees the same `run`
      }
    }
  }
  if (warp == 1) {
    tc_alloc(&sh.tmem_base, kTmemCols);
    tc_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = sh.tmem_base;
  // The prefix kernel that follows may be scheduled from here on (it waits
  // for this grid before reading what it writes).  Only now: every CTA of
  // this grid holds its tensor memory, so a CTA of the next kernel on the
  // same SM waits for it in its own allocation, never the other way round.
  asm volatile("griddepcontrol.launch_dependents;");
  const int n_units = (int)(end - start);
  const int G = p.group, Hq = p.num_q_heads, bs = p.block_size;
  const int ppt = kTok / bs;  // pages per tile

  if (warp == 0 && n_units > 0) {
    // ===================== page walk and tiled copies =====================
    Walker wk;
    wk.init(p, sh.s_begin, sh.off_begin, sh.P_begin, lane);
    // Tile u's descriptor; its page ids start moving into shared memory.
    auto fetch = [&](int u) -> Tile {
      Tile x;
      x.s = wk.s;
      x.h = wk.h;
      x.ntok = min(kTok, wk.len - wk.j * kTok);
      x.npg = (x.ntok + bs - 1) / bs;
      const bool first = wk.j == 0 || u == 0;
      const bool pair_end = wk.j == wk.n - 1;
      const bool last = pair_end || u == n_units - 1;
      const bool direct = wk.P >= start && wk.P + wk.n <= end;
      x.flags = (first ? kFirst : 0) | (last ? kLast : 0) | (direct ? kDirect : 0) |
                (pair_end ? kPairEnd : 0);
      const int slot = (start < wk.P) ? 1 : 0;
      x.row = direct ? wk.s * Hq + wk.h * G : (c * 2 + slot) * Hq + wk.h * G;
      if (pair_end && lane == 0) {
        // the owner of the pair's last tile tells the prefix kernel where
        // its partials are
        const int32_t c_first = owner(wk.P, T, g_eff);
        const int64_t st_first = (int64_t)c_first * T / g_eff;
        reinterpret_cast<int4 *>(p.merge)[(int64_t)wk.s * p.num_kv_heads + wk.h] =
            make_int4(c_first, c - c_first + 1, st_first < wk.P ? 1 : 0, 0);
      }
      const int32_t *trow =
          p.block_tables + (int64_t)wk.s * p.table_stride + p.prefix_blocks + wk.j * ppt;
      if (lane < x.npg) cp_async_4(&sh.pids[u % kRing][lane], trow + lane);
      if (pair_end && p.slot_mapping != nullptr && lane == 0)
        cp_async_8(&sh.slots[u % kRing], p.slot_mapping + wk.s);
      cp_async_commit();
      if (u + 1 < n_units) wk.advance(p, lane);
      return x;
    };
    Tile t0 = fetch(0), t1 = t0, tv = t0;
    if (n_units > 1) {
      t1 = fetch(1);
    } else {
      cp_async_commit();
    }
    const uint32_t page_bytes = (uint32_t)bs * 128u;
    int32_t pb_prev = 0;
    int qseg = 0, issued_k = 0, issued_v = 0;
    bool ok = true;
    for (int u = 0; u <= n_units && ok; ++u) {
      int32_t pb = 0;
      if (u < n_units) {
        // tile u's page ids have landed (tile u + 1's may still be moving)
        cp_async_wait<1>();
        const bool in = lane < t0.npg;
        pb = in ? sh.pids[u % kRing][lane] : 0;
        const bool bad_pb = in && (pb < 0 || pb >= p.num_blocks);
        if (bad_pb) pb = 0;  // any valid page: the pair's output is flagged
        bool bad = __any_sync(0xffffffffu, bad_pb);
        if (bad && lane == 0) set_error(p.err_word, PA_DEVERR_BLOCK_ID);
        if ((t0.flags & kPairEnd) && p.slot_mapping != nullptr) {
          // the pair's newest token (its last tile's last token) must have
          // been written to the slot the table gives it
          const int64_t slot = __shfl_sync(0xffffffffu, sh.slots[u % kRing], 0);
          const int32_t pb_last = __shfl_sync(0xffffffffu, pb, t0.npg - 1);
          const int64_t want = (int64_t)pb_last * bs + (t0.ntok - 1) % bs;
          if (slot >= 0 && (bad || slot != want)) {
            bad = true;
            if (lane == 0) set_error(p.err_word, PA_DEVERR_SLOT);
          }
        }
        if (u >= kRing && !wait_all(&sh.dempty[u % kRing], ((u / kRing) - 1) & 1, sh, p, lane)) {
          ok = false;
          break;
        }
        if (lane == 0) {
          Desc d;
          d.s = t0.s;
          d.h = t0.h;
          d.ntok = t0.ntok;
          d.flags = t0.flags | (bad ? kBad : 0);
          d.row = t0.row;
          d.pad[0] = d.pad[1] = d.pad[2] = 0;
          sh.desc[u % kRing] = d;
          mbar_arrive(&sh.dfull[u % kRing]);
        }
        if (t0.flags & kFirst) {
          const int qs = qseg % kQStages;
          if (qseg >= kQStages &&
              !wait_all(&sh.qempty[qs], ((qseg / kQStages) - 1) & 1, sh, p, lane)) {
            ok = false;
            break;
          }
          if (lane == 0) {
            mbar_arrive_expect_tx(&sh.qfull[qs], (uint32_t)(NH * C::kQBox));
            for (int dh = 0; dh < NH; ++dh)
              tma_load_3d(q_stage(qs) + dh * C::kQBox, &p.tmap_q, dh * 64, t0.h * G, t0.s,
                          &sh.qfull[qs]);
          }
          ++qseg;
        }
        const int ks = u % KS;
        if (u >= KS && !wait_all(&sh.kempty[ks], ((u / KS) - 1) & 1, sh, p, lane)) {
          ok = false;
          break;
        }
        if (lane == 0)
          mbar_arrive_expect_tx(&sh.kfull[ks], (uint32_t)NH * (uint32_t)t0.npg * page_bytes);
        __syncwarp();
        if (lane < t0.npg) {
          for (int dh = 0; dh < NH; ++dh)
            tma_load_3d(k_stage(ks) + dh * kTileBox + lane * page_bytes, &p.tmap_k, dh * 64,
                        pb * bs, t0.h, &sh.kfull[ks]);
        }
        issued_k = u + 1;
      }
      if (u >= 1) {
        // V runs one tile behind K: it is needed only after the softmax
        const int v = u - 1, vs = v % kVStages;
        if (v >= kVStages && !wait_all(&sh.vempty[vs], ((v / kVStages) - 1) & 1, sh, p, lane)) {
          ok = false;
          break;
        }
        if (lane == 0)
          mbar_arrive_expect_tx(&sh.vfull[vs], (uint32_t)NH * (uint32_t)tv.npg * page_bytes);
        __syncwarp();
        if (lane < tv.npg) {
          for (int dh = 0; dh < NH; ++dh)
            tma_load_3d(v_stage(vs) + dh * kTileBox + lane * page_bytes, &p.tmap_v, dh * 64,
                        pb_prev * bs, tv.h, &sh.vfull[vs]);
        }
        issued_v = u;
      }
      if (u < n_units) {
        tv = t0;
        pb_prev = pb;
        t0 = t1;
        if (u + 2 < n_units) {
          t1 = fetch(u + 2);
        } else {
          cp_async_commit();  // keeps one group per tile for the wait above
        }
      }
    }
    cp_async_wait<0>();
    // Drain: every issued copy lands before the CTA exits (they have in the
    // normal course; after an abort some may still be in flight).
    if (lane == 0) {
      volatile int32_t never = 0;
      for (int i = (issued_k > KS ? issued_k - KS : 0); i < issued_k; ++i)
        mbar_wait(&sh.kfull[i % KS], (i / KS) & 1, &never);
      for (int i = (issued_v > kVStages ? issued_v - kVStages : 0); i < issued_v; ++i)
        mbar_wait(&sh.vfull[i % kVStages], (i / kVStages) & 1, &never);
      for (int i = (qseg > kQStages ? qseg - kQStages : 0); i < qseg; ++i)
        mbar_wait(&sh.qfull[i % kQStages], (i / kQStages) & 1, &never);
    }
    __syncwarp();
  } else if (warp == 1 && n_units > 0) {
    // ===================== tensor-core issue =====================
    // Two products are pending at a time, S = Q K^T of the next tile and
    // O += P V of an earlier one; whichever has its inputs first is issued
    // first (a bounded poll, like every wait).  A pair's last P V thus never
    // waits for the next tile's K, and its epilogue starts as early as it can.
    const uint32_t id_s = idesc_bf16(M, kTok, false);
    const uint32_t id_o = idesc_bf16(M, D, true);
    struct Pend {
      int32_t flags, ntok, seg;
    };
    auto ready = [&](uint64_t *bar, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, mbar_test_wait(bar, parity));
    };
    auto issue_pv = [&](int v, const Pend &x) {
      const int b = v & 1, vs = v % kVStages;
      const bool first = (x.flags & kFirst) != 0;
      if (x.ntok < kTok) {
        // rows past the pair's tokens may hold anything (0 * NaN is NaN)
        unsigned char *vsm = v_stage(vs);
        const int units = (kTok - x.ntok) * 8;
        for (int i = lane; i < units * NH; i += 32) {
          const int dh = i / units, rem = i - dh * units;
          *reinterpret_cast<uint4 *>(vsm + dh * kTileBox + (x.ntok + (rem >> 3)) * 128 +
                                     (rem & 7) * 16) = make_uint4(0u, 0u, 0u, 0u);
        }
        fence_proxy_async_smem();
      }
      __syncwarp();
      tc_fence_after();
      if (lane == 0) {
        const uint32_t va = smem_u32(v_stage(vs));
        for (int ks = 0; ks < kTok / 16; ++ks)
          tc_mma_ts(tm + C::O, tm + C::P + 64 * b + 8 * ks,
                    sw128_desc(va + 2048 * ks, (uint32_t)kTileBox, 1024), id_o,
                    (first && ks == 0) ? 0u : 1u);
        tc_commit(&sh.pfree[b]);
        tc_commit(&sh.vempty[vs]);
        if (x.flags & kLast) tc_commit(&sh.ofull);
      }
      __syncwarp();
    };
    Pend pend0{0, 0, 0}, pend1{0, 0, 0};  // tiles whose S is issued, by parity
    Desc du{};
    bool have_d = false;  // descriptor of tile u read
    int u = 0, v = 0;     // next S, next P V
    int seg = -1;         // pair segment of tile u (once its descriptor is read)
    uint64_t t_last = global_ns();
    for (uint32_t spin = 0; v < n_units; ++spin) {
      bool progressed = false;
      if (v < u) {
        const Pend x = (v & 1) ? pend1 : pend0;
        // a pair's first product overwrites O: the previous pair's epilogue
        // must have read it
        if (ready(&sh.vfull[v % kVStages], (v / kVStages) & 1) &&
            ready(&sh.pfull[v & 1], (v >> 1) & 1) &&
            (!(x.flags & kFirst) || x.seg == 0 || ready(&sh.ofree, (x.seg - 1) & 1))) {
          issue_pv(v, x);
          ++v;
          progressed = true;
        }
      }
      if (u < n_units && u - v <= 1) {
        if (!have_d && ready(&sh.dfull[u % kRing], (u / kRing) & 1)) {
          du = sh.desc[u % kRing];
          __syncwarp();
          if (lane == 0) mbar_arrive(&sh.dempty[u % kRing]);
          if (du.flags & kFirst) ++seg;
          have_d = true;
          progressed = true;
        }
        const int b = u & 1, ks = u % KS;
        if (have_d &&
            (!(du.flags & kFirst) || ready(&sh.qfull[seg % kQStages], (seg / kQStages) & 1)) &&
            ready(&sh.kfull[ks], (u / KS) & 1) &&
            (u < 2 || ready(&sh.sfree[b], ((u >> 1) - 1) & 1))) {
          tc_fence_after();
          if (lane == 0) {
            const uint32_t qa = smem_u32(q_stage(seg % kQStages)), ka = smem_u32(k_stage(ks));
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t qoff = (uint32_t)(kk >> 2) * C::kQBox + (uint32_t)(kk & 3) * 32;
              const uint32_t koff = (uint32_t)(kk >> 2) * kTileBox + (uint32_t)(kk & 3) * 32;
              tc_mma_ss(tm + C::S + kTok * b, sw128_desc(qa + qoff, 16, 1024),
                        sw128_desc(ka + koff, 16, 1024), id_s, kk > 0 ? 1u : 0u);
            }
            tc_commit(&sh.sfull[b]);
            tc_commit(&sh.kempty[ks]);  // K stage free once S is computed
            if (du.flags & kLast) tc_commit(&sh.qempty[seg % kQStages]);
          }
          __syncwarp();
          const Pend x{du.flags, du.ntok, seg};
          if (u & 1) {
            pend1 = x;
          } else {
            pend0 = x;
          }
          ++u;
          have_d = false;
          progressed = true;
        }
      }
      if (progressed) {
        t_last = global_ns();
      } else if ((spin & 15) == 0 &&
                 (*reinterpret_cast<volatile int32_t *>(&sh.abort_flag) ||
                  global_ns() - t_last > kWaitLimitNs)) {
        if (lane == 0) {
          sh.abort_flag = 1;
          set_error(p.err_word, PA_DEVERR_TIMEOUT);
        }
        break;
      }
    }
  } else if (warp >= 2 && warp < 10 && n_units > 0) {
    // ===================== softmax and epilogue =====================
    const int sp = warp & 3;           // tensor-memory subpartition
    const int half = (warp - 2) >> 2;  // which 64 of a tile's 128 columns
    const uint32_t lane_base = (uint32_t)(32 * sp) << 16;
    const bool row_ok = (M == 128) || lane < 16;
    // this thread's row of the tile (M = 64: lanes 16-31 get spare indices)
    const int r = (M == 128) ? 32 * sp + lane : 16 * sp + (lane & 15) + (lane >= 16 ? 64 : 0);
    constexpr int HC = kTok / 2;  // score columns per thread
    constexpr int HD = D / 2;     // output columns per thread
    auto pair_sync = [&](uint64_t *bar, uint32_t parity) -> bool {
      mbar_arrive(bar);
      return wait_all(bar, parity, sh, p, lane);
    };
    const float sl = p.scale_log2;
    float m_used = -INFINITY, l = 0.f;
    bool seg_bad = false;
    int seg = -1;
    for (int u = 0; u < n_units; ++u) {
      const int b = u & 1;
      if (!wait_all(&sh.dfull[u % kRing], (u / kRing) & 1, sh, p, lane)) break;
      const Desc d = sh.desc[u % kRing];
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh.dempty[u % kRing]);
      const bool first = (d.flags & kFirst) != 0;
      if (first) {
        ++seg;
        m_used = -INFINITY;
        l = 0.f;
        seg_bad = false;
      }
      seg_bad |= (d.flags & kBad) != 0;
      const int ntok = d.ntok;
      if (!wait_all(&sh.sfull[b], (u >> 1) & 1, sh, p, lane)) break;
      tc_fence_after();
      float sc[HC];
#pragma unroll
      for (int cc = 0; cc < HC / 16; ++cc) {
        uint32_t raw[16];
        tc_ld16(tm + lane_base + C::S + kTok * b + HC * half + 16 * cc, raw);
#pragma unroll
        for (int j = 0; j < 16; ++j) sc[16 * cc + j] = __uint_as_float(raw[j]);
      }
      tc_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh.sfree[b]);
      // with scale > 0 the maximum of the scaled scores is the scaled
      // maximum: full tiles stay raw, 2^(s scale - m) is one multiply-add
      const bool scaled = ntok < kTok || sl < 0.f;
      if (scaled) {
#pragma unroll
        for (int j = 0; j < HC; ++j) sc[j] = (HC * half + j < ntok) ? sc[j] * sl : -INFINITY;
      }
      float mx = -INFINITY;
#pragma unroll
      for (int j = 0; j < HC; ++j) mx = fmaxf(mx, sc[j]);
      sh.xm[b][half][r] = scaled ? mx : mx * sl;
      if (!pair_sync(&sh.xbar[sp][b], (u >> 1) & 1)) break;
      const float m_new = fmaxf(m_used, fmaxf(sh.xm[b][0][r], sh.xm[b][1][r]));
      const bool need = row_ok && m_new > m_used + kSlack;
      if (__any_sync(0xffffffffu, need)) {
        const float f = need ? ex2(m_used - m_new) : 1.f;
        if (!first) {
          // O holds this pair's earlier tiles: wait for the last product,
          // rescale this warp's half of the columns
          if (!wait_all(&sh.pfree[(u - 1) & 1], ((u - 1) >> 1) & 1, sh, p, lane)) break;
          tc_fence_after();
#pragma unroll 1
          for (int cc = 0; cc < HD / 16; ++cc) {
            uint32_t o16[16];
            tc_ld16(tm + lane_base + C::O + HD * half + 16 * cc, o16);
            tc_wait_ld();
#pragma unroll
            for (int j = 0; j < 16; ++j) o16[j] = __float_as_uint(__uint_as_float(o16[j]) * f);
            tc_st16(tm + lane_base + C::O + HD * half + 16 * cc, o16);
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
      if (u >= 2 && !wait_all(&sh.pfree[b], ((u >> 1) - 1) & 1, sh, p, lane)) break;
      tc_fence_after();
#pragma unroll
      for (int cc = 0; cc < HC / 32; ++cc) {
        uint32_t w16[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) w16[j] = pk[16 * cc + j];
        tc_st16(tm + lane_base + C::P + (kTok / 2) * b + (HC / 2) * half + 16 * cc, w16);
      }
      tc_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh.pfull[b]);
      if (d.flags & kLast) {
        // ---- epilogue of this pair segment
        if (!wait_all(&sh.ofull, seg & 1, sh, p, lane)) break;
        tc_fence_after();
        sh.xl[half][r] = l;  // the pair of warps' normalisers add up to the row's
        if (!pair_sync(&sh.xend[sp], seg & 1)) break;
        const float l_row = sh.xl[0][r] + sh.xl[1][r];
        uint32_t o[HD / 16][16];
#pragma unroll
        for (int cc = 0; cc < HD / 16; ++cc)
          tc_ld16(tm + lane_base + C::O + HD * half + 16 * cc, o[cc]);
        tc_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh.ofree);  // the next pair may overwrite O
        const bool direct = (d.flags & kDirect) != 0;
        const float inv = seg_bad ? 0.f : 1.f / l_row;
        if constexpr (M == 64) {
          // Stage the rows in the 128-byte-swizzled layout of tiled stores
          // of 32 x 64 boxes; one thread stores them and does not wait: a
          // global store, or a wait for one, in these warps would queue
          // behind this SM's tile copies.  The staging buffer is reused once
          // the previous pair's stores have read it.
          if (seg >= 1 && !wait_all(&sh.stfree, (seg - 1) & 1, sh, p, lane)) break;
          if (row_ok) {
#pragma unroll
            for (int cc = 0; cc < HD / 16; ++cc) {
#pragma unroll
              for (int j = 0; j < 16; j += 4) {
                const int col = HD * half + 16 * cc + j;
                const int bx = col >> 5, ch = (col & 31) >> 2;
                *reinterpret_cast<float4 *>(stg + bx * (M * 128) + r * 128 + ((ch ^ (r & 7)) << 4)) =
                    make_float4(__uint_as_float(o[cc][j]) * inv, __uint_as_float(o[cc][j + 1]) * inv,
                                __uint_as_float(o[cc][j + 2]) * inv,
                                __uint_as_float(o[cc][j + 3]) * inv);
              }
            }
            if (half == 0) sh.mlst[r] = make_float2(m_used, seg_bad ? -1.f : l_row);
          }
          if (warp == 2 && lane == 0) {
            sh.st_row = d.row;
            sh.st_direct = direct ? 1 : 0;
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&sh.staged);
        } else if (row_ok) {
          const int64_t row = (int64_t)d.row + r;
          float *dst = (direct ? p.seq_o : p.part_o) + row * D + HD * half;
#pragma unroll
          for (int cc = 0; cc < HD / 16; ++cc) {
#pragma unroll
            for (int j = 0; j < 16; j += 4)
              *reinterpret_cast<float4 *>(dst + 16 * cc + j) = make_float4(
                  __uint_as_float(o[cc][j]) * inv, __uint_as_float(o[cc][j + 1]) * inv,
                  __uint_as_float(o[cc][j + 2]) * inv, __uint_as_float(o[cc][j + 3]) * inv);
          }
          if (half == 0)
            reinterpret_cast<float2 *>(direct ? p.seq_ml : p.part_ml)[row] =
                make_float2(m_used, seg_bad ? -1.f : l_row);
        }
      }
    }
    if constexpr (M == 64) {
      // no more pairs: once the last one has left the staging buffer, tell
      // the store warp (a row of -1)
      if (seg >= 0) wait_all(&sh.stfree, seg & 1, sh, p, lane);
      if (warp == 2 && lane == 0) sh.st_row = -1;
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh.staged);
    }
  } else if (warp == 10 && M == 64 && n_units > 0) {
    // ===================== output stores (group 64) =====================
    // Tiled stores of each staged pair: issuing them waits while this SM's
    // copy engine is busy with tile loads, so they get a warp of their own.
    for (int g = 0;; ++g) {
      if (!wait_all(&sh.staged, g & 1, sh, p, lane)) break;
      const int32_t row = sh.st_row;
      if (row < 0) break;
      if (lane == 0) {
        const CUtensorMap *map = sh.st_direct ? &p.tmap_seq_o : &p.tmap_part_o;
        for (int bx = 0; bx < D / 32; ++bx) tma_store_2d(map, bx * 32, row, stg + bx * (M * 128));
        bulk_s2g((sh.st_direct ? p.seq_ml : p.part_ml) + (int64_t)row * 2, sh.mlst,
                 (uint32_t)(M * 8));
        bulk_commit();
        bulk_wait_read();
        mbar_arrive(&sh.stfree);  // the softmax warps may stage the next pair
      }
      __syncwarp();
    }
    // the stores are complete before the CTA ends
    if (lane == 0) bulk_wait_all();
    __syncwarp();
  }

  // ---- Sequences with no suffix tile: an empty record for each pair (and
  // a flag, and zeroed output through `bad`, for a length outside the table).
  for (int s = c; s < p.batch; s += gridDim.x) {
    if (suffix_len(p, s) > 0) continue;
    const int32_t ctx = p.context_lens[s];
    const bool bad_len = ctx < 0 || (int64_t)ctx > (int64_t)p.table_stride * bs;
    for (int x = tid; x < p.num_kv_heads; x += kThreads)
      reinterpret_cast<int4 *>(p.merge)[(int64_t)s * p.num_kv_heads + x] =
          make_int4(0, 0, 0, bad_len ? 1 : 0);
    if (tid == 0 && bad_len) set_error(p.err_word, PA_DEVERR_CONTEXT_LEN);
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

// ---------------------------------------------------------------------------
// pa_decode on this path (no prefix): each (sequence, KV head) pair's G rows
// from its one result or from the partials of the CTAs that cut it (the
// running-max merge), as bf16; zeros for an empty pair, a bad page, a bad
// new-token slot or a length outside the table.  One block per pair.
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(128) finish_kernel(const __grid_constant__ SuffixParams p,
                                                     __nv_bfloat16 *out) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int pair = blockIdx.x;
  const int s = pair / p.num_kv_heads, h = pair - s * p.num_kv_heads;
  const int4 md = __ldcg(reinterpret_cast<const int4 *>(p.merge) + pair);
  const int n = md.w != 0 ? 0 : md.y;
  const float2 *mls = reinterpret_cast<const float2 *>(n == 1 ? p.seq_ml : p.part_ml);
  const float *obase = n == 1 ? p.seq_o : p.part_o;
  for (int f = threadIdx.x * 4; f < p.group * D; f += blockDim.x * 4) {
    const int hh = f / D, d0 = f - hh * D;
    const int64_t row = (int64_t)s * p.num_q_heads + (int64_t)h * p.group + hh;
    auto crow = [&](int x) -> int64_t {
      return n == 1 ? row
                    : ((int64_t)(md.x + x) * 2 + (x == 0 ? md.z : 0)) * p.num_q_heads +
                          (int64_t)h * p.group + hh;
    };
    float M = -INFINITY;
    bool bad = false;
    for (int x = 0; x < n; ++x) {
      const float2 ml = __ldcg(mls + crow(x));
      bad |= ml.y < 0.f;
      if (ml.y > 0.f) M = fmaxf(M, ml.x);
    }
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float W = 0.f;
    if (!bad) {
      for (int x = 0; x < n; ++x) {
        const int64_t cr = crow(x);
        const float2 ml = __ldcg(mls + cr);
        if (!(ml.y > 0.f)) continue;
        const float w = ml.y * ex2(ml.x - M);
        const float4 o = __ldcg(reinterpret_cast<const float4 *>(obase + cr * D + d0));
        W += w;
        acc.x += w * o.x;
        acc.y += w * o.y;
        acc.z += w * o.z;
        acc.w += w * o.w;
      }
    }
    const float inv = W > 0.f ? 1.f / W : 0.f;
    Elem<__nv_bfloat16>::store4(out, row * D + d0,
                                make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv));
  }
}

template <int D, int M>
size_t smem_bytes() {
  using C = Cfg<D, M>;
  const size_t need = sizeof(Shared) + 1024 +
                      (size_t)C::NH * (kQStages * C::kQBox + (C::KS + kVStages) * kTileBox) +
                      C::kStage;
  return need < kMinSmem ? kMinSmem : need;
}

template <int D, int M>
cudaError_t launch_dm(const SuffixParams &p, cudaStream_t stream) {
  auto kern = suffix_attention_kernel<D, M>;
  const size_t smem = smem_bytes<D, M>();
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
  cfg.gridDim = dim3((unsigned)p.grid);
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

}  // namespace suffix

size_t suffix_smem_bytes(int head_dim, int group) {
  if (head_dim == 64) return group == 64 ? suffix::smem_bytes<64, 64>() : suffix::smem_bytes<64, 128>();
  return group == 64 ? suffix::smem_bytes<128, 64>() : suffix::smem_bytes<128, 128>();
}

cudaError_t launch_finish(const SuffixParams &p, void *out, int head_dim, cudaStream_t stream) {
  const int64_t blocks = (int64_t)p.batch * p.num_kv_heads;
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
  __nv_bfloat16 *o = static_cast<__nv_bfloat16 *>(out);
  if (head_dim == 64) return cudaLaunchKernelEx(&cfg, suffix::finish_kernel<64>, p, o);
  if (head_dim == 128) return cudaLaunchKernelEx(&cfg, suffix::finish_kernel<128>, p, o);
  return cudaErrorInvalidValue;
}

cudaError_t launch_suffix(const SuffixParams &p, int head_dim, cudaStream_t stream) {
  if (p.grid <= 0 || p.group != p.num_q_heads / p.num_kv_heads) return cudaErrorInvalidValue;
  if (p.block_size < 8 || p.block_size > suffix::kTok || suffix::kTok % p.block_size != 0)
    return cudaErrorInvalidValue;
  if (head_dim == 64 && p.group == 64) return suffix::launch_dm<64, 64>(p, stream);
  if (head_dim == 64 && p.group == 128) return suffix::launch_dm<64, 128>(p, stream);
  if (head_dim == 128 && p.group == 64) return suffix::launch_dm<128, 64>(p, stream);
  if (head_dim == 128 && p.group == 128) return suffix::launch_dm<128, 128>(p, stream);
  return cudaErrorInvalidValue;
}

}  // namespace pa
