// api.cu -- the extern "C" entry points of libpa (declared in include/pa.h).
//
// This layer validates arguments on the host, lays out the decode workspace
// and enqueues kernels on the caller's stream.  It never allocates, never
// synchronises and has no CPU fallback: every step of the computation runs in
// the kernels of write_kv.cu, decode_stream.cuh (persistent page-stream decode
// and its merge kernel), decode.cu (partition decode for split-K and the
// shapes the stream kernel does not cover) and reduce.cu.
#include <cudaTypedefs.h>
#include <math.h>
#include <stdio.h>
#include <string.h>

#include "../../include/pa.h"
#include "pa_launch.h"

namespace {

constexpr int32_t kDecodePartitionTokens = 256;
constexpr int32_t kMaxPartitionPages = 1024;  // block-table slice held in smem
constexpr size_t kAlign = 256;

thread_local char g_msg[512] = "";

pa_status fail(pa_status s, const char *fmt, const char *detail = nullptr,
               long long v = 0) {
  snprintf(g_msg, sizeof g_msg, fmt, detail ? detail : "", v);
  return s;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t round_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

bool is_pow2(int32_t x) { return x > 0 && (x & (x - 1)) == 0; }

// Bytes of one cache element, and of one element of q / out / the new rows.
int32_t elem_bytes(int32_t dtype) {
  return dtype == PA_DTYPE_F32 ? 4 : dtype == PA_DTYPE_FP8_E4M3 ? 1 : 2;
}
int32_t act_bytes(int32_t dtype) { return dtype == PA_DTYPE_F32 ? 4 : 2; }

pa_status check_cache(const pa_cache_desc *c) {
  if (c == nullptr) return fail(PA_ERR_INVALID_ARG, "cache descriptor is NULL%s");
  if (c->dtype != PA_DTYPE_F32 && c->dtype != PA_DTYPE_BF16 && c->dtype != PA_DTYPE_FP8_E4M3)
    return fail(PA_ERR_INVALID_ARG, "dtype %s%lld is not F32, BF16 or FP8_E4M3", "", c->dtype);
  if (c->dtype == PA_DTYPE_FP8_E4M3) {
    if (!(c->k_scale > 0.f && c->k_scale <= 3.4e38f && c->v_scale > 0.f && c->v_scale <= 3.4e38f))
      return fail(PA_ERR_INVALID_ARG, "FP8 pages need finite scales > 0%s");
    if (c->head_dim != 128)
      return fail(PA_ERR_UNSUPPORTED, "FP8 pages need head_dim 128%s (got %lld)", "", c->head_dim);
  }
  if (c->num_blocks <= 0)
    return fail(PA_ERR_INVALID_ARG, "num_blocks must be > 0%s (got %lld)", "", c->num_blocks);
  if (c->num_kv_heads <= 0)
    return fail(PA_ERR_INVALID_ARG, "num_kv_heads must be > 0%s (got %lld)", "", c->num_kv_heads);
  if (!is_pow2(c->block_size) || c->block_size > 256)
    return fail(PA_ERR_UNSUPPORTED, "block_size must be a power of two in [1, 256]%s (got %lld)",
                "", c->block_size);
  if (c->head_dim != 64 && c->head_dim != 128)
    return fail(PA_ERR_UNSUPPORTED, "head_dim must be 64 or 128%s (got %lld)", "", c->head_dim);
  return PA_OK;
}

pa_status check_ptr(const void *p, const char *name) {
  if (p == nullptr) return fail(PA_ERR_INVALID_ARG, "%s is NULL", name);
  if (!aligned16(p)) return fail(PA_ERR_INVALID_ARG, "%s is not 16-byte aligned", name);
  return PA_OK;
}

// Checks shared by pa_decode and pa_decode_splitk.
pa_status check_decode_common(const pa_cache_desc *cache, const void *q,
                              const void *key_cache, const void *value_cache,
                              const int32_t *block_tables,
                              const int32_t *context_lens, int32_t batch,
                              int32_t num_q_heads, int32_t max_blocks,
                              float scale) {
  pa_status s = check_cache(cache);
  if (s != PA_OK) return s;
  if (batch < 0 || batch > 65535)
    return fail(PA_ERR_INVALID_ARG, "batch must be in [0, 65535]%s (got %lld)", "", batch);
  if (num_q_heads <= 0 || num_q_heads % cache->num_kv_heads != 0)
    return fail(PA_ERR_INVALID_ARG,
                "num_q_heads must be a positive multiple of num_kv_heads%s (got %lld)", "",
                num_q_heads);
  const int32_t group = num_q_heads / cache->num_kv_heads;
  if (group > 512)
    return fail(PA_ERR_UNSUPPORTED, "more than 512 query heads per KV head%s (%lld)", "", group);
  const int32_t gt = pa::decode_head_tile(group);
  if ((int64_t)cache->num_kv_heads * ((group + gt - 1) / gt) > 65535)
    return fail(PA_ERR_UNSUPPORTED, "too many KV heads x head tiles%s (%lld)", "",
                (long long)cache->num_kv_heads * ((group + gt - 1) / gt));
  if (max_blocks < 0 || (int64_t)max_blocks * cache->block_size > 0x7fffffffLL)
    return fail(PA_ERR_INVALID_ARG, "max_blocks_per_seq * block_size must fit int32%s (%lld)", "",
                max_blocks);
  if (!isfinite(scale)) return fail(PA_ERR_INVALID_ARG, "scale is not finite%s");
  if (batch == 0) return PA_OK;
  if ((s = check_ptr(q, "q")) != PA_OK) return s;
  if ((s = check_ptr(key_cache, "key_cache")) != PA_OK) return s;
  if ((s = check_ptr(value_cache, "value_cache")) != PA_OK) return s;
  if (context_lens == nullptr) return fail(PA_ERR_INVALID_ARG, "context_lens is NULL%s");
  if (max_blocks > 0 && block_tables == nullptr)
    return fail(PA_ERR_INVALID_ARG, "block_tables is NULL%s");
  return PA_OK;
}

// Shape plan of the persistent decode kernel; ok == false means the shape is
// served by the partition kernel of decode.cu instead.
struct StreamPlan {
  bool ok;
  bool tile;  // bf16 pages of >= 16 tokens: tensor copies of swizzled boxes
  int32_t vbs, log2_vbs, log2_vpp, row_bytes, row_pitch, vpage_stride, q_bytes, pps, stages,
      stage_bytes, box_bytes, n_dhalf;
  int32_t heads_per_warp, warps_per_kv;
  bool fp8;               // E4M3 pages: fp16 fragments built from the codes
  bool pair;              // 8-token blocks, two per 16-token page (tile path)
  size_t smem;
};

int32_t ilog2(int32_t x) {
  int32_t l = 0;
  while ((1 << l) < x) ++l;
  return l;
}

StreamPlan plan_stream(const pa_cache_desc *c, int32_t num_q_heads, bool allow_tile = true) {
  namespace st = pa::stream;
  StreamPlan s{};
  s.ok = false;
  const int32_t hkv = c->num_kv_heads;
  const int32_t group = num_q_heads / hkv;
  // fp8 pages take the token-row tensor-core consumers (fp16 fragments)
  const bool fp8 = c->dtype == PA_DTYPE_FP8_E4M3;
  const bool bf16 = c->dtype == PA_DTYPE_BF16 || fp8;
  s.fp8 = fp8;
  if (bf16) {
    // tensor-core consumers: one warp per (KV head, 16 query heads) when the
    // group is a multiple of 16, else per (KV head, up to 8 query heads)
    auto ncw_ok = [&](int32_t per_kv) {
      const int32_t ncw = hkv * per_kv;
      return ncw == 4 || ncw == 8 || ncw == 16;
    };
    if (group % 16 == 0 && ncw_ok(group / 16)) {
      s.heads_per_warp = 16;
      s.warps_per_kv = group / 16;
    } else {
      if (group > 8 && group % 8 != 0) return s;
      s.heads_per_warp = group < 8 ? group : 8;
      s.warps_per_kv = group > 8 ? group / 8 : 1;
      if (!ncw_ok(s.warps_per_kv)) return s;
    }
  } else {
    // CUDA-core consumers: one warp per KV head
    if (hkv != 4 && hkv != 8) return s;
    if (group != 1 && group != 2 && group != 4 && group != 8) return s;
    s.heads_per_warp = group;
    s.warps_per_kv = 1;
  }
  const int32_t elt = elem_bytes(c->dtype);
  s.row_bytes = hkv * c->head_dim * elt;
  if (s.row_bytes + 16 > st::kVPageBytes) return s;
  int32_t rows = st::kVPageBytes / s.row_bytes;  // power of two
  if (fp8) {
    // 32-token virtual pages (two MMA tiles), one warp per KV head
    if (c->block_size < 16 || (hkv != 4 && hkv != 8) || s.warps_per_kv != 1 ||
        s.heads_per_warp > 8)
      return s;
    rows = 32;
  }
  s.vbs = c->block_size < rows ? c->block_size : rows;
  // 8-token blocks of bf16, head_dim 128, one warp per KV head: pages of two
  // blocks, so that the tensor-core tiles (16 tokens) and the tiled copies
  // serve them as they serve 16-token blocks
  s.pair = allow_tile && !fp8 && bf16 && c->block_size == 8 && rows >= 16 &&
           c->head_dim == 128 && s.warps_per_kv == 1 && s.heads_per_warp <= 8 &&
           (hkv == 4 || hkv == 8);
  if (s.pair) s.vbs = 16;
  // FP8 pages of 16-token blocks: two blocks per 32-token page
  if (allow_tile && fp8 && c->block_size == 16) {
    s.pair = true;
    s.vbs = 32;
  }
  s.log2_vbs = ilog2(s.vbs);
  s.log2_vpp = s.pair ? 0 : ilog2(c->block_size / s.vbs);
  s.tile = allow_tile && bf16 && s.vbs >= 16 && hkv <= 256;
  s.n_dhalf = c->head_dim / 64;
  s.box_bytes = 128 * s.vbs * hkv;
  if (s.tile) {
    // boxes land back to back: no padding, the swizzle keeps ldmatrix conflict-free
    s.row_pitch = s.row_bytes;
    s.vpage_stride = s.vbs * s.row_bytes;
  } else if (bf16) {
    // row copies at a 16-byte padded pitch; tiles span 16 rows, so slots get >= 16
    s.row_pitch = s.row_bytes + 16;
    s.vpage_stride = (s.vbs < 16 ? 16 : s.vbs) * s.row_pitch;
  } else {
    s.row_pitch = s.row_bytes;
    s.vpage_stride = s.vbs * s.row_bytes;
  }
  s.q_bytes = num_q_heads * c->head_dim * act_bytes(c->dtype);
  s.pps = st::kVPageBytes / s.vpage_stride;
  if (s.pps > st::kMaxPPS) s.pps = st::kMaxPPS;
  if (s.pps < 1) s.pps = 1;
  if (fp8 && !s.tile) return s;
  const int32_t avail = st::kSmemLimit - st::kHdrBytes - 1024;  // 1 KB alignment slack
  for (;;) {
    s.stage_bytes = (int32_t)(((size_t)2 * s.pps * s.vpage_stride + (size_t)s.pps * s.q_bytes +
                               1023) / 1024 * 1024);
    s.stages = avail / s.stage_bytes;
    if (s.stages > st::kMaxStages) s.stages = st::kMaxStages;
    if (s.stages >= 3 || s.pps == 1) break;
    --s.pps;
  }
  if (s.stages < 2) return s;
  s.smem = (size_t)st::kHdrBytes + 1024 + (size_t)s.stages * s.stage_bytes;
  s.ok = true;
  return s;
}

// cuTensorMapEncodeTiled, fetched from the driver once.
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static bool tried = false;
  if (!tried) {
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    tried = true;
  }
  return fn;
}

// 3-D view (head_dim, token row of the pool, KV head) of a cache with boxes
// of 128 bytes x vbs x Hkv and 128-byte swizzle: 64 bf16 elements (one box
// per 64-wide half of head_dim) or 128 E4M3 codes (one box per row).
bool encode_cache_map(CUtensorMap *map, const void *base, const pa_cache_desc *c, int32_t vbs) {
  PFN_cuTensorMapEncodeTiled_v12000 fn = tensor_map_encoder();
  if (fn == nullptr) return false;
  const bool fp8 = c->dtype == PA_DTYPE_FP8_E4M3;
  const cuuint64_t elt = fp8 ? 1 : 2;
  const cuuint64_t dims[3] = {(cuuint64_t)c->head_dim,
                              (cuuint64_t)c->num_blocks * (cuuint64_t)c->block_size,
                              (cuuint64_t)c->num_kv_heads};
  const cuuint64_t strides[2] = {(cuuint64_t)c->num_kv_heads * c->head_dim * elt,
                                 (cuuint64_t)c->head_dim * elt};
  const cuuint32_t box[3] = {(cuuint32_t)(128 / elt), (cuuint32_t)vbs, (cuuint32_t)c->num_kv_heads};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(map, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                        3, const_cast<void *>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int device_sm_count() {
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    cache[dev] = n;
  }
  return cache[dev];
}

struct WorkspaceLayout {
  size_t part_max, part_sum, part_out, counters, total;
  int32_t max_parts;
  bool stream;
  bool tensor;  // the tensor-core path (suffix.cu) with no prefix
};

bool suffix_kernel_serves(const pa_cache_desc *c, int32_t group);
struct SuffixLayout {
  size_t part_ml, part_o, merge, seq_ml, seq_o, total;
};
SuffixLayout suffix_layout(const pa_cache_desc *c, int32_t batch, int32_t num_q_heads);

WorkspaceLayout decode_layout(const pa_cache_desc *c, int32_t batch,
                              int32_t num_q_heads, int32_t max_blocks,
                              bool allow_tensor = true) {
  WorkspaceLayout w{};
  if (allow_tensor && suffix_kernel_serves(c, num_q_heads / c->num_kv_heads)) {
    // groups of 64 or 128 query heads: decode on the tensor cores
    w.tensor = true;
    w.total = suffix_layout(c, batch, num_q_heads).total;
    return w;
  }
  const StreamPlan sp = plan_stream(c, num_q_heads);
  if (sp.ok) {
    // persistent kernel: (max, sum) and output per (CTA, head/tail slot, query
    // head); one merge record (4 x int32) per sequence
    const size_t slots = (size_t)pa::stream::kMaxGrid * 2 * num_q_heads;
    w.stream = true;
    w.max_parts = 0;
    w.part_max = 0;  // (max, sum) pairs
    w.part_sum = 0;
    w.part_out = round_up(slots * 2 * sizeof(float));
    w.counters = round_up(w.part_out + slots * c->head_dim * sizeof(float));
    w.total = round_up(w.counters + (size_t)batch * 4 * sizeof(int32_t));
    return w;
  }
  const int64_t tokens = (int64_t)max_blocks * c->block_size;
  w.max_parts = (int32_t)((tokens + kDecodePartitionTokens - 1) / kDecodePartitionTokens);
  const size_t n = (size_t)batch * num_q_heads * w.max_parts;
  const int32_t group = num_q_heads / c->num_kv_heads;
  const int32_t gt = pa::decode_head_tile(group);
  const size_t ncnt = (size_t)batch * c->num_kv_heads * ((group + gt - 1) / gt);
  w.part_max = 0;
  w.part_sum = round_up(w.part_max + n * sizeof(float));
  w.part_out = round_up(w.part_sum + n * sizeof(float));
  w.counters = round_up(w.part_out + n * c->head_dim * sizeof(float));
  w.total = round_up(w.counters + ncnt * sizeof(int32_t));
  w.stream = false;
  return w;
}

// pa_decode_shared_prefix with the suffix on the tensor cores (suffix.cu):
// the shapes it serves, and its workspace (partials per (CTA, slot, query
// head), one merge record per (sequence, KV head), the per-row results).
bool suffix_kernel_serves(const pa_cache_desc *c, int32_t group) {
  return c->dtype == PA_DTYPE_BF16 && (group == 64 || group == 128) &&
         (c->head_dim == 64 || c->head_dim == 128) && c->block_size >= 8 &&
         c->block_size <= 128;
}

SuffixLayout suffix_layout(const pa_cache_desc *c, int32_t batch, int32_t num_q_heads) {
  SuffixLayout l{};
  const size_t slots = (size_t)pa::stream::kMaxGrid * 2 * num_q_heads;
  const size_t rows = (size_t)batch * num_q_heads;
  l.part_ml = 0;
  l.part_o = round_up(slots * 2 * sizeof(float));
  l.merge = round_up(l.part_o + slots * c->head_dim * sizeof(float));
  l.seq_ml = round_up(l.merge + (size_t)batch * c->num_kv_heads * 4 * sizeof(int32_t));
  l.seq_o = round_up(l.seq_ml + rows * 2 * sizeof(float));
  l.total = round_up(l.seq_o + rows * (size_t)c->head_dim * sizeof(float));
  return l;
}

// Arguments and tensor maps of the suffix kernel: q (boxes of 64 x group x
// 1), the caches (64 x block_size x 1), and the fp32 rows it stores.
pa_status make_suffix_params(const pa_cache_desc *cache, const void *q, const void *key_cache,
                             const void *value_cache, const int32_t *block_tables,
                             const int32_t *context_lens, int32_t batch, int32_t num_q_heads,
                             int32_t max_blocks_per_seq, int32_t prefix_blocks, float scale,
                             char *ws, int32_t *err_word, pa::SuffixParams *sp) {
  PFN_cuTensorMapEncodeTiled_v12000 fn = tensor_map_encoder();
  if (fn == nullptr) return fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable%s");
  const int sms = device_sm_count();
  if (sms <= 0) return fail(PA_ERR_CUDA, "cannot query the device%s");
  const int32_t group = num_q_heads / cache->num_kv_heads;
  const int32_t bs = cache->block_size;
  const SuffixLayout l = suffix_layout(cache, batch, num_q_heads);
  *sp = pa::SuffixParams{};
  {
    const cuuint64_t dims[3] = {(cuuint64_t)cache->head_dim, (cuuint64_t)num_q_heads,
                                (cuuint64_t)batch};
    const cuuint64_t strides[2] = {(cuuint64_t)cache->head_dim * 2,
                                   (cuuint64_t)num_q_heads * cache->head_dim * 2};
    const cuuint32_t box[3] = {64, (cuuint32_t)group, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    if (fn(&sp->tmap_q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(q), dims, strides,
           box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return fail(PA_ERR_CUDA, "cannot describe q for the tensor copies%s");
  }
  {
    const cuuint64_t dims[3] = {(cuuint64_t)cache->head_dim,
                                (cuuint64_t)cache->num_blocks * (cuuint64_t)bs,
                                (cuuint64_t)cache->num_kv_heads};
    const cuuint64_t strides[2] = {(cuuint64_t)cache->num_kv_heads * cache->head_dim * 2,
                                   (cuuint64_t)cache->head_dim * 2};
    const cuuint32_t box[3] = {64, (cuuint32_t)bs, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    for (int which = 0; which < 2; ++which) {
      if (fn(which ? &sp->tmap_v : &sp->tmap_k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
             const_cast<void *>(which ? value_cache : key_cache), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return fail(PA_ERR_CUDA, "cannot describe the caches for the tensor copies%s");
    }
  }
  // fp32 rows of D (seq_o, part_o) for the epilogue's tiled stores
  auto encode_rows = [&](CUtensorMap *map, char *base, size_t rows) -> bool {
    const cuuint64_t dims[2] = {(cuuint64_t)cache->head_dim, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)cache->head_dim * 4};
    const cuuint32_t box[2] = {32, (cuuint32_t)group};
    const cuuint32_t estr[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, base, dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
  };
  if (!encode_rows(&sp->tmap_seq_o, ws + l.seq_o, (size_t)batch * num_q_heads) ||
      !encode_rows(&sp->tmap_part_o, ws + l.part_o,
                   (size_t)pa::stream::kMaxGrid * 2 * num_q_heads))
    return fail(PA_ERR_CUDA, "cannot describe the suffix results for the tensor copies%s");
  sp->block_tables = block_tables;
  sp->context_lens = context_lens;
  sp->seq_ml = reinterpret_cast<float *>(ws + l.seq_ml);
  sp->seq_o = reinterpret_cast<float *>(ws + l.seq_o);
  sp->part_ml = reinterpret_cast<float *>(ws + l.part_ml);
  sp->part_o = reinterpret_cast<float *>(ws + l.part_o);
  sp->merge = reinterpret_cast<int32_t *>(ws + l.merge);
  sp->slot_mapping = nullptr;
  sp->err_word = err_word;
  sp->batch = batch;
  sp->num_q_heads = num_q_heads;
  sp->num_kv_heads = cache->num_kv_heads;
  sp->group = group;
  sp->block_size = bs;
  sp->table_stride = max_blocks_per_seq;
  sp->prefix_blocks = prefix_blocks;
  sp->num_blocks = cache->num_blocks;
  sp->grid = sms < pa::stream::kMaxGrid ? sms : pa::stream::kMaxGrid;
  sp->scale_log2 = scale * 1.4426950408889634f;
  return PA_OK;
}

}  // namespace

namespace pa {
void set_last_error_message(const char *msg) { snprintf(g_msg, sizeof g_msg, "%s", msg); }
}  // namespace pa

// Arguments of the persistent page-stream kernel common to pa_decode (and its
// variants) and pa_decode_splitk: shapes, the tensor maps of the caches (or a
// row-copy plan when they cannot be described), the stage layout and the
// scales.  The caller fills in the outputs and the workspace pointers.
static pa_status stream_params(const pa_cache_desc *cache, const void *q, const void *key_cache,
                               const void *value_cache, const int32_t *block_tables,
                               const int32_t *context_lens, int32_t batch, int32_t num_q_heads,
                               int32_t max_blocks_per_seq, int32_t prefix_blocks, float scale,
                               int32_t *err_word, pa::stream::Params *pp, StreamPlan *plan) {
  const bool fp8 = cache->dtype == PA_DTYPE_FP8_E4M3;
  StreamPlan sp = plan_stream(cache, num_q_heads);
  const int sms = device_sm_count();
  if (sms <= 0) return fail(PA_ERR_CUDA, "cannot query the device%s");
  pa::stream::Params &p = *pp;
  // boxes of a page's rows of all KV heads (two-block pages: of a block's)
  const int32_t box_tok = sp.pair ? cache->block_size : sp.vbs;
  if (sp.tile && !(encode_cache_map(&p.tmap_k, key_cache, cache, box_tok) &&
                   encode_cache_map(&p.tmap_v, value_cache, cache, box_tok))) {
    if (fp8) return fail(PA_ERR_CUDA, "cannot describe the FP8 caches for the tensor copies%s");
    sp = plan_stream(cache, num_q_heads, /*allow_tile=*/false);
  }
  if (!sp.ok) return fail(PA_ERR_UNSUPPORTED, "no page-stream plan for these shapes%s");
  p.q = q;
  p.key_cache = const_cast<void *>(key_cache);
  p.value_cache = const_cast<void *>(value_cache);
  p.block_tables = block_tables + prefix_blocks;
  p.context_lens = context_lens;
  p.err_word = err_word;
  p.num_blocks = cache->num_blocks;
  p.block_size = cache->block_size;
  p.num_kv_heads = cache->num_kv_heads;
  p.num_q_heads = num_q_heads;
  p.max_blocks = max_blocks_per_seq - prefix_blocks;
  p.table_stride = max_blocks_per_seq;
  p.tok_offset = prefix_blocks * cache->block_size;
  p.batch = batch;
  p.vbs = sp.vbs;
  p.log2_vbs = sp.log2_vbs;
  p.log2_vpp = sp.log2_vpp;
  p.log2_bs = ilog2(cache->block_size);
  p.pair = sp.pair ? 1 : 0;
  p.row_bytes = sp.row_bytes;
  p.row_pitch = sp.row_pitch;
  p.vpage_stride = sp.vpage_stride;
  p.q_bytes = sp.q_bytes;
  p.pps = sp.pps;
  p.stages = sp.stages;
  p.stage_bytes = sp.stage_bytes;
  p.hdr_bytes = pa::stream::kHdrBytes;
  p.grid = sms < pa::stream::kMaxGrid ? sms : pa::stream::kMaxGrid;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.fp8 = fp8 ? 1 : 0;
  p.out_scale = 1.f;
  p.k_scale = cache->k_scale;
  p.v_scale = cache->v_scale;
  if (fp8) {
    // the consumers see the code values: k_scale goes into the score scale,
    // v_scale into the output
    p.scale_log2 *= cache->k_scale;
    p.out_scale = cache->v_scale;
  }
  p.group = num_q_heads / cache->num_kv_heads;
  p.heads_per_warp = sp.heads_per_warp;
  p.warps_per_kv = sp.warps_per_kv;
  p.tile = sp.tile ? 1 : 0;
  p.box_bytes = sp.box_bytes;
  p.n_dhalf = sp.n_dhalf;
  *plan = sp;
  return PA_OK;
}

static cudaError_t launch_stream(const pa::stream::Params &p, const pa_cache_desc *cache,
                                 const StreamPlan &sp, cudaStream_t stream) {
  if (cache->dtype == PA_DTYPE_FP8_E4M3)
    return pa::stream::launch_fp8(p, cache->num_kv_heads, sp.smem, stream);
  if (cache->dtype == PA_DTYPE_F32)
    return pa::stream::launch_f32(p, cache->head_dim, p.group, cache->num_kv_heads, sp.smem,
                                  stream);
  return pa::stream::launch_bf16(p, cache->head_dim, p.group, cache->num_kv_heads, sp.smem,
                                 stream);
}

// pa_decode, and pa_forward_decode when k_new / v_new / slot_mapping are set.
// With prefix_blocks > 0 (pa_decode_shared_prefix, persistent kernel only):
// the first prefix_blocks pages of every sequence are left out and each
// (sequence, query head) result goes to seq_ml / seq_o as a partial.
static pa_status decode_impl(const pa_cache_desc *cache, void *out, const void *q, void *key_cache,
                      void *value_cache, const void *k_new, const void *v_new,
                      const int64_t *slot_mapping, const int32_t *block_tables,
                      const int32_t *context_lens, int32_t batch, int32_t num_q_heads,
                      int32_t max_blocks_per_seq, float scale, void *workspace,
                      size_t workspace_bytes, int32_t *err_word, pa_stream_t stream,
                      int32_t prefix_blocks = 0, float *seq_ml = nullptr,
                      float *seq_o = nullptr, bool allow_tensor = true) {
  pa_status s = check_decode_common(cache, q, key_cache, value_cache, block_tables,
                                    context_lens, batch, num_q_heads,
                                    max_blocks_per_seq, scale);
  if (s != PA_OK) return s;
  const bool fused = slot_mapping != nullptr;
  if (fused && batch > 0) {
    if ((s = check_ptr(k_new, "k_new")) != PA_OK) return s;
    if ((s = check_ptr(v_new, "v_new")) != PA_OK) return s;
  }
  if (batch == 0) return PA_OK;
  if ((s = check_ptr(out, "out")) != PA_OK) return s;
  const WorkspaceLayout w = decode_layout(cache, batch, num_q_heads, max_blocks_per_seq,
                                          allow_tensor && prefix_blocks == 0);
  if (workspace_bytes < w.total)
    return fail(PA_ERR_INVALID_ARG, "workspace too small%s: need %lld bytes", "",
                (long long)w.total);
  if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)) != 0)
    return fail(PA_ERR_INVALID_ARG, "workspace must be non-NULL and 256-byte aligned%s");
  char *ws = static_cast<char *>(workspace);
  if (w.tensor) {
    // groups of 64 or 128 query heads per KV head: the tensor-core kernel
    // over 128-token tiles of every (sequence, KV head) pair, then one pass
    // that merges pairs cut between CTAs and writes bf16 out
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (fused) {
      const int64_t row_bytes =
          (int64_t)cache->num_kv_heads * cache->head_dim * elem_bytes(cache->dtype);
      const cudaError_t e = pa::launch_write_kv(cache->dtype, cache->block_size,
                                                cache->num_blocks, row_bytes, key_cache,
                                                value_cache, k_new, v_new, slot_mapping, batch,
                                                err_word, st, block_tables, context_lens,
                                                max_blocks_per_seq, cache->k_scale,
                                                cache->v_scale);
      if (e != cudaSuccess) return fail(PA_ERR_CUDA, "write_kv launch: %s", cudaGetErrorString(e));
    }
    pa::SuffixParams sp;
    s = make_suffix_params(cache, q, key_cache, value_cache, block_tables, context_lens, batch,
                           num_q_heads, max_blocks_per_seq, 0, scale, ws, err_word, &sp);
    if (s != PA_OK) return s;
    sp.slot_mapping = slot_mapping;
    cudaError_t e = pa::launch_suffix(sp, cache->head_dim, st);
    if (e != cudaSuccess) return fail(PA_ERR_CUDA, "decode launch: %s", cudaGetErrorString(e));
    e = pa::launch_finish(sp, out, cache->head_dim, st);
    if (e != cudaSuccess) return fail(PA_ERR_CUDA, "decode launch: %s", cudaGetErrorString(e));
    return PA_OK;
  }
  if (prefix_blocks > 0 && !w.stream)
    return fail(PA_ERR_UNSUPPORTED, "shared-prefix decode needs the persistent kernel's shapes%s");
  const bool fp8 = cache->dtype == PA_DTYPE_FP8_E4M3;
  if (fp8 && (!w.stream || prefix_blocks > 0))
    return fail(PA_ERR_UNSUPPORTED,
                "FP8 pages: head_dim 128, block_size >= 16, 4 or 8 KV heads and at most 8 "
                "query heads per KV head%s");
  if (w.stream) {
    pa::stream::Params p{};
    StreamPlan sp{};
    s = stream_params(cache, q, key_cache, value_cache, block_tables, context_lens, batch,
                      num_q_heads, max_blocks_per_seq, prefix_blocks, scale, err_word, &p, &sp);
    if (s != PA_OK) return s;
    p.out = out;
    p.k_new = k_new;
    p.v_new = v_new;
    p.slot_mapping = slot_mapping;
    p.seq_ml = seq_ml;
    p.seq_o = seq_o;
    p.part_ml = reinterpret_cast<float *>(ws + w.part_max);
    p.part_o = reinterpret_cast<float *>(ws + w.part_out);
    p.seq_merge = reinterpret_cast<int32_t *>(ws + w.counters);
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e = launch_stream(p, cache, sp, st);
    if (e != cudaSuccess) return fail(PA_ERR_CUDA, "decode launch: %s", cudaGetErrorString(e));
    e = cache->dtype == PA_DTYPE_F32 ? pa::stream::launch_merge_f32(p, cache->head_dim, st)
                                     : pa::stream::launch_merge_bf16(p, cache->head_dim, st);
    if (e != cudaSuccess) return fail(PA_ERR_CUDA, "merge launch: %s", cudaGetErrorString(e));
    return PA_OK;
  }
  if (fused) {
    // shapes of the partition kernel: the same checked write, then the decode
    const int64_t row_bytes =
        (int64_t)cache->num_kv_heads * cache->head_dim * elem_bytes(cache->dtype);
    cudaError_t e = pa::launch_write_kv(cache->dtype, cache->block_size, cache->num_blocks,
                                        row_bytes, key_cache, value_cache, k_new, v_new,
                                        slot_mapping, batch, err_word,
                                        static_cast<cudaStream_t>(stream), block_tables,
                                        context_lens, max_blocks_per_seq, cache->k_scale,
                                        cache->v_scale);
    if (e != cudaSuccess) return fail(PA_ERR_CUDA, "write_kv launch: %s", cudaGetErrorString(e));
  }
  pa::DecodeArgs a{};
  a.q = q;
  a.out = out;
  a.key_cache = key_cache;
  a.value_cache = value_cache;
  a.block_tables = block_tables;
  a.context_lens = context_lens;
  a.part_max = reinterpret_cast<float *>(ws + w.part_max);
  a.part_sum = reinterpret_cast<float *>(ws + w.part_sum);
  a.part_out = reinterpret_cast<float *>(ws + w.part_out);
  a.counters = reinterpret_cast<int32_t *>(ws + w.counters);
  a.err_word = err_word;
  a.dtype = cache->dtype;
  a.num_blocks = cache->num_blocks;
  a.block_size = cache->block_size;
  a.num_kv_heads = cache->num_kv_heads;
  a.head_dim = cache->head_dim;
  a.batch = batch;
  a.num_q_heads = num_q_heads;
  a.max_blocks = max_blocks_per_seq;
  a.part_tokens = kDecodePartitionTokens;
  a.max_parts = w.max_parts;
  a.scale = scale;
  a.merge = true;
  a.slot_mapping = slot_mapping;
  cudaError_t e = pa::launch_decode(a, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(PA_ERR_CUDA, "decode launch: %s", cudaGetErrorString(e));
  return PA_OK;
}

namespace pa {
// pa_decode restricted to the page-stream and partition kernels, and its
// workspace size: the tensor-core path's workspace (per-row results and
// per-CTA partials of 64 or 128 query heads) outgrows pa_decode_noalloc's
// fixed scratch.
size_t decode_workspace_bytes_streamed(const pa_cache_desc *cache, int32_t batch,
                                       int32_t num_q_heads, int32_t max_blocks_per_seq) {
  if (check_cache(cache) != PA_OK || batch < 0 || num_q_heads <= 0 ||
      num_q_heads % cache->num_kv_heads != 0 || max_blocks_per_seq < 0)
    return 0;
  return decode_layout(cache, batch, num_q_heads, max_blocks_per_seq, false).total;
}
pa_status decode_streamed(const pa_cache_desc *cache, void *out, const void *q,
                          const void *key_cache, const void *value_cache,
                          const int32_t *block_tables, const int32_t *context_lens,
                          int32_t batch, int32_t num_q_heads, int32_t max_blocks_per_seq,
                          float scale, void *workspace, size_t workspace_bytes,
                          int32_t *err_word, pa_stream_t stream) {
  return decode_impl(cache, out, q, const_cast<void *>(key_cache),
                     const_cast<void *>(value_cache), nullptr, nullptr, nullptr, block_tables,
                     context_lens, batch, num_q_heads, max_blocks_per_seq, scale, workspace,
                     workspace_bytes, err_word, stream, 0, nullptr, nullptr, false);
}
}  // namespace pa

extern "C" {

int32_t pa_version(void) { return 300; }

const char *pa_status_string(int32_t status) {
  switch (status) {
    case PA_OK: return "PA_OK";
    case PA_ERR_INVALID_ARG: return "PA_ERR_INVALID_ARG";
    case PA_ERR_UNSUPPORTED: return "PA_ERR_UNSUPPORTED";
    case PA_ERR_CUDA: return "PA_ERR_CUDA";
    default: return "PA_UNKNOWN_STATUS";
  }
}

const char *pa_last_error_message(void) { return g_msg; }

pa_status pa_write_kv_cache(const pa_cache_desc *cache, void *key_cache,
                            void *value_cache, const void *k_new,
                            const void *v_new, const int64_t *slot_mapping,
                            int32_t num_tokens, int32_t *err_word,
                            pa_stream_t stream) {
  pa_status s = check_cache(cache);
  if (s != PA_OK) return s;
  if (num_tokens < 0)
    return fail(PA_ERR_INVALID_ARG, "num_tokens must be >= 0%s (got %lld)", "", num_tokens);
  if (num_tokens == 0) return PA_OK;
  if ((s = check_ptr(key_cache, "key_cache")) != PA_OK) return s;
  if ((s = check_ptr(value_cache, "value_cache")) != PA_OK) return s;
  if ((s = check_ptr(k_new, "k_new")) != PA_OK) return s;
  if ((s = check_ptr(v_new, "v_new")) != PA_OK) return s;
  if (slot_mapping == nullptr) return fail(PA_ERR_INVALID_ARG, "slot_mapping is NULL%s");
  const int64_t row_bytes =
      (int64_t)cache->num_kv_heads * cache->head_dim * elem_bytes(cache->dtype);
  cudaError_t e = pa::launch_write_kv(cache->dtype, cache->block_size,
                                      cache->num_blocks, row_bytes, key_cache,
                                      value_cache, k_new, v_new, slot_mapping,
                                      num_tokens, err_word,
                                      static_cast<cudaStream_t>(stream), nullptr, nullptr, 0,
                                      cache->k_scale, cache->v_scale);
  if (e != cudaSuccess) return fail(PA_ERR_CUDA, "write_kv launch: %s", cudaGetErrorString(e));
  return PA_OK;
}

size_t pa_decode_workspace_bytes(const pa_cache_desc *cache, int32_t batch,
                                 int32_t num_q_heads, int32_t max_blocks_per_seq) {
  if (check_cache(cache) != PA_OK || batch < 0 || num_q_heads <= 0 ||
      num_q_heads % cache->num_kv_heads != 0 || max_blocks_per_seq < 0)
    return 0;
  return decode_layout(cache, batch, num_q_heads, max_blocks_per_seq).total;
}

pa_status pa_decode(const pa_cache_desc *cache, void *out, const void *q,
                    const void *key_cache, const void *value_cache,
                    const int32_t *block_tables, const int32_t *context_lens,
                    int32_t batch, int32_t num_q_heads,
                    int32_t max_blocks_per_seq, float scale, void *workspace,
                    size_t workspace_bytes, int32_t *err_word,
                    pa_stream_t stream) {
  // the caches are only read when no slot mapping is given
  return decode_impl(cache, out, q, const_cast<void *>(key_cache),
                     const_cast<void *>(value_cache), nullptr, nullptr, nullptr, block_tables,
                     context_lens, batch, num_q_heads, max_blocks_per_seq, scale, workspace,
                     workspace_bytes, err_word, stream);
}


pa_status pa_forward_decode(const pa_cache_desc *cache, void *out, const void *q,
                            void *key_cache, void *value_cache, const void *k_new,
                            const void *v_new, const int64_t *slot_mapping,
                            const int32_t *block_tables, const int32_t *context_lens,
                            int32_t batch, int32_t num_q_heads, int32_t max_blocks_per_seq,
                            float scale, void *workspace, size_t workspace_bytes,
                            int32_t *err_word, pa_stream_t stream) {
  if (slot_mapping == nullptr && batch > 0)
    return fail(PA_ERR_INVALID_ARG, "slot_mapping is NULL%s");
  return decode_impl(cache, out, q, key_cache, value_cache, k_new, v_new, slot_mapping,
                     block_tables, context_lens, batch, num_q_heads, max_blocks_per_seq, scale,
                     workspace, workspace_bytes, err_word, stream);
}

size_t pa_decode_shared_prefix_workspace_bytes(const pa_cache_desc *cache, int32_t batch,
                                               int32_t num_q_heads, int32_t max_blocks_per_seq,
                                               int32_t prefix_blocks) {
  if (check_cache(cache) != PA_OK || batch < 0 || num_q_heads <= 0 ||
      num_q_heads % cache->num_kv_heads != 0 || prefix_blocks < 0 ||
      max_blocks_per_seq < prefix_blocks)
    return 0;
  const WorkspaceLayout w =
      decode_layout(cache, batch, num_q_heads, max_blocks_per_seq, /*allow_tensor=*/false);
  const size_t rows = (size_t)batch * num_q_heads;
  const size_t stream_path = w.total + round_up(rows * 2 * sizeof(float)) +
                             round_up(rows * (size_t)cache->head_dim * sizeof(float));
  const size_t tensor_path = suffix_layout(cache, batch, num_q_heads).total;
  return stream_path > tensor_path ? stream_path : tensor_path;
}

pa_status pa_decode_shared_prefix(const pa_cache_desc *cache, void *out, const void *q,
                                  const void *key_cache, const void *value_cache,
                                  const int32_t *block_tables, const int32_t *context_lens,
                                  int32_t batch, int32_t num_q_heads, int32_t max_blocks_per_seq,
                                  int32_t prefix_blocks, float scale, void *workspace,
                                  size_t workspace_bytes, int32_t *err_word, pa_stream_t stream) {
  pa_status s = check_decode_common(cache, q, key_cache, value_cache, block_tables,
                                    context_lens, batch, num_q_heads, max_blocks_per_seq, scale);
  if (s != PA_OK) return s;
  if (prefix_blocks < 0 || prefix_blocks > max_blocks_per_seq)
    return fail(PA_ERR_INVALID_ARG, "prefix_blocks must be in [0, max_blocks_per_seq]%s (%lld)",
                "", prefix_blocks);
  if (prefix_blocks == 0)
    return pa_decode(cache, out, q, key_cache, value_cache, block_tables, context_lens, batch,
                     num_q_heads, max_blocks_per_seq, scale, workspace, workspace_bytes,
                     err_word, stream);
  const int32_t group = num_q_heads / cache->num_kv_heads;
  const int32_t bs = cache->block_size;
  if (cache->dtype != PA_DTYPE_BF16)
    return fail(PA_ERR_UNSUPPORTED, "shared-prefix decode is bf16 only%s");
  if (group > 128 || 128 % group != 0)
    return fail(PA_ERR_UNSUPPORTED,
                "shared-prefix decode needs 128 %% (query heads per KV head) == 0%s (%lld)", "",
                group);
  if (bs < 8 || bs > 128)
    return fail(PA_ERR_UNSUPPORTED, "shared-prefix decode needs block_size in [8, 128]%s (%lld)",
                "", bs);
  if (prefix_blocks > pa::kMaxPrefixBlocks)
    return fail(PA_ERR_UNSUPPORTED, "more than 2048 shared prefix blocks%s (%lld)", "",
                prefix_blocks);
  if (batch == 0) return PA_OK;
  if ((s = check_ptr(out, "out")) != PA_OK) return s;
  const size_t need = pa_decode_shared_prefix_workspace_bytes(cache, batch, num_q_heads,
                                                              max_blocks_per_seq, prefix_blocks);
  if (workspace_bytes < need)
    return fail(PA_ERR_INVALID_ARG, "workspace too small%s: need %lld bytes", "", (long long)need);
  if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)) != 0)
    return fail(PA_ERR_INVALID_ARG, "workspace must be non-NULL and 256-byte aligned%s");
  char *ws = static_cast<char *>(workspace);
  PFN_cuTensorMapEncodeTiled_v12000 fn = tensor_map_encoder();
  if (fn == nullptr) return fail(PA_ERR_CUDA, "cannot describe tensors for the tensor copies%s");
  // q (head_dim, query head, sequence) with boxes of 64 x rows_h x rows_s
  auto encode_q = [&](CUtensorMap *map, cuuint32_t rows_h, cuuint32_t rows_s) -> bool {
    const cuuint64_t dims[3] = {(cuuint64_t)cache->head_dim, (cuuint64_t)num_q_heads,
                                (cuuint64_t)batch};
    const cuuint64_t strides[2] = {(cuuint64_t)cache->head_dim * 2,
                                   (cuuint64_t)num_q_heads * cache->head_dim * 2};
    const cuuint32_t box[3] = {64, rows_h, rows_s};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(q), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
  };
  pa::PrefixParams pp{};
  if (!encode_q(&pp.tmap_q, (cuuint32_t)group, (cuuint32_t)(128 / group)))
    return fail(PA_ERR_CUDA, "cannot describe q for the tensor copies%s");
  {
    // caches (head_dim, token row of the pool, KV head), boxes of 64 x bs x 1
    const cuuint64_t dims[3] = {(cuuint64_t)cache->head_dim,
                                (cuuint64_t)cache->num_blocks * (cuuint64_t)bs,
                                (cuuint64_t)cache->num_kv_heads};
    const cuuint64_t strides[2] = {(cuuint64_t)cache->num_kv_heads * cache->head_dim * 2,
                                   (cuuint64_t)cache->head_dim * 2};
    const cuuint32_t box[3] = {64, (cuuint32_t)bs, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    for (int which = 0; which < 2; ++which) {
      if (fn(which ? &pp.tmap_v : &pp.tmap_k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
             const_cast<void *>(which ? value_cache : key_cache), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return fail(PA_ERR_CUDA, "cannot describe the caches for the tensor copies%s");
    }
  }
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  const float scale_log2 = scale * 1.4426950408889634f;
  // 1. the suffix of every (sequence, KV head): on the tensor cores for
  //    groups of 64 or 128 query heads, else on the page-stream kernel; one
  //    (max, normaliser, normalised output) per row, or partials of cut pairs
  if (suffix_kernel_serves(cache, group)) {
    pa::SuffixParams sp;
    s = make_suffix_params(cache, q, key_cache, value_cache, block_tables, context_lens, batch,
                           num_q_heads, max_blocks_per_seq, prefix_blocks, scale, ws, err_word,
                           &sp);
    if (s != PA_OK) return s;
    const cudaError_t e = pa::launch_suffix(sp, cache->head_dim, st);
    if (e != cudaSuccess) return fail(PA_ERR_CUDA, "suffix launch: %s", cudaGetErrorString(e));
    pp.seq_ml = sp.seq_ml;
    pp.seq_o = sp.seq_o;
    pp.merge = sp.merge;
    pp.part_ml = sp.part_ml;
    pp.part_o = sp.part_o;
  } else {
    const WorkspaceLayout w =
        decode_layout(cache, batch, num_q_heads, max_blocks_per_seq, /*allow_tensor=*/false);
    const size_t rows = (size_t)batch * num_q_heads;
    float *seq_ml = reinterpret_cast<float *>(ws + w.total);
    float *seq_o = reinterpret_cast<float *>(ws + w.total + round_up(rows * 2 * sizeof(float)));
    s = decode_impl(cache, out, q, const_cast<void *>(key_cache), const_cast<void *>(value_cache),
                    nullptr, nullptr, nullptr, block_tables, context_lens, batch, num_q_heads,
                    max_blocks_per_seq, scale, workspace, w.total, err_word, stream, prefix_blocks,
                    seq_ml, seq_o);
    if (s != PA_OK) return s;
    pp.seq_ml = seq_ml;
    pp.seq_o = seq_o;
    pp.merge = nullptr;
  }
  // 2. the shared prefix on the tensor cores, folded with the suffix
  pp.block_tables = block_tables;
  pp.context_lens = context_lens;
  pp.out = out;
  pp.err_word = err_word;
  pp.batch = batch;
  pp.num_q_heads = num_q_heads;
  pp.num_kv_heads = cache->num_kv_heads;
  pp.group = group;
  pp.block_size = bs;
  pp.table_stride = max_blocks_per_seq;
  pp.prefix_blocks = prefix_blocks;
  pp.num_blocks = cache->num_blocks;
  pp.scale_log2 = scale_log2;
  const cudaError_t e = pa::launch_prefix(pp, cache->head_dim, st);
  if (e != cudaSuccess) return fail(PA_ERR_CUDA, "prefix launch: %s", cudaGetErrorString(e));
  return PA_OK;
}

pa_status pa_prefill(const pa_cache_desc *cache, void *out, const void *q,
                     const void *key_cache, const void *value_cache,
                     const int32_t *block_tables, const int32_t *context_lens,
                     const int32_t *query_start, int32_t batch, int32_t num_tokens,
                     int32_t num_q_heads, int32_t max_blocks_per_seq, int32_t max_query_len,
                     float scale, int32_t *err_word, pa_stream_t stream) {
  pa_status s = check_cache(cache);
  if (s != PA_OK) return s;
  if (batch < 0 || batch > 65535)
    return fail(PA_ERR_INVALID_ARG, "batch must be in [0, 65535]%s (got %lld)", "", batch);
  if (num_tokens < 0)
    return fail(PA_ERR_INVALID_ARG, "num_tokens must be >= 0%s (got %lld)", "", num_tokens);
  if (max_query_len < 0)
    return fail(PA_ERR_INVALID_ARG, "max_query_len must be >= 0%s (got %lld)", "", max_query_len);
  if (num_q_heads <= 0 || num_q_heads % cache->num_kv_heads != 0)
    return fail(PA_ERR_INVALID_ARG,
                "num_q_heads must be a positive multiple of num_kv_heads%s (got %lld)", "",
                num_q_heads);
  if (max_blocks_per_seq < 0 || (int64_t)max_blocks_per_seq * cache->block_size > 0x7fffffffLL)
    return fail(PA_ERR_INVALID_ARG, "max_blocks_per_seq * block_size must fit int32%s (%lld)", "",
                max_blocks_per_seq);
  if (!isfinite(scale)) return fail(PA_ERR_INVALID_ARG, "scale is not finite%s");
  const int32_t group = num_q_heads / cache->num_kv_heads;
  const int32_t bs = cache->block_size;
  if (cache->dtype != PA_DTYPE_BF16) return fail(PA_ERR_UNSUPPORTED, "prefill is bf16 only%s");
  if (group > 128 || 128 % group != 0)
    return fail(PA_ERR_UNSUPPORTED, "prefill needs 128 %% (query heads per KV head) == 0%s (%lld)",
                "", group);
  if (bs < 8 || bs > 128)
    return fail(PA_ERR_UNSUPPORTED, "prefill needs block_size in [8, 128]%s (%lld)", "", bs);
  if (max_blocks_per_seq > pa::kMaxPrefillBlocks)
    return fail(PA_ERR_UNSUPPORTED, "prefill reads at most 4096 table entries per sequence%s (%lld)",
                "", max_blocks_per_seq);
  if (cache->num_kv_heads > 65535)
    return fail(PA_ERR_UNSUPPORTED, "more than 65535 KV heads%s (%lld)", "", cache->num_kv_heads);
  const int64_t tiles = ((int64_t)max_query_len * group + 127) / 128;
  if (tiles > 0x7fffffffLL)
    return fail(PA_ERR_INVALID_ARG, "max_query_len too large%s (%lld)", "", max_query_len);
  if (batch == 0 || num_tokens == 0 || max_query_len == 0) return PA_OK;
  if ((s = check_ptr(q, "q")) != PA_OK) return s;
  if ((s = check_ptr(out, "out")) != PA_OK) return s;
  if ((s = check_ptr(key_cache, "key_cache")) != PA_OK) return s;
  if ((s = check_ptr(value_cache, "value_cache")) != PA_OK) return s;
  if (context_lens == nullptr) return fail(PA_ERR_INVALID_ARG, "context_lens is NULL%s");
  if (query_start == nullptr) return fail(PA_ERR_INVALID_ARG, "query_start is NULL%s");
  if (block_tables == nullptr) return fail(PA_ERR_INVALID_ARG, "block_tables is NULL%s");
  PFN_cuTensorMapEncodeTiled_v12000 fn = tensor_map_encoder();
  if (fn == nullptr) return fail(PA_ERR_CUDA, "cannot describe tensors for the tensor copies%s");
  pa::PrefillParams pp{};
  {
    // q (head_dim, query head, token) with boxes of 64 x group x 128 / group
    const cuuint64_t dims[3] = {(cuuint64_t)cache->head_dim, (cuuint64_t)num_q_heads,
                                (cuuint64_t)num_tokens};
    const cuuint64_t strides[2] = {(cuuint64_t)cache->head_dim * 2,
                                   (cuuint64_t)num_q_heads * cache->head_dim * 2};
    const cuuint32_t box[3] = {64, (cuuint32_t)group, (cuuint32_t)(128 / group)};
    const cuuint32_t estr[3] = {1, 1, 1};
    if (fn(&pp.tmap_q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(q), dims, strides,
           box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return fail(PA_ERR_CUDA, "cannot describe q for the tensor copies%s");
  }
  {
    // caches (head_dim, token row of the pool, KV head), boxes of 64 x bs x 1
    const cuuint64_t dims[3] = {(cuuint64_t)cache->head_dim,
                                (cuuint64_t)cache->num_blocks * (cuuint64_t)bs,
                                (cuuint64_t)cache->num_kv_heads};
    const cuuint64_t strides[2] = {(cuuint64_t)cache->num_kv_heads * cache->head_dim * 2,
                                   (cuuint64_t)cache->head_dim * 2};
    const cuuint32_t box[3] = {64, (cuuint32_t)bs, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    for (int which = 0; which < 2; ++which) {
      if (fn(which ? &pp.tmap_v : &pp.tmap_k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
             const_cast<void *>(which ? value_cache : key_cache), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return fail(PA_ERR_CUDA, "cannot describe the caches for the tensor copies%s");
    }
  }
  pp.block_tables = block_tables;
  pp.context_lens = context_lens;
  pp.query_start = query_start;
  pp.out = out;
  pp.err_word = err_word;
  pp.batch = batch;
  pp.num_tokens = num_tokens;
  pp.num_q_heads = num_q_heads;
  pp.num_kv_heads = cache->num_kv_heads;
  pp.group = group;
  pp.block_size = bs;
  pp.table_stride = max_blocks_per_seq;
  pp.num_blocks = cache->num_blocks;
  pp.tiles_per_seq = (int32_t)tiles;
  pp.scale_log2 = scale * 1.4426950408889634f;
  const cudaError_t e = pa::launch_prefill(pp, cache->head_dim, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(PA_ERR_CUDA, "prefill launch: %s", cudaGetErrorString(e));
  return PA_OK;
}

pa_status pa_decode_splitk(const pa_cache_desc *cache, const void *q,
                           const void *key_cache, const void *value_cache,
                           const int32_t *block_tables,
                           const int32_t *context_lens, int32_t batch,
                           int32_t num_q_heads, int32_t max_blocks_per_seq,
                           float scale, int32_t partition_tokens,
                           int32_t max_partitions, float *part_max,
                           float *part_sum, float *part_out, int32_t *err_word,
                           pa_stream_t stream) {
  pa_status s = check_decode_common(cache, q, key_cache, value_cache, block_tables,
                                    context_lens, batch, num_q_heads,
                                    max_blocks_per_seq, scale);
  if (s != PA_OK) return s;
  // the page-stream kernel serves the shape when partitions hold whole
  // virtual pages (two-block pages of 8-token blocks: 16 tokens)
  const StreamPlan spl = plan_stream(cache, num_q_heads);
  const bool streamed = spl.ok && partition_tokens > 0 && partition_tokens % spl.vbs == 0;
  if (cache->dtype == PA_DTYPE_FP8_E4M3 && !streamed)
    return fail(PA_ERR_UNSUPPORTED,
                "FP8 pages: head_dim 128, block_size >= 16, 4 or 8 KV heads and at most 8 "
                "query heads per KV head%s");
  if (partition_tokens <= 0 || partition_tokens % cache->block_size != 0)
    return fail(PA_ERR_INVALID_ARG,
                "partition_tokens must be a positive multiple of block_size%s (got %lld)", "",
                partition_tokens);
  if (!streamed && partition_tokens / cache->block_size > kMaxPartitionPages)
    return fail(PA_ERR_UNSUPPORTED, "more than 1024 blocks per partition%s (%lld)", "",
                partition_tokens / cache->block_size);
  const int64_t need =
      ((int64_t)max_blocks_per_seq * cache->block_size + partition_tokens - 1) / partition_tokens;
  if (max_partitions < need || max_partitions <= 0)
    return fail(PA_ERR_INVALID_ARG,
                "max_partitions must be >= ceil(max_blocks_per_seq*block_size/partition_tokens)%s"
                " = %lld",
                "", need);
  if (batch == 0) return PA_OK;
  if ((s = check_ptr(part_max, "part_max")) != PA_OK) return s;
  if ((s = check_ptr(part_sum, "part_sum")) != PA_OK) return s;
  if ((s = check_ptr(part_out, "part_out")) != PA_OK) return s;
  if (streamed) {
    // the persistent page-stream kernel in split-K mode: CTA ranges end on
    // partition boundaries, so every partition is written by one CTA and
    // no workspace is needed
    pa::stream::Params p{};
    StreamPlan sp{};
    s = stream_params(cache, q, key_cache, value_cache, block_tables, context_lens, batch,
                      num_q_heads, max_blocks_per_seq, 0, scale, err_word, &p, &sp);
    if (s != PA_OK) return s;
    p.sk_max = part_max;
    p.sk_sum = part_sum;
    p.sk_o = part_out;
    p.part_pages = partition_tokens / sp.vbs;
    p.max_parts = max_partitions;
    const cudaError_t e = launch_stream(p, cache, sp, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess)
      return fail(PA_ERR_CUDA, "decode_splitk launch: %s", cudaGetErrorString(e));
    return PA_OK;
  }
  pa::DecodeArgs a{};
  a.q = q;
  a.out = nullptr;
  a.key_cache = key_cache;
  a.value_cache = value_cache;
  a.block_tables = block_tables;
  a.context_lens = context_lens;
  a.part_max = part_max;
  a.part_sum = part_sum;
  a.part_out = part_out;
  a.counters = nullptr;
  a.err_word = err_word;
  a.dtype = cache->dtype;
  a.num_blocks = cache->num_blocks;
  a.block_size = cache->block_size;
  a.num_kv_heads = cache->num_kv_heads;
  a.head_dim = cache->head_dim;
  a.batch = batch;
  a.num_q_heads = num_q_heads;
  a.max_blocks = max_blocks_per_seq;
  a.part_tokens = partition_tokens;
  a.max_parts = max_partitions;
  a.scale = scale;
  a.merge = false;
  cudaError_t e = pa::launch_decode(a, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess)
    return fail(PA_ERR_CUDA, "decode_splitk launch: %s", cudaGetErrorString(e));
  return PA_OK;
}

pa_status pa_reduce(void *out, const float *part_max, const float *part_sum,
                    const float *part_out, const int32_t *context_lens,
                    int32_t batch, int32_t num_q_heads, int32_t head_dim,
                    int32_t partition_tokens, int32_t max_partitions,
                    int32_t out_dtype, int32_t *err_word, pa_stream_t stream) {
  if (out_dtype != PA_DTYPE_F32 && out_dtype != PA_DTYPE_BF16)
    return fail(PA_ERR_INVALID_ARG, "out_dtype %s%lld is neither F32 nor BF16", "", out_dtype);
  if (batch < 0 || num_q_heads <= 0 || head_dim <= 0 || partition_tokens <= 0 ||
      max_partitions <= 0)
    return fail(PA_ERR_INVALID_ARG, "sizes must be positive%s");
  if ((int64_t)batch * num_q_heads > 0x7fffffffLL)
    return fail(PA_ERR_UNSUPPORTED, "batch * num_q_heads too large%s");
  if (head_dim % 4 != 0) return fail(PA_ERR_INVALID_ARG, "head_dim must be a multiple of 4%s");
  // the kernel keeps one weight per partition and head_dim-wide group sums
  // of its threads in shared memory
  if (head_dim > 1024 ||
      (size_t)((max_partitions + 3) & ~3) * 4 +
              (size_t)(pa::kReduceThreads / (head_dim / 4)) * head_dim * 4 >
          (size_t)227 * 1024)
    return fail(PA_ERR_UNSUPPORTED,
                "head_dim above 1024 or more than about 56000 partitions%s");
  if (batch == 0) return PA_OK;
  pa_status s;
  if ((s = check_ptr(out, "out")) != PA_OK) return s;
  if ((s = check_ptr(part_max, "part_max")) != PA_OK) return s;
  if ((s = check_ptr(part_sum, "part_sum")) != PA_OK) return s;
  if ((s = check_ptr(part_out, "part_out")) != PA_OK) return s;
  if (context_lens == nullptr) return fail(PA_ERR_INVALID_ARG, "context_lens is NULL%s");
  cudaError_t e = pa::launch_reduce(out, part_max, part_sum, part_out, context_lens, batch,
                                    num_q_heads, head_dim, partition_tokens, max_partitions,
                                    out_dtype, err_word, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(PA_ERR_CUDA, "reduce launch: %s", cudaGetErrorString(e));
  return PA_OK;
}

}  // extern "C"
