// bf16 instantiations of the persistent paged decode kernel (tensor-core
// consumers): groups that are a multiple of 16 query heads use the head-row
// consumer (16 heads per warp), others the token-row consumer (up to 8 heads
// per warp); NCW = KV heads x warps per KV head, 4, 8 or 16.
#include "decode_stream.cuh"

namespace pa {
namespace stream {

template <int D, int CONS>
static cudaError_t launch_ncw(const Params &p, int ncw, size_t smem, cudaStream_t stream) {
  switch (ncw) {
    case 4: return launch_one<__nv_bfloat16, D, CONS, 4>(p, smem, stream);
    case 8: return launch_one<__nv_bfloat16, D, CONS, 8>(p, smem, stream);
    case 16: return launch_one<__nv_bfloat16, D, CONS, 16>(p, smem, stream);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_bf16(const Params &p, int head_dim, int group, int hkv, size_t smem,
                        cudaStream_t stream) {
  (void)group;
  const int ncw = hkv * p.warps_per_kv;
  const bool rows = p.heads_per_warp == 16;
  if (p.pair) {
    // 8-token blocks, two per page: head_dim 128, one warp per KV head, 4
    // or 8 KV heads
    if (head_dim != 128 || rows || p.warps_per_kv != 1) return cudaErrorInvalidValue;
    switch (ncw) {
      case 4: return launch_one<__nv_bfloat16, 128, 0, 4, true>(p, smem, stream);
      case 8: return launch_one<__nv_bfloat16, 128, 0, 8, true>(p, smem, stream);
      default: return cudaErrorInvalidValue;
    }
  }
  if (head_dim == 64)
    return rows ? launch_ncw<64, 16>(p, ncw, smem, stream) : launch_ncw<64, 0>(p, ncw, smem, stream);
  if (head_dim == 128)
    return rows ? launch_ncw<128, 16>(p, ncw, smem, stream)
                : launch_ncw<128, 0>(p, ncw, smem, stream);
  return cudaErrorInvalidValue;
}

cudaError_t launch_merge_bf16(const Params &p, int head_dim, cudaStream_t stream) {
  if (head_dim == 64) return launch_merge_one<__nv_bfloat16, 64>(p, stream);
  if (head_dim == 128) return launch_merge_one<__nv_bfloat16, 128>(p, stream);
  return cudaErrorInvalidValue;
}

}  // namespace stream
}  // namespace pa
