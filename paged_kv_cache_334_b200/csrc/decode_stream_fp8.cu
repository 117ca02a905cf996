// FP8 (E4M3) page instantiations of the persistent paged decode kernel:
// head_dim 128, token-row consumers (up to 8 query heads per warp, one warp
// per KV head), NCW = KV heads (4 or 8); 32-token pages, made of two blocks
// when blocks hold 16 tokens.
#include "decode_stream.cuh"

namespace pa {
namespace stream {

cudaError_t launch_fp8(const Params &p, int hkv, size_t smem, cudaStream_t stream) {
  if (p.heads_per_warp > 8 || p.warps_per_kv != 1) return cudaErrorInvalidValue;
  if (p.pair) {
    // 16-token blocks, two per 32-token page
    switch (hkv) {
      case 4: return launch_one<Fp8E4M3, 128, 0, 4, true>(p, smem, stream);
      case 8: return launch_one<Fp8E4M3, 128, 0, 8, true>(p, smem, stream);
      default: return cudaErrorInvalidValue;
    }
  }
  switch (hkv) {
    case 4: return launch_one<Fp8E4M3, 128, 0, 4>(p, smem, stream);
    case 8: return launch_one<Fp8E4M3, 128, 0, 8>(p, smem, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace stream
}  // namespace pa
