// fp32 instantiations of the persistent paged decode kernel (CUDA-core
// consumers; one warp per KV head, 4 or 8 KV heads, group 1/2/4/8).
#include "decode_stream.cuh"

namespace pa {
namespace stream {

template <int D, int G>
static cudaError_t launch_hkv(const Params &p, int hkv, size_t smem, cudaStream_t stream) {
  if (hkv == 4) return launch_one<float, D, G, 4>(p, smem, stream);
  if (hkv == 8) return launch_one<float, D, G, 8>(p, smem, stream);
  return cudaErrorInvalidValue;
}

template <int D>
static cudaError_t launch_group(const Params &p, int group, int hkv, size_t smem,
                                cudaStream_t stream) {
  switch (group) {
    case 1: return launch_hkv<D, 1>(p, hkv, smem, stream);
    case 2: return launch_hkv<D, 2>(p, hkv, smem, stream);
    case 4: return launch_hkv<D, 4>(p, hkv, smem, stream);
    case 8: return launch_hkv<D, 8>(p, hkv, smem, stream);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_f32(const Params &p, int head_dim, int group, int hkv, size_t smem,
                       cudaStream_t stream) {
  if (head_dim == 64) return launch_group<64>(p, group, hkv, smem, stream);
  if (head_dim == 128) return launch_group<128>(p, group, hkv, smem, stream);
  return cudaErrorInvalidValue;
}

cudaError_t launch_merge_f32(const Params &p, int head_dim, cudaStream_t stream) {
  if (head_dim == 64) return launch_merge_one<float, 64>(p, stream);
  if (head_dim == 128) return launch_merge_one<float, 128>(p, stream);
  return cudaErrorInvalidValue;
}

}  // namespace stream
}  // namespace pa
