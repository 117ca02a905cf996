// bf16 instantiations of the persistent paged decode kernel (tensor-core
// consumers; any group size, NCW = KV heads x ceil(group / 8) warps).
#include "decode_stream.cuh"

namespace pa {
namespace stream {

template <int D>
static cudaError_t launch_ncw(const Params &p, int ncw, size_t smem, cudaStream_t stream) {
  switch (ncw) {
    case 4: return launch_one<__nv_bfloat16, D, 0, 4>(p, smem, stream);
    case 8: return launch_one<__nv_bfloat16, D, 0, 8>(p, smem, stream);
    case 16: return launch_one<__nv_bfloat16, D, 0, 16>(p, smem, stream);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_bf16(const Params &p, int head_dim, int group, int hkv, size_t smem,
                        cudaStream_t stream) {
  const int ncw = hkv * (group > 8 ? group / 8 : 1);
  if (head_dim == 64) return launch_ncw<64>(p, ncw, smem, stream);
  if (head_dim == 128) return launch_ncw<128>(p, ncw, smem, stream);
  return cudaErrorInvalidValue;
}

cudaError_t launch_merge_bf16(const Params &p, int head_dim, cudaStream_t stream) {
  if (head_dim == 64) return launch_merge_one<__nv_bfloat16, 64>(p, stream);
  if (head_dim == 128) return launch_merge_one<__nv_bfloat16, 128>(p, stream);
  return cudaErrorInvalidValue;
}

}  // namespace stream
}  // namespace pa
