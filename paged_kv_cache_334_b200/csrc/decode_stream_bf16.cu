// bf16 instantiations of the persistent paged decode kernel.
#include "decode_stream.cuh"

namespace pa {
namespace stream {
cudaError_t launch_bf16(const Params &p, int head_dim, int group, int hkv, size_t smem,
                        cudaStream_t stream) {
  return launch_stream_dtype<__nv_bfloat16>(p, head_dim, group, hkv, smem, stream);
}
}  // namespace stream
}  // namespace pa
