// fp32 instantiations of the persistent paged decode kernel.
#include "decode_stream.cuh"

namespace pa {
namespace stream {
cudaError_t launch_f32(const Params &p, int head_dim, int group, int hkv, size_t smem,
                        cudaStream_t stream) {
  return launch_stream_dtype<float>(p, head_dim, group, hkv, smem, stream);
}
}  // namespace stream
}  // namespace pa
