// Paged-decode kernels for __half storage, head_dim 64.
#include "paged_decode_impl.cuh"

namespace pa {

cudaError_t launch_cascade_decode_f16_d64(const DecodeArgs& pre, const DecodeArgs& own,
                                          int g_own, cudaStream_t stream) {
  return launch_cascade_typed<__half, 64>(pre, own, g_own, PA_F16, stream);
}

cudaError_t launch_decode_f16_d64(const DecodeArgs& a, int group, cudaStream_t stream) {
  return launch_decode_typed<__half, 64>(a, group, PA_F16, stream);
}

}  // namespace pa
