// Paged-decode kernels for __half storage, head_dim 128.
#include "paged_decode_impl.cuh"

namespace pa {

cudaError_t launch_cascade_decode_f16_d128(const DecodeArgs& pre, const DecodeArgs& own,
                                           int g_own, cudaStream_t stream) {
  return launch_cascade_typed<__half, 128>(pre, own, g_own, PA_F16, stream);
}

cudaError_t launch_decode_f16_d128(const DecodeArgs& a, int group, cudaStream_t stream) {
  return launch_decode_typed<__half, 128>(a, group, PA_F16, stream);
}

}  // namespace pa
