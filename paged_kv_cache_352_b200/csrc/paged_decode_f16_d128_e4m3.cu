// Paged-decode kernels for __half queries over E4M3 caches, head_dim 128.
#include "paged_decode_impl.cuh"

namespace pa {

cudaError_t launch_cascade_decode_f16_d128_e4m3(const DecodeArgs& pre, const DecodeArgs& own,
                                                int g_own, cudaStream_t stream) {
  return launch_cascade_typed<__half, 128, E4M3>(pre, own, g_own, PA_F16, stream);
}

cudaError_t launch_decode_f16_d128_e4m3(const DecodeArgs& a, int group, cudaStream_t stream) {
  return launch_decode_typed<__half, 128, E4M3>(a, group, PA_F16, stream);
}

}  // namespace pa
