// Paged-decode kernels for __nv_bfloat16 queries over E4M3 caches, head_dim 64.
#include "paged_decode_impl.cuh"

namespace pa {

cudaError_t launch_cascade_decode_bf16_d64_e4m3(const DecodeArgs& pre, const DecodeArgs& own,
                                                int g_own, cudaStream_t stream) {
  return launch_cascade_typed<__nv_bfloat16, 64, E4M3>(pre, own, g_own, PA_BF16, stream);
}

cudaError_t launch_decode_bf16_d64_e4m3(const DecodeArgs& a, int group, cudaStream_t stream) {
  return launch_decode_typed<__nv_bfloat16, 64, E4M3>(a, group, PA_BF16, stream);
}

}  // namespace pa
