// Paged decode attention (sm_100a): one launch computes
//   out[s][h] = softmax(scale * K_s q[s][h]) V_s
// with K_s / V_s read block by block through the sequence's block table
// ("vLLM: PagedAttention and continuous batching", direct answer;
// "PagedAttention: The vLLM Paper", "The Core Idea", block-table figure note).
//
// Work decomposition
//   grid = (num_kv_heads, max_parts, num_seqs): one CTA per (sequence, KV head,
//   split-KV partition of part_blocks blocks). The CTA serves all G query heads
//   that read its KV head, so every K/V byte is fetched from HBM once. CTAs of
//   uneven length are balanced by the hardware scheduler; a CTA's pipeline ramp
//   and merge overlap with the other CTAs resident on its SM.
//
// Data movement
//   A (block, KV head) tile is 16 tokens x head_dim contiguous elements. Each
//   warp owns a ring of STAGES shared-memory stages; lane 0 fills a stage with
//   the block's K and V tiles by async bulk copies (1-D for the CUDA-core path,
//   2-D swizzled tensor copies for the tensor-core path) that complete on the
//   stage's mbarrier. Warp w takes blocks w, w + WARPS, ... of the partition,
//   so a CTA keeps WARPS x STAGES tiles in flight with no cross-warp
//   synchronisation in its main loop.
//
// Merging
//   Each warp leaves its softmax state in shared memory, the CTA merges the
//   warps, and finish_partition writes `out` (single partition) or the
//   partition's state, the last partition of a (sequence, KV head) merging them
//   all in logical order. Results depend only on logical token positions: not on
//   physical placement, sharing or timing.
//
// E4M3 caches (8-bit codes with a key and a value scale) run the same kernel:
// the key scale folds into the softmax scale, the value scale multiplies the
// normalised output, and tiles are widened from codes on the chip.
//
// The kernel template lives in paged_decode_impl.cuh and is instantiated once
// per (storage type, head_dim) in paged_decode_<type>_d<dim>.cu and once per
// (query type, head_dim) over E4M3 caches in paged_decode_<type>_d<dim>_e4m3.cu.
#include <cuda_runtime.h>

#include <atomic>
#include <cstdlib>

#include "pa_internal.h"

namespace pa {

cudaError_t launch_decode_f16_d64(const DecodeArgs& a, int group, cudaStream_t stream);
cudaError_t launch_decode_f16_d128(const DecodeArgs& a, int group, cudaStream_t stream);
cudaError_t launch_decode_bf16_d64(const DecodeArgs& a, int group, cudaStream_t stream);
cudaError_t launch_decode_bf16_d128(const DecodeArgs& a, int group, cudaStream_t stream);
cudaError_t launch_decode_f16_d64_e4m3(const DecodeArgs& a, int group, cudaStream_t stream);
cudaError_t launch_decode_f16_d128_e4m3(const DecodeArgs& a, int group, cudaStream_t stream);
cudaError_t launch_decode_bf16_d64_e4m3(const DecodeArgs& a, int group, cudaStream_t stream);
cudaError_t launch_decode_bf16_d128_e4m3(const DecodeArgs& a, int group, cudaStream_t stream);
cudaError_t launch_cascade_decode_f16_d64(const DecodeArgs& pre, const DecodeArgs& own,
                                          int g_own, cudaStream_t stream);
cudaError_t launch_cascade_decode_f16_d128(const DecodeArgs& pre, const DecodeArgs& own,
                                           int g_own, cudaStream_t stream);
cudaError_t launch_cascade_decode_bf16_d64(const DecodeArgs& pre, const DecodeArgs& own,
                                           int g_own, cudaStream_t stream);
cudaError_t launch_cascade_decode_bf16_d128(const DecodeArgs& pre, const DecodeArgs& own,
                                            int g_own, cudaStream_t stream);
cudaError_t launch_cascade_decode_f16_d64_e4m3(const DecodeArgs& pre, const DecodeArgs& own,
                                               int g_own, cudaStream_t stream);
cudaError_t launch_cascade_decode_f16_d128_e4m3(const DecodeArgs& pre, const DecodeArgs& own,
                                                int g_own, cudaStream_t stream);
cudaError_t launch_cascade_decode_bf16_d64_e4m3(const DecodeArgs& pre, const DecodeArgs& own,
                                                int g_own, cudaStream_t stream);
cudaError_t launch_cascade_decode_bf16_d128_e4m3(const DecodeArgs& pre, const DecodeArgs& own,
                                                 int g_own, cudaStream_t stream);

namespace {
std::atomic<unsigned long long> g_stall_request{0};
}  // namespace

unsigned long long take_stall_request() {
  if (g_stall_request.load(std::memory_order_relaxed) == 0) return 0;
  return g_stall_request.exchange(0);
}

void set_stall_request(unsigned long long wait_limit_ns) { g_stall_request.store(wait_limit_ns); }

cudaError_t launch_paged_decode(const DecodeArgs& args, int head_dim, int group, int dtype,
                                int cache_dtype, cudaStream_t stream) {
  DecodeArgs a = args;
  if (const unsigned long long ns = take_stall_request()) {
    a.stall_first_block = 1;
    a.wait_limit_ns = ns;
  }
  const bool fp8 = cache_dtype == PA_FP8_E4M3;
  if (!fp8 && cache_dtype != dtype) return cudaErrorInvalidValue;
  if (dtype == PA_F16) {
    if (head_dim == 64) return fp8 ? launch_decode_f16_d64_e4m3(a, group, stream)
                                   : launch_decode_f16_d64(a, group, stream);
    if (head_dim == 128) return fp8 ? launch_decode_f16_d128_e4m3(a, group, stream)
                                    : launch_decode_f16_d128(a, group, stream);
  } else {
    if (head_dim == 64) return fp8 ? launch_decode_bf16_d64_e4m3(a, group, stream)
                                   : launch_decode_bf16_d64(a, group, stream);
    if (head_dim == 128) return fp8 ? launch_decode_bf16_d128_e4m3(a, group, stream)
                                    : launch_decode_bf16_d128(a, group, stream);
  }
  return cudaErrorInvalidValue;
}

// Whether launch_cascade_decode has a form for this shape: 8 stacked heads per
// KV head over 1, 2 or 4 own query heads per KV head, a supported head_dim and
// query type, a cache of the query type or of E4M3 codes, and no
// PA_DECODE_PATH override (which forces one policy for every decode).
bool cascade_single_launch(int head_dim, int g_own, int stacked, int dtype, int cache_dtype) {
  if (getenv("PA_DECODE_PATH")) return false;
  if (stacked != 8 || (g_own != 1 && g_own != 2 && g_own != 4)) return false;
  if (head_dim != 64 && head_dim != 128) return false;
  if (dtype != PA_F16 && dtype != PA_BF16) return false;
  return cache_dtype == dtype || cache_dtype == PA_FP8_E4M3;
}

cudaError_t launch_cascade_decode(const DecodeArgs& pre_args, const DecodeArgs& own_args,
                                  int head_dim, int g_own, int dtype, int cache_dtype,
                                  cudaStream_t stream) {
  const bool fp8 = cache_dtype == PA_FP8_E4M3;
  if (!fp8 && cache_dtype != dtype) return cudaErrorNotSupported;
  DecodeArgs pre = pre_args, own = own_args;
  if (const unsigned long long ns = take_stall_request()) {
    pre.stall_first_block = own.stall_first_block = 1;
    pre.wait_limit_ns = own.wait_limit_ns = ns;
  }
  if (dtype == PA_F16) {
    if (head_dim == 64)
      return fp8 ? launch_cascade_decode_f16_d64_e4m3(pre, own, g_own, stream)
                 : launch_cascade_decode_f16_d64(pre, own, g_own, stream);
    if (head_dim == 128)
      return fp8 ? launch_cascade_decode_f16_d128_e4m3(pre, own, g_own, stream)
                 : launch_cascade_decode_f16_d128(pre, own, g_own, stream);
  } else {
    if (head_dim == 64)
      return fp8 ? launch_cascade_decode_bf16_d64_e4m3(pre, own, g_own, stream)
                 : launch_cascade_decode_bf16_d64(pre, own, g_own, stream);
    if (head_dim == 128)
      return fp8 ? launch_cascade_decode_bf16_d128_e4m3(pre, own, g_own, stream)
                 : launch_cascade_decode_bf16_d128(pre, own, g_own, stream);
  }
  return cudaErrorNotSupported;
}

}  // namespace pa
