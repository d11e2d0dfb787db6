// Cache-maintenance kernels (sm_100a): writing new tokens into their slots and
// whole-block copies for copy-on-write. Both are pure byte movement, so they
// move 16-byte vectors with every thread's loads issued before its stores.
//
// reshape_and_cache: every generated token's keys and values are cached
// ("PagedAttention: The vLLM Paper", "Background and Motivation") in the slot
// the block manager assigned as the token arrived ("PagedAttention and
// Continuous Batching", "Pages, from operating systems").
//
// copy_blocks: a shared block is duplicated only when one sharer must write to
// it, as with fork and copy-on-write ("Pages, from operating systems"; "The OS
// paging analogy", page sharing).
//
// reshape_and_cache_fp8: the same write into 8-bit E4M3 caches, quantizing each
// element by the tensor's scale (KV-cache quantization, "PagedAttention: The
// vLLM Paper", "Impact and Follow-Ups" and "Limitations").
//
// swap_blocks: the same copy between two pools, the device pool and a pinned
// host pool, to preempt a request by swapping its blocks to CPU memory ("The OS
// paging analogy", swapping).
#include <cuda_runtime.h>

#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {
namespace {

// One thread per 16-byte chunk of a (token, KV head) row; a row of head_dim
// elements is head_dim/8 chunks and lands as one contiguous run in the cache.
__global__ void __launch_bounds__(256)
    reshape_and_cache_kernel(const uint4* __restrict__ key, const uint4* __restrict__ value,
                             int64_t key_stride_v, int64_t value_stride_v, uint4* k_cache,
                             uint4* v_cache, const int64_t* __restrict__ slot_mapping,
                             int64_t total_chunks, int chunks_per_row, int num_kv_heads,
                             int64_t num_slots, int* dev_error) {
  allow_dependents();  // a following decode may launch; it waits for this kernel
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= total_chunks) return;
  const int64_t per_token = (int64_t)chunks_per_row * num_kv_heads;
  const int64_t t = idx / per_token;
  const int r = (int)(idx - t * per_token);
  const int h = r / chunks_per_row;
  const int c = r - h * chunks_per_row;
  const int64_t slot = __ldg(slot_mapping + t);
  if (slot < 0) return;
  if (slot >= num_slots) {
    if (c == 0 && h == 0) report(dev_error, PA_DEVERR_SLOT_RANGE);
    return;
  }
  const int64_t block = slot / kBlockSize;
  const int64_t offset = slot - block * kBlockSize;
  const uint4 kv = __ldg(key + t * key_stride_v + r);
  const uint4 vv = __ldg(value + t * value_stride_v + r);
  const int64_t dst = ((block * num_kv_heads + h) * kBlockSize + offset) * chunks_per_row + c;
  k_cache[dst] = kv;
  v_cache[dst] = vv;
}

// E4M3 caches: one thread per 16 codes (16 bytes of the cache row) of a
// (token, KV head) row; it reads the matching 16 elements of the 16-bit input,
// divides each by the tensor's scale in fp32 (round to nearest) and stores the
// nearest E4M3 codes, saturating at +-448.
template <typename T>
__global__ void __launch_bounds__(256)
    reshape_and_cache_fp8_kernel(const uint4* __restrict__ key, const uint4* __restrict__ value,
                                 int64_t key_stride_v, int64_t value_stride_v, uint4* k_cache,
                                 uint4* v_cache, const int64_t* __restrict__ slot_mapping,
                                 int64_t total_chunks, int chunks_per_row, int num_kv_heads,
                                 int64_t num_slots, float k_scale, float v_scale,
                                 int* dev_error) {
  allow_dependents();  // a following decode may launch; it waits for this kernel
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= total_chunks) return;
  const int64_t per_token = (int64_t)chunks_per_row * num_kv_heads;
  const int64_t t = idx / per_token;
  const int r = (int)(idx - t * per_token);
  const int h = r / chunks_per_row;
  const int c = r - h * chunks_per_row;
  const int64_t slot = __ldg(slot_mapping + t);
  if (slot < 0) return;
  if (slot >= num_slots) {
    if (c == 0 && h == 0) report(dev_error, PA_DEVERR_SLOT_RANGE);
    return;
  }
  const int64_t block = slot / kBlockSize;
  const int64_t offset = slot - block * kBlockSize;
  const int64_t dst = ((block * num_kv_heads + h) * kBlockSize + offset) * chunks_per_row + c;
  const uint4* srcs[2] = {key + t * key_stride_v + 2 * r, value + t * value_stride_v + 2 * r};
  uint4* caches[2] = {k_cache, v_cache};
  const float scales[2] = {k_scale, v_scale};
#pragma unroll
  for (int kv = 0; kv < 2; ++kv) {
    float f[2][8];  // elements 0-7 and 8-15 of the chunk
    Storage<T>::to_f32(__ldg(srcs[kv]), f[0]);
    Storage<T>::to_f32(__ldg(srcs[kv] + 1), f[1]);
    uint32_t w[4];  // w[i]: codes of elements 4i .. 4i+3, lowest byte first
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float* g = f[i >> 1] + 4 * (i & 1);
      const uint32_t p0 =
          f32x2_to_e4m3x2(__fdiv_rn(g[0], scales[kv]), __fdiv_rn(g[1], scales[kv]));
      const uint32_t p1 =
          f32x2_to_e4m3x2(__fdiv_rn(g[2], scales[kv]), __fdiv_rn(g[3], scales[kv]));
      w[i] = (p0 & 0xffffu) | (p1 << 16);
    }
    caches[kv][dst] = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

constexpr int kCopyThreads = 256;
constexpr int kCopyUnroll = 4;

// grid = (chunks of one pair's K+V bytes, pair). Each thread copies kCopyUnroll
// 16-byte vectors from block src of the source pool to block dst of the
// destination pool; the first half of the index space is the K block, the
// second V. The two pools are the same for copy-on-write copies and differ
// (device <-> pinned host) for swapping; plain loads, since host memory may be
// on either side.
__global__ void __launch_bounds__(kCopyThreads)
    copy_pool_blocks_kernel(const uint4* src_k, const uint4* src_v, uint4* dst_k, uint4* dst_v,
                            const __grid_constant__ CopyPairs pairs, int64_t vecs_per_block) {
  allow_dependents();  // a following decode may launch; it waits for this kernel
  const int pair = blockIdx.y;
  const int64_t src = pairs.src[pair];
  const int64_t dst = pairs.dst[pair];
  const int64_t base = (int64_t)blockIdx.x * kCopyThreads * kCopyUnroll + threadIdx.x;
  uint4 buf[kCopyUnroll];
  bool live[kCopyUnroll];
#pragma unroll
  for (int u = 0; u < kCopyUnroll; ++u) {
    const int64_t i = base + (int64_t)u * kCopyThreads;
    live[u] = i < 2 * vecs_per_block;
    if (live[u]) {
      const bool is_v = i >= vecs_per_block;
      const uint4* pool = is_v ? src_v : src_k;
      const int64_t off = is_v ? i - vecs_per_block : i;
      buf[u] = pool[src * vecs_per_block + off];
    }
  }
#pragma unroll
  for (int u = 0; u < kCopyUnroll; ++u) {
    const int64_t i = base + (int64_t)u * kCopyThreads;
    if (live[u]) {
      const bool is_v = i >= vecs_per_block;
      uint4* pool = is_v ? dst_v : dst_k;
      const int64_t off = is_v ? i - vecs_per_block : i;
      pool[dst * vecs_per_block + off] = buf[u];
    }
  }
}

}  // namespace

cudaError_t launch_reshape_and_cache(const void* key, const void* value, int64_t key_stride,
                                     int64_t value_stride, void* k_cache, void* v_cache,
                                     const int64_t* slot_mapping, int num_tokens,
                                     int num_kv_heads, int head_dim, int num_blocks,
                                     int* dev_error, cudaStream_t stream) {
  const int chunks_per_row = head_dim / 8;
  const int64_t total = (int64_t)num_tokens * num_kv_heads * chunks_per_row;
  if (total == 0) return cudaSuccess;
  const int threads = 256;
  const int64_t blocks = (total + threads - 1) / threads;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
  reshape_and_cache_kernel<<<(unsigned)blocks, threads, 0, stream>>>(
      static_cast<const uint4*>(key), static_cast<const uint4*>(value), key_stride / 8,
      value_stride / 8, static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache), slot_mapping,
      total, chunks_per_row, num_kv_heads, (int64_t)num_blocks * kBlockSize, dev_error);
  return cudaGetLastError();
}

cudaError_t launch_reshape_and_cache_fp8(const void* key, const void* value, int64_t key_stride,
                                         int64_t value_stride, void* k_cache, void* v_cache,
                                         const int64_t* slot_mapping, int num_tokens,
                                         int num_kv_heads, int head_dim, int num_blocks,
                                         int src_dtype, float k_scale, float v_scale,
                                         int* dev_error, cudaStream_t stream) {
  const int chunks_per_row = head_dim / 16;
  const int64_t total = (int64_t)num_tokens * num_kv_heads * chunks_per_row;
  if (total == 0) return cudaSuccess;
  const int threads = 256;
  const int64_t blocks = (total + threads - 1) / threads;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
  auto kern = src_dtype == PA_F16 ? reshape_and_cache_fp8_kernel<__half>
                                  : reshape_and_cache_fp8_kernel<__nv_bfloat16>;
  kern<<<(unsigned)blocks, threads, 0, stream>>>(
      static_cast<const uint4*>(key), static_cast<const uint4*>(value), key_stride / 8,
      value_stride / 8, static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache), slot_mapping,
      total, chunks_per_row, num_kv_heads, (int64_t)num_blocks * kBlockSize, k_scale, v_scale,
      dev_error);
  return cudaGetLastError();
}

cudaError_t launch_copy_pool_blocks(const void* src_k, const void* src_v, void* dst_k,
                                    void* dst_v, const CopyPairs& pairs, int n,
                                    int64_t block_bytes, cudaStream_t stream) {
  if (n == 0) return cudaSuccess;
  const int64_t vecs = block_bytes / 16;
  const int64_t per_cta = (int64_t)kCopyThreads * kCopyUnroll;
  const int64_t gx = (2 * vecs + per_cta - 1) / per_cta;
  dim3 grid((unsigned)gx, (unsigned)n);
  copy_pool_blocks_kernel<<<grid, kCopyThreads, 0, stream>>>(
      static_cast<const uint4*>(src_k), static_cast<const uint4*>(src_v),
      static_cast<uint4*>(dst_k), static_cast<uint4*>(dst_v), pairs, vecs);
  return cudaGetLastError();
}

}  // namespace pa
