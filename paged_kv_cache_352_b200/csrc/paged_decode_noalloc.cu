// pa_paged_decode_noalloc: paged decode for callers that may not allocate
// device memory.
//
// Some callers cannot hand libpa a workspace. Examples are a plugin running
// inside a host runtime that owns every device allocation, and a latency-critical
// loop that must never reach cudaMalloc, which can synchronise the device. The
// split-KV merge still needs scratch memory: partial results and per-sequence
// counters. This variant takes that scratch from one fixed array compiled into
// the library. It then runs the same kernel as pa_paged_decode.
//
// How the array is used:
//   * The array is a file-scope __device__ object of PA_NOALLOC_WORKSPACE_BYTES.
//     Every GPU that loads the library holds it until the process exits.
//   * Host code cannot use the array's name as a device address. Once per
//     device, with that device current, the first call asks the runtime for the
//     array's address (cudaGetSymbolAddress) and caches it. Make that first call
//     before any stream capture on the device.
//   * All calls share the array, and it keeps whatever the last call left in it.
//     Each call first clears the counters the merge relies on (an async memset
//     on the caller's stream). Calls whose kernels overlap on the GPU race on
//     the array: run them on one stream or order them with events.
//   * Sizes whose scratch would exceed the array are rejected with
//     PA_ERR_UNSUPPORTED, and nothing is launched.
#include <cuda_runtime.h>

#include <mutex>

#include "pa_internal.h"

namespace {

constexpr size_t kScratchBytes = PA_NOALLOC_WORKSPACE_BYTES;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device (looked up once per device).
int scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess)
    return pa::fail(PA_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices)
    return pa::fail(PA_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr)
      return pa::fail(PA_ERR_CUDA, "cudaGetSymbolAddress of the built-in scratch: %s",
                      cudaGetErrorString(e));
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return PA_OK;
}

}  // namespace

extern "C" int pa_paged_decode_noalloc(void* out, const void* q, const void* k_cache,
                                       const void* v_cache, const int32_t* block_tables,
                                       int max_blocks_per_seq, const int32_t* context_lens,
                                       const int32_t* seq_order, int num_seqs,
                                       int max_context_len, int num_q_heads,
                                       int num_kv_heads, int head_dim, int block_size,
                                       int num_blocks, float scale, int partition_tokens,
                                       int* dev_error, int dtype, void* stream) {
  pa::clear_error();
  size_t need = 0;
  if (int st = pa_paged_decode_workspace_size(num_seqs, num_q_heads, num_kv_heads, head_dim,
                                              max_context_len, block_size, partition_tokens,
                                              &need))
    return st;
  if (need > kScratchBytes)
    return pa::fail(PA_ERR_UNSUPPORTED,
                    "this batch needs %zu bytes of split-KV scratch but the built-in array "
                    "holds %zu; use a larger partition_tokens, fewer sequences per call, or "
                    "pa_paged_decode with a caller-owned workspace",
                    need, kScratchBytes);
  void* scratch = nullptr;
  if (need > 0) {
    if (int st = scratch_address(&scratch)) return st;
    // The merge counters sit at the start of the workspace layout: one int per
    // (sequence, KV head). Clear them so a stale value from an earlier call
    // (for example one that timed out) cannot mislead this one.
    const size_t counter_bytes = (size_t)num_seqs * num_kv_heads * sizeof(int);
    const cudaError_t e =
        cudaMemsetAsync(scratch, 0, counter_bytes, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess)
      return pa::fail(PA_ERR_CUDA, "clearing the built-in scratch: %s", cudaGetErrorString(e));
  }
  return pa_paged_decode(out, q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens,
                         seq_order, num_seqs, max_context_len, num_q_heads, num_kv_heads, head_dim,
                         block_size, num_blocks, scale, partition_tokens, scratch,
                         need > 0 ? kScratchBytes : 0, dev_error, dtype, stream);
}
