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
//     array's address (cudaGetSymbolAddress) and caches it with the id of the
//     device's current context. A later call that finds another context current
//     (after cudaDeviceReset, say) looks the address up again. Make the first
//     call on a device, and the first after a reset, before any stream capture.
//   * Every call checks that out, q, both caches, the tables and the lengths
//     are device memory of the current device, and that the stream belongs to
//     it; otherwise it returns PA_ERR_INVALID_ARG and launches nothing (a
//     kernel handed another GPU's memory would fault instead of failing).
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
struct ScratchSlot {
  void* addr = nullptr;
  unsigned long long ctx_id = 0;
};
ScratchSlot g_scratch[kMaxDevices];

// cuCtxGetId from the driver, reached through the runtime (the library links
// no driver library). Null when the driver does not provide it; the address is
// then cached once per device for the life of the process.
using CtxGetIdFn = int (*)(void* ctx, unsigned long long* id);
CtxGetIdFn ctx_get_id() {
  static CtxGetIdFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess) {
      cudaGetLastError();
      return static_cast<CtxGetIdFn>(nullptr);
    }
    return reinterpret_cast<CtxGetIdFn>(p);
  }();
  return fn;
}

// Id of the context current on this thread; 0 when none is current or the id is
// unavailable.
unsigned long long current_ctx_id() {
  CtxGetIdFn fn = ctx_get_id();
  unsigned long long id = 0;
  if (fn == nullptr || fn(nullptr, &id) != 0) return 0;
  return id;
}

// Device address of g_noalloc_scratch in the current device's current context.
int scratch_address(int dev, void** out) {
  if (dev < 0 || dev >= kMaxDevices)
    return pa::fail(PA_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  ScratchSlot& slot = g_scratch[dev];
  const unsigned long long id = current_ctx_id();
  const bool have_ids = ctx_get_id() != nullptr;
  if (slot.addr == nullptr || (have_ids && (id == 0 || id != slot.ctx_id))) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr)
      return pa::fail(PA_ERR_CUDA, "cudaGetSymbolAddress of the built-in scratch: %s",
                      cudaGetErrorString(e));
    slot.addr = p;
    slot.ctx_id = current_ctx_id();  // the lookup made the device's context current
  }
  *out = slot.addr;
  return PA_OK;
}

// PA_OK when `p` is device (or managed) memory of device `dev`.
int on_device(const void* p, const char* name, int dev) {
  cudaPointerAttributes a{};
  const cudaError_t e = cudaPointerGetAttributes(&a, p);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return pa::fail(PA_ERR_INVALID_ARG, "%s: not a CUDA pointer (%s)", name,
                    cudaGetErrorString(e));
  }
  if (a.type != cudaMemoryTypeDevice && a.type != cudaMemoryTypeManaged)
    return pa::fail(PA_ERR_INVALID_ARG, "%s is not device memory", name);
  if (a.device != dev)
    return pa::fail(PA_ERR_INVALID_ARG,
                    "%s is memory of device %d but device %d is current; make the tensors' "
                    "device current before the call", name, a.device, dev);
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
  const pa::NvtxRange nvtx_range("pa_paged_decode_noalloc");
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
  int dev = 0;
  cudaError_t e = cudaSuccess;
  if (num_seqs > 0) {
    e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
      return pa::fail(PA_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    const struct {
      const void* p;
      const char* name;
    } bufs[] = {{out, "out"},         {q, "q"},
                {k_cache, "k_cache"}, {v_cache, "v_cache"},
                {block_tables, "block_tables"}, {context_lens, "context_lens"}};
    for (const auto& b : bufs) {
      if (b.p == nullptr) return pa::fail(PA_ERR_INVALID_ARG, "%s is null", b.name);
      if (int st = on_device(b.p, b.name, dev)) return st;
    }
    int stream_dev = dev;
    e = cudaStreamGetDevice(static_cast<cudaStream_t>(stream), &stream_dev);
    if (e != cudaSuccess) {
      cudaGetLastError();
      return pa::fail(PA_ERR_INVALID_ARG, "stream: %s", cudaGetErrorString(e));
    }
    if (stream_dev != dev)
      return pa::fail(PA_ERR_INVALID_ARG,
                      "the stream belongs to device %d but device %d is current", stream_dev, dev);
  }
  void* scratch = nullptr;
  if (need > 0 && num_seqs > 0) {
    if (int st = scratch_address(dev, &scratch)) return st;
    // The merge counters sit at the start of the workspace layout: one int per
    // (sequence, KV head). Clear them so a stale value from an earlier call
    // (for example one that timed out) cannot mislead this one.
    const size_t counter_bytes = (size_t)num_seqs * num_kv_heads * sizeof(int);
    e = cudaMemsetAsync(scratch, 0, counter_bytes, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess)
      return pa::fail(PA_ERR_CUDA, "clearing the built-in scratch: %s", cudaGetErrorString(e));
  }
  return pa_paged_decode(out, q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens,
                         seq_order, num_seqs, max_context_len, num_q_heads, num_kv_heads, head_dim,
                         block_size, num_blocks, scale, partition_tokens, scratch,
                         need > 0 ? kScratchBytes : 0, dev_error, dtype, stream);
}
