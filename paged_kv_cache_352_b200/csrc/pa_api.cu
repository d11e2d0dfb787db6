// C interface of libpa: argument checks on the host, then kernel launches on the
// caller's stream. Nothing here synchronises or allocates device memory.
#include <cuda_runtime.h>
#include <stdarg.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <string>
#include <unordered_set>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "pa_internal.h"

namespace pa {

static thread_local std::string g_last_error;

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

void clear_error() { g_last_error.clear(); }

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Element bytes of a cache type (PA_F16, PA_BF16: 2; PA_FP8_E4M3: 1).
int64_t elem_bytes(int dtype) { return dtype == PA_FP8_E4M3 ? 1 : 2; }

int check_cache_shape(int num_kv_heads, int head_dim, int block_size, int num_blocks, int dtype,
                      bool allow_fp8 = false) {
  if (dtype != PA_F16 && dtype != PA_BF16 && !(allow_fp8 && dtype == PA_FP8_E4M3))
    return fail(PA_ERR_UNSUPPORTED, "dtype %d: expected PA_F16 or PA_BF16%s", dtype,
                allow_fp8 ? " or PA_FP8_E4M3" : "");
  if (block_size != kBlockSize)
    return fail(PA_ERR_UNSUPPORTED, "block_size %d: only %d is supported", block_size,
                kBlockSize);
  if (head_dim != 64 && head_dim != 128)
    return fail(PA_ERR_UNSUPPORTED, "head_dim %d: only 64 and 128 are supported", head_dim);
  if (num_kv_heads <= 0) return fail(PA_ERR_INVALID_ARG, "num_kv_heads must be positive");
  if (num_blocks <= 0) return fail(PA_ERR_INVALID_ARG, "num_blocks must be positive");
  return PA_OK;
}

// Device-addressable form of a pool pointer: device or managed memory as is,
// pinned host memory through its device alias; pageable memory is refused.
int device_view(const void* p, const char* name, void** out) {
  cudaPointerAttributes attr;
  const cudaError_t e = cudaPointerGetAttributes(&attr, p);
  if (e != cudaSuccess) {
    cudaGetLastError();  // the query's error is not sticky: clear it
    return fail(PA_ERR_INVALID_ARG, "%s: not memory the GPU can address (%s)", name,
                cudaGetErrorString(e));
  }
  if (attr.type == cudaMemoryTypeDevice || attr.type == cudaMemoryTypeManaged) {
    *out = const_cast<void*>(p);
    return PA_OK;
  }
  if (attr.type == cudaMemoryTypeHost && attr.devicePointer != nullptr) {
    *out = attr.devicePointer;
    return PA_OK;
  }
  return fail(PA_ERR_INVALID_ARG,
              "%s: not memory the GPU can address (pageable host memory must be pinned)", name);
}

int cuda_status(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return PA_OK;
  return fail(PA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool positive_finite(float x) { return x > 0.f && x <= 3.4028234663852886e38f; }

}  // namespace

int default_partition_blocks(int num_seqs, int num_kv_heads, int max_blocks, bool ordered) {
  // A CTA streams best over a long run of blocks: every extra partition costs its
  // CTA's pipeline ramp and a merge. Long partitions, though, leave a tail of
  // lone CTAs at the end of the launch. Partitions are therefore capped at
  // kMaxPartitionBlocks, and made shorter (never below kMinPartitionBlocks)
  // when the batch alone cannot give the GPU ~kSplitTargetUnits CTAs.
  const long long units = (long long)num_seqs * num_kv_heads;
  if (max_blocks < 1) return 1;
  long long pb = max_blocks;
  if (units < kSplitTargetUnits) {
    const long long parts = (kSplitTargetUnits + units - 1) / (units > 0 ? units : 1);
    pb = (max_blocks + parts - 1) / parts;
    if (pb < kMinPartitionBlocks) pb = kMinPartitionBlocks;
  }
  const int cap = ordered ? kMaxPartitionBlocksOrdered : kMaxPartitionBlocks;
  if (pb > cap) pb = cap;
  return (int)(pb < max_blocks ? pb : max_blocks);
}

// One warp per partition (plus a merge launch) pays off only for short partitions
// of long sequences, and only while its grid, WARPS = 4 times smaller, still
// fills the GPU. A CTA takes four consecutive partitions of one sequence, so a
// sequence with fewer partitions leaves warps idle: measured on 256 lognormal
// contexts (median ~660 tokens) at 1024-token partitions, warp mode took 2.2x
// the time of one CTA per partition. The library's own short partitions arise
// for small batches, which keep one CTA per partition.
constexpr int kWarpPartMinParts = 16;

bool use_warp_parts(int num_seqs, int num_kv_heads, int part_blocks, int max_parts) {
  static const int forced = [] {
    const char* e = getenv("PA_DECODE_SPLIT");
    if (e && !strcmp(e, "cta")) return 0;
    if (e && !strcmp(e, "warp")) return 1;
    return -1;
  }();
  if (max_parts <= 1) return false;
  if (forced >= 0) return forced == 1;
  const long long ctas = (long long)num_kv_heads * num_seqs * ((max_parts + 3) / 4);
  return part_blocks <= kWarpPartMaxBlocks && max_parts >= kWarpPartMinParts &&
         ctas >= kSplitTargetUnits;
}

int decode_layout(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                  int max_context_len, int partition_tokens, bool ordered, DecodeLayout* lay) {
  if (partition_tokens < 0 || partition_tokens % kBlockSize != 0)
    return fail(PA_ERR_INVALID_ARG, "partition_tokens %d: must be 0 or a positive multiple of %d",
                partition_tokens, kBlockSize);
  if (max_context_len < 0) return fail(PA_ERR_INVALID_ARG, "max_context_len must be >= 0");
  const int group = num_q_heads / num_kv_heads;
  const int max_blocks = (max_context_len + kBlockSize - 1) / kBlockSize;
  const int part_blocks = partition_tokens == 0
                              ? default_partition_blocks(num_seqs, num_kv_heads, max_blocks,
                                                         ordered)
                              : partition_tokens / kBlockSize;
  int max_parts = (max_blocks + part_blocks - 1) / part_blocks;
  if (max_parts < 1) max_parts = 1;
  if (max_parts > 65535)
    return fail(PA_ERR_UNSUPPORTED, "%d partitions per sequence exceed the grid limit", max_parts);
  lay->part_blocks = part_blocks;
  lay->max_parts = max_parts;
  if (max_parts == 1) {
    lay->count_off = lay->ml_off = lay->acc_off = lay->bytes = 0;
    return PA_OK;
  }
  auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
  const size_t units = (size_t)num_seqs * num_kv_heads;
  lay->count_off = 0;
  lay->ml_off = up(units * sizeof(int));
  lay->acc_off = up(lay->ml_off + units * max_parts * group * 2 * sizeof(float));
  lay->bytes = up(lay->acc_off + units * max_parts * group * head_dim * sizeof(float));
  return PA_OK;
}

}  // namespace pa

pa::NvtxRange::NvtxRange(const char* name) { nvtxRangePushA(name); }
pa::NvtxRange::~NvtxRange() { nvtxRangePop(); }

using namespace pa;

extern "C" {

const char* pa_last_error(void) { return g_last_error.c_str(); }

int pa_version(void) { return 111; }

int pa_test_stall_next_decode(unsigned long long wait_limit_ns) {
  clear_error();
  if (wait_limit_ns < 1000ull || wait_limit_ns > 100000000ull)
    return fail(PA_ERR_INVALID_ARG, "wait_limit_ns %llu: must be in [1 us, 100 ms]",
                wait_limit_ns);
  set_stall_request(wait_limit_ns);
  return PA_OK;
}

int pa_reshape_and_cache(const void* key, const void* value, int64_t key_token_stride,
                         int64_t value_token_stride, void* k_cache, void* v_cache,
                         const int64_t* slot_mapping, int num_tokens, int num_kv_heads,
                         int head_dim, int block_size, int num_blocks, int dtype,
                         int* dev_error, void* stream) {
  const NvtxRange nvtx_range("pa_reshape_and_cache");
  clear_error();
  if (int st = check_cache_shape(num_kv_heads, head_dim, block_size, num_blocks, dtype)) return st;
  if (num_tokens < 0) return fail(PA_ERR_INVALID_ARG, "num_tokens must be >= 0");
  if (num_tokens == 0) return PA_OK;
  if (!key || !value || !k_cache || !v_cache || !slot_mapping)
    return fail(PA_ERR_INVALID_ARG, "null pointer argument");
  const int64_t row = (int64_t)num_kv_heads * head_dim;
  if (key_token_stride < row || value_token_stride < row || key_token_stride % 8 ||
      value_token_stride % 8)
    return fail(PA_ERR_INVALID_ARG,
                "token strides (%lld, %lld) must be >= num_kv_heads*head_dim (%lld) and a "
                "multiple of 8",
                (long long)key_token_stride, (long long)value_token_stride, (long long)row);
  if (!aligned16(key) || !aligned16(value) || !aligned16(k_cache) || !aligned16(v_cache))
    return fail(PA_ERR_INVALID_ARG, "key, value and cache pointers must be 16-byte aligned");
  return cuda_status(launch_reshape_and_cache(key, value, key_token_stride, value_token_stride,
                                              k_cache, v_cache, slot_mapping, num_tokens,
                                              num_kv_heads, head_dim, num_blocks, dev_error,
                                              static_cast<cudaStream_t>(stream)),
                     "reshape_and_cache launch");
}

int pa_copy_blocks(void* k_cache, void* v_cache, const int64_t* pairs, int num_pairs,
                   int num_kv_heads, int head_dim, int block_size, int num_blocks, int dtype,
                   void* stream) {
  const NvtxRange nvtx_range("pa_copy_blocks");
  clear_error();
  if (int st = check_cache_shape(num_kv_heads, head_dim, block_size, num_blocks, dtype, true))
    return st;
  if (num_pairs < 0) return fail(PA_ERR_INVALID_ARG, "num_pairs must be >= 0");
  if (num_pairs == 0) return PA_OK;
  if (!k_cache || !v_cache || !pairs) return fail(PA_ERR_INVALID_ARG, "null pointer argument");
  if (!aligned16(k_cache) || !aligned16(v_cache))
    return fail(PA_ERR_INVALID_ARG, "cache pointers must be 16-byte aligned");
  std::unordered_set<int64_t> dsts, srcs;
  dsts.reserve(num_pairs * 2);
  srcs.reserve(num_pairs * 2);
  for (int i = 0; i < num_pairs; ++i) {
    const int64_t s = pairs[2 * i], d = pairs[2 * i + 1];
    if (s < 0 || s >= num_blocks || d < 0 || d >= num_blocks)
      return fail(PA_ERR_INVALID_ARG, "pair %d (%lld -> %lld) outside the pool of %d blocks", i,
                  (long long)s, (long long)d, num_blocks);
    if (!dsts.insert(d).second)
      return fail(PA_ERR_INVALID_ARG, "destination block %lld appears twice", (long long)d);
    srcs.insert(s);
  }
  for (int64_t d : dsts)
    if (srcs.count(d))
      return fail(PA_ERR_INVALID_ARG, "block %lld is both a source and a destination",
                  (long long)d);
  const int64_t block_bytes = (int64_t)num_kv_heads * kBlockSize * head_dim * elem_bytes(dtype);
  for (int first = 0; first < num_pairs; first += kMaxCopyPairsPerLaunch) {
    const int n = std::min(kMaxCopyPairsPerLaunch, num_pairs - first);
    CopyPairs cp;
    for (int i = 0; i < n; ++i) {
      cp.src[i] = (int32_t)pairs[2 * (first + i)];
      cp.dst[i] = (int32_t)pairs[2 * (first + i) + 1];
    }
    if (int st = cuda_status(launch_copy_pool_blocks(k_cache, v_cache, k_cache, v_cache, cp, n,
                                                     block_bytes, static_cast<cudaStream_t>(stream)),
                             "copy_blocks launch"))
      return st;
  }
  return PA_OK;
}

int pa_swap_blocks(const void* src_k, const void* src_v, int src_num_blocks, void* dst_k,
                   void* dst_v, int dst_num_blocks, const int64_t* pairs, int num_pairs,
                   int num_kv_heads, int head_dim, int block_size, int dtype, void* stream) {
  const NvtxRange nvtx_range("pa_swap_blocks");
  clear_error();
  if (int st = check_cache_shape(num_kv_heads, head_dim, block_size, src_num_blocks, dtype, true))
    return st;
  if (dst_num_blocks <= 0) return fail(PA_ERR_INVALID_ARG, "dst_num_blocks must be positive");
  if (num_pairs < 0) return fail(PA_ERR_INVALID_ARG, "num_pairs must be >= 0");
  if (num_pairs == 0) return PA_OK;
  if (!src_k || !src_v || !dst_k || !dst_v || !pairs)
    return fail(PA_ERR_INVALID_ARG, "null pointer argument");
  if (src_k == dst_k || src_v == dst_v || src_k == dst_v || src_v == dst_k)
    return fail(PA_ERR_INVALID_ARG, "source and destination must be different pools");
  if (!aligned16(src_k) || !aligned16(src_v) || !aligned16(dst_k) || !aligned16(dst_v))
    return fail(PA_ERR_INVALID_ARG, "pool pointers must be 16-byte aligned");
  std::unordered_set<int64_t> dsts;
  dsts.reserve(num_pairs * 2);
  for (int i = 0; i < num_pairs; ++i) {
    const int64_t s = pairs[2 * i], d = pairs[2 * i + 1];
    if (s < 0 || s >= src_num_blocks || d < 0 || d >= dst_num_blocks)
      return fail(PA_ERR_INVALID_ARG, "pair %d (%lld -> %lld) outside the pools (%d, %d blocks)",
                  i, (long long)s, (long long)d, src_num_blocks, dst_num_blocks);
    if (!dsts.insert(d).second)
      return fail(PA_ERR_INVALID_ARG, "destination block %lld appears twice", (long long)d);
  }
  void *sk, *sv, *dk, *dv;
  if (int st = device_view(src_k, "src_k", &sk)) return st;
  if (int st = device_view(src_v, "src_v", &sv)) return st;
  if (int st = device_view(dst_k, "dst_k", &dk)) return st;
  if (int st = device_view(dst_v, "dst_v", &dv)) return st;
  const int64_t block_bytes = (int64_t)num_kv_heads * kBlockSize * head_dim * elem_bytes(dtype);
  for (int first = 0; first < num_pairs; first += kMaxCopyPairsPerLaunch) {
    const int n = std::min(kMaxCopyPairsPerLaunch, num_pairs - first);
    CopyPairs cp;
    for (int i = 0; i < n; ++i) {
      cp.src[i] = (int32_t)pairs[2 * (first + i)];
      cp.dst[i] = (int32_t)pairs[2 * (first + i) + 1];
    }
    if (int st = cuda_status(
            launch_copy_pool_blocks(sk, sv, dk, dv, cp, n, block_bytes,
                                    static_cast<cudaStream_t>(stream)),
            "swap_blocks launch"))
      return st;
  }
  return PA_OK;
}

int pa_paged_decode_workspace_size(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                                   int max_context_len, int block_size, int partition_tokens,
                                   size_t* bytes) {
  clear_error();
  if (!bytes) return fail(PA_ERR_INVALID_ARG, "bytes must not be NULL");
  if (block_size != kBlockSize)
    return fail(PA_ERR_UNSUPPORTED, "block_size %d: only %d is supported", block_size,
                kBlockSize);
  if (num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || num_q_heads % num_kv_heads)
    return fail(PA_ERR_INVALID_ARG, "bad sequence or head counts");
  DecodeLayout lay;
  // Without an order the default partitions are shorter, so that layout is the
  // larger of the two.
  if (int st = decode_layout(num_seqs, num_q_heads, num_kv_heads, head_dim, max_context_len,
                             partition_tokens, false, &lay))
    return st;
  *bytes = lay.bytes;
  return PA_OK;
}

int pa_paged_decode_plan(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                         int max_context_len, int block_size, int partition_tokens, int ordered,
                         int* part_blocks, int* max_parts, int* launches) {
  clear_error();
  if (!part_blocks || !max_parts || !launches)
    return fail(PA_ERR_INVALID_ARG, "null output pointer");
  if (block_size != kBlockSize)
    return fail(PA_ERR_UNSUPPORTED, "block_size %d: only %d is supported", block_size,
                kBlockSize);
  if (num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || num_q_heads % num_kv_heads)
    return fail(PA_ERR_INVALID_ARG, "bad sequence or head counts");
  DecodeLayout lay;
  if (int st = decode_layout(num_seqs, num_q_heads, num_kv_heads, head_dim, max_context_len,
                             partition_tokens, ordered != 0, &lay))
    return st;
  *part_blocks = lay.part_blocks;
  *max_parts = lay.max_parts;
  *launches = num_seqs == 0 ? 0
              : use_warp_parts(num_seqs, num_kv_heads, lay.part_blocks, lay.max_parts) ? 2 : 1;
  return PA_OK;
}

int pa_longest_first_order(const int32_t* context_lens, int n, int32_t* order) {
  clear_error();
  if (n < 0) return fail(PA_ERR_INVALID_ARG, "n must be >= 0");
  if (n == 0) return PA_OK;
  if (!context_lens || !order) return fail(PA_ERR_INVALID_ARG, "null pointer argument");
  for (int i = 0; i < n; ++i) order[i] = i;
  std::stable_sort(order, order + n, [context_lens](int32_t x, int32_t y) {
    return context_lens[x] > context_lens[y];
  });
  return PA_OK;
}

int pa_cascade_order(const int32_t* context_lens, const int32_t* seq_group,
                     const int32_t* group_prefix_blocks, int num_groups, int n, int32_t* order) {
  clear_error();
  if (n < 0 || num_groups < 0) return fail(PA_ERR_INVALID_ARG, "n and num_groups must be >= 0");
  if (n == 0) return PA_OK;
  if (!context_lens || !order || (num_groups > 0 && (!seq_group || !group_prefix_blocks)))
    return fail(PA_ERR_INVALID_ARG, "null pointer argument");
  // the tokens a sequence's own-block decode reads: its context after the prefix
  // of its group (its whole context outside any group)
  std::vector<int64_t> own(n);
  for (int i = 0; i < n; ++i) {
    const int g = num_groups > 0 ? seq_group[i] : -1;
    const int64_t pre = g >= 0 && g < num_groups ? (int64_t)group_prefix_blocks[g] * kBlockSize : 0;
    own[i] = std::max<int64_t>(0, (int64_t)context_lens[i] - pre);
  }
  for (int i = 0; i < n; ++i) order[i] = i;
  std::stable_sort(order, order + n, [&own](int32_t x, int32_t y) { return own[x] > own[y]; });
  return PA_OK;
}

}  // extern "C"

namespace {

// pa_paged_decode over a cache of type cache_dtype (dtype itself, or E4M3 with
// key and value scales).
int paged_decode_impl(void* out, const void* q, const void* k_cache, const void* v_cache,
                      const int32_t* block_tables, int max_blocks_per_seq,
                      const int32_t* context_lens, const int32_t* seq_order, int num_seqs,
                      int max_context_len, int num_q_heads, int num_kv_heads, int head_dim,
                      int block_size, int num_blocks, float scale, float k_scale, float v_scale,
                      int partition_tokens, void* workspace, size_t workspace_bytes,
                      int* dev_error, int dtype, int cache_dtype, void* stream) {
  if (int st = check_cache_shape(num_kv_heads, head_dim, block_size, num_blocks, dtype)) return st;
  if (num_seqs < 0) return fail(PA_ERR_INVALID_ARG, "num_seqs must be >= 0");
  if (num_seqs > 65535)
    return fail(PA_ERR_UNSUPPORTED, "num_seqs %d exceeds 65535 per call", num_seqs);
  if (num_q_heads <= 0 || num_q_heads % num_kv_heads)
    return fail(PA_ERR_INVALID_ARG, "num_q_heads %d must be a positive multiple of num_kv_heads %d",
                num_q_heads, num_kv_heads);
  const int group = num_q_heads / num_kv_heads;
  if (group != 1 && group != 2 && group != 4 && group != 8)
    return fail(PA_ERR_UNSUPPORTED, "query heads per KV head = %d: supported 1, 2, 4, 8", group);
  if (num_kv_heads > 65535) return fail(PA_ERR_UNSUPPORTED, "too many KV heads");
  if (max_blocks_per_seq <= 0) return fail(PA_ERR_INVALID_ARG, "max_blocks_per_seq must be > 0");
  if (!(scale == scale)) return fail(PA_ERR_INVALID_ARG, "scale is NaN");
  if (num_seqs == 0) return PA_OK;
  if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens)
    return fail(PA_ERR_INVALID_ARG, "null pointer argument");
  if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache))
    return fail(PA_ERR_INVALID_ARG, "out, q and cache pointers must be 16-byte aligned");
  DecodeLayout lay;
  if (int st = decode_layout(num_seqs, num_q_heads, num_kv_heads, head_dim, max_context_len,
                             partition_tokens, seq_order != nullptr, &lay))
    return st;
  if (lay.bytes > 0) {
    if (!workspace || workspace_bytes < lay.bytes)
      return fail(PA_ERR_INVALID_ARG, "workspace of %zu bytes needed, %zu given", lay.bytes,
                  workspace ? workspace_bytes : (size_t)0);
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
      return fail(PA_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  }
  DecodeArgs a;
  a.out = out;
  a.q = q;
  a.k_cache = k_cache;
  a.v_cache = v_cache;
  a.block_tables = block_tables;
  a.context_lens = context_lens;
  a.seq_order = seq_order;
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  a.ws_count = lay.bytes ? reinterpret_cast<int*>(ws + lay.count_off) : nullptr;
  a.ws_m = lay.bytes ? reinterpret_cast<float*>(ws + lay.ml_off) : nullptr;
  a.ws_l = lay.bytes ? a.ws_m + (size_t)num_seqs * num_kv_heads * lay.max_parts * group : nullptr;
  a.ws_acc = lay.bytes ? reinterpret_cast<float*>(ws + lay.acc_off) : nullptr;
  a.dev_error = dev_error;
  a.max_blocks_per_seq = max_blocks_per_seq;
  a.max_context_len = max_context_len;
  a.num_seqs = num_seqs;
  a.num_q_heads = num_q_heads;
  a.num_kv_heads = num_kv_heads;
  a.num_blocks = num_blocks;
  a.part_blocks = lay.part_blocks;
  a.max_parts = lay.max_parts;
  a.scale_log2 = scale * 1.4426950408889634f * k_scale;
  a.out_scale = v_scale;
  a.warp_parts = use_warp_parts(num_seqs, num_kv_heads, lay.part_blocks, lay.max_parts);
  a.states_only = 0;
  const cudaError_t e = launch_paged_decode(a, head_dim, group, dtype, cache_dtype,
                                            static_cast<cudaStream_t>(stream));
  if (e == cudaErrorInvalidConfiguration)
    return fail(PA_ERR_UNSUPPORTED,
                "%d partitions per sequence need more shared memory than the kernel allows; "
                "use a larger partition_tokens",
                lay.max_parts);
  return cuda_status(e, "paged_decode launch");
}

// Workspace of a cascade decode: stacked queries, the groups' prefix tables and
// lengths, the own-block tables and lengths, then the partition states of the
// decode over the groups' prefixes and of the decode over the own blocks.
struct CascadeLayout {
  int g_part_blocks, g_parts, s_part_blocks, s_parts;
  size_t gq_off, gt_off, gctx_off, st_off, sctx_off, spb_off, snp_off;
  size_t gcount_off, gml_off, gacc_off, scount_off, sml_off, sacc_off, bytes;
};

int cascade_layout(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                   int max_context_len, int max_blocks_per_seq, int num_groups, int group_size,
                   int max_prefix_blocks, CascadeLayout* L) {
  if (num_seqs < 0 || num_seqs > 65535)
    return fail(PA_ERR_INVALID_ARG, "num_seqs %d: expected 0 .. 65535", num_seqs);
  if (num_q_heads <= 0 || num_kv_heads <= 0 || num_q_heads % num_kv_heads)
    return fail(PA_ERR_INVALID_ARG, "num_q_heads %d must be a positive multiple of num_kv_heads %d",
                num_q_heads, num_kv_heads);
  if (head_dim != 64 && head_dim != 128)
    return fail(PA_ERR_UNSUPPORTED, "head_dim %d: only 64 and 128 are supported", head_dim);
  const int gh = num_q_heads / num_kv_heads;
  if (gh != 1 && gh != 2 && gh != 4 && gh != 8)
    return fail(PA_ERR_UNSUPPORTED, "query heads per KV head = %d: supported 1, 2, 4, 8", gh);
  if (max_context_len < 0) return fail(PA_ERR_INVALID_ARG, "max_context_len must be >= 0");
  if (max_blocks_per_seq <= 0) return fail(PA_ERR_INVALID_ARG, "max_blocks_per_seq must be > 0");
  if (num_groups < 0 || num_groups > 65535)
    return fail(PA_ERR_INVALID_ARG, "num_groups %d: expected 0 .. 65535", num_groups);
  const int gg = group_size * gh;
  if (group_size < 1 || (gg != 1 && gg != 2 && gg != 4 && gg != 8))
    return fail(PA_ERR_UNSUPPORTED,
                "group_size %d x %d query heads per KV head must be 1, 2, 4 or 8", group_size, gh);
  if (num_groups > 0 && (max_prefix_blocks < 1 || max_prefix_blocks > max_blocks_per_seq))
    return fail(PA_ERR_INVALID_ARG, "max_prefix_blocks %d: expected 1 .. max_blocks_per_seq (%d)",
                max_prefix_blocks, max_blocks_per_seq);
  const int ng = num_groups > 0 ? num_groups : 0;
  const int pmax = num_groups > 0 ? max_prefix_blocks : 1;
  // The own-block CTAs run beside the prefix CTAs (in the same launch, or on a
  // second stream), so they count toward filling the GPU: a prefix is split
  // below the cap only when groups and sequences together give fewer than
  // kSplitTargetUnits (group or sequence, KV head) pairs. On 16 groups of 8
  // samples with 62-block prefixes and 32 KV heads, one partition per prefix
  // measured faster than two: 62.3 -> 58.0 us over 8-bit caches, 88.9 -> 88.5 us
  // over 16-bit ones (16- or 21-block partitions: slower still).
  L->g_part_blocks = default_partition_blocks(ng + num_seqs, num_kv_heads, pmax, false);
  L->g_parts = (pmax + L->g_part_blocks - 1) / L->g_part_blocks;
  const int own_blocks = std::max(1, (max_context_len + kBlockSize - 1) / kBlockSize);
  L->s_part_blocks = default_partition_blocks(num_seqs > 0 ? num_seqs : 1, num_kv_heads,
                                              own_blocks, false);
  L->s_parts = (own_blocks + L->s_part_blocks - 1) / L->s_part_blocks;
  if (L->g_parts > 65535 || L->s_parts > 65535)
    return fail(PA_ERR_UNSUPPORTED, "too many partitions per sequence");
  // prefix-state rows are addressed with 32-bit indices
  if ((long long)ng * num_kv_heads * L->g_parts * gg >= 0x7fffffffLL)
    return fail(PA_ERR_UNSUPPORTED, "too many groups x KV heads x partitions");
  auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o = up(o + bytes);
    return at;
  };
  const size_t gu = (size_t)ng * num_kv_heads, su = (size_t)num_seqs * num_kv_heads;
  L->gq_off = take((size_t)ng * num_kv_heads * gg * head_dim * 2);
  L->gt_off = take((size_t)ng * max_blocks_per_seq * 4);
  L->gctx_off = take((size_t)ng * 4);
  L->st_off = take((size_t)num_seqs * max_blocks_per_seq * 4);
  L->sctx_off = take((size_t)num_seqs * 4);
  L->spb_off = take((size_t)num_seqs * 4);
  L->snp_off = take((size_t)num_seqs * 4);
  L->gcount_off = take(gu * sizeof(int));
  L->gml_off = take(gu * L->g_parts * gg * 2 * sizeof(float));
  L->gacc_off = take(gu * L->g_parts * gg * head_dim * sizeof(float));
  L->scount_off = take(su * sizeof(int));
  L->sml_off = take(su * L->s_parts * gh * 2 * sizeof(float));
  L->sacc_off = take(su * L->s_parts * gh * head_dim * sizeof(float));
  L->bytes = o;
  return PA_OK;
}

// The decode over the groups' prefixes runs on a second stream beside the
// own-block decode on the caller's stream (the two read disjoint blocks and
// write disjoint states), forked after the prepare kernel and joined before the
// merge by events. One stream and two events per device and host thread, made
// on first use and kept for the life of the process.
struct AuxStream {
  cudaStream_t stream = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
};

constexpr int kMaxAuxDevices = 64;

int aux_stream(AuxStream** out) {
  thread_local AuxStream aux[kMaxAuxDevices];
  int dev = 0;
  if (int st = cuda_status(cudaGetDevice(&dev), "cudaGetDevice")) return st;
  if (dev < 0 || dev >= kMaxAuxDevices) return fail(PA_ERR_UNSUPPORTED, "device %d", dev);
  AuxStream& a = aux[dev];
  if (!a.stream) {
    if (int st = cuda_status(cudaStreamCreateWithFlags(&a.stream, cudaStreamNonBlocking),
                             "auxiliary stream"))
      return st;
    if (int st = cuda_status(cudaEventCreateWithFlags(&a.fork, cudaEventDisableTiming),
                             "fork event"))
      return st;
    if (int st = cuda_status(cudaEventCreateWithFlags(&a.join, cudaEventDisableTiming),
                             "join event"))
      return st;
  }
  *out = &a;
  return PA_OK;
}

int paged_decode_cascade_impl(void* out, const void* q, const void* k_cache, const void* v_cache,
                              const int32_t* block_tables, int max_blocks_per_seq,
                              const int32_t* context_lens, const int32_t* seq_order,
                              int num_seqs, int max_context_len,
                              int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                              int num_blocks, float scale, float k_scale, float v_scale,
                              const int32_t* group_members, const int32_t* group_prefix_blocks,
                              const int32_t* seq_group, const int32_t* seq_member,
                              int num_groups, int group_size, int max_prefix_blocks,
                              void* workspace, size_t workspace_bytes, int* dev_error,
                              int dtype, int cache_dtype, void* stream) {
  if (int st = check_cache_shape(num_kv_heads, head_dim, block_size, num_blocks, dtype)) return st;
  CascadeLayout lay;
  if (int st = cascade_layout(num_seqs, num_q_heads, num_kv_heads, head_dim, max_context_len,
                              max_blocks_per_seq, num_groups, group_size, max_prefix_blocks, &lay))
    return st;
  if (!(scale == scale)) return fail(PA_ERR_INVALID_ARG, "scale is NaN");
  if (num_seqs == 0) return PA_OK;
  if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens || !seq_group ||
      !seq_member || (num_groups > 0 && (!group_members || !group_prefix_blocks)))
    return fail(PA_ERR_INVALID_ARG, "null pointer argument");
  if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache))
    return fail(PA_ERR_INVALID_ARG, "out, q and cache pointers must be 16-byte aligned");
  if (!workspace || workspace_bytes < lay.bytes)
    return fail(PA_ERR_INVALID_ARG, "workspace of %zu bytes needed, %zu given", lay.bytes,
                workspace ? workspace_bytes : (size_t)0);
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(PA_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  const int gh = num_q_heads / num_kv_heads;
  const int gg = group_size * gh;
  CascadeArgs c;
  c.q = q;
  c.block_tables = block_tables;
  c.context_lens = context_lens;
  c.group_members = group_members;
  c.group_prefix_blocks = group_prefix_blocks;
  c.seq_group = seq_group;
  c.seq_member = seq_member;
  c.gq = ws + lay.gq_off;
  c.g_tables = reinterpret_cast<int32_t*>(ws + lay.gt_off);
  c.g_ctx = reinterpret_cast<int32_t*>(ws + lay.gctx_off);
  c.s_tables = reinterpret_cast<int32_t*>(ws + lay.st_off);
  c.s_ctx = reinterpret_cast<int32_t*>(ws + lay.sctx_off);
  c.s_pbase = reinterpret_cast<int32_t*>(ws + lay.spb_off);
  c.s_np = reinterpret_cast<int32_t*>(ws + lay.snp_off);
  const size_t gu = (size_t)num_groups * num_kv_heads, su = (size_t)num_seqs * num_kv_heads;
  float* gm = reinterpret_cast<float*>(ws + lay.gml_off);
  float* sm = reinterpret_cast<float*>(ws + lay.sml_off);
  c.g_m = gm;
  c.g_l = gm + gu * lay.g_parts * gg;
  c.g_acc = reinterpret_cast<float*>(ws + lay.gacc_off);
  c.s_m = sm;
  c.s_l = sm + su * lay.s_parts * gh;
  c.s_acc = reinterpret_cast<float*>(ws + lay.sacc_off);
  c.out = out;
  c.dev_error = dev_error;
  c.num_seqs = num_seqs;
  c.num_groups = num_groups;
  c.group_size = group_size;
  c.num_q_heads = num_q_heads;
  c.num_kv_heads = num_kv_heads;
  c.max_blocks_per_seq = max_blocks_per_seq;
  c.max_prefix_blocks = num_groups > 0 ? max_prefix_blocks : 0;
  c.max_context_len = max_context_len;
  c.g_parts = lay.g_parts;
  c.g_part_blocks = lay.g_part_blocks;
  c.s_parts = lay.s_parts;
  c.s_part_blocks = lay.s_part_blocks;
  c.out_scale = v_scale;
  // Both decodes in one launch where the shapes allow (8 stacked query heads
  // per KV head): its prefix CTAs read the members' query rows and the leader's
  // table in place, so prepare stacks no queries. Otherwise two decodes on two
  // streams, the prefix decode over prepare's stacked queries and tables.
  const bool single = num_groups > 0 && cascade_single_launch(head_dim, gh, gg, dtype, cache_dtype);
  if (int e = cuda_status(launch_cascade_prepare(c, head_dim, !single, st),
                          "cascade prepare launch"))
    return e;

  // both decodes leave partition states only; the merge writes `out`
  DecodeArgs a{};
  a.out = out;
  a.k_cache = k_cache;
  a.v_cache = v_cache;
  a.seq_order = nullptr;
  a.dev_error = dev_error;
  a.max_blocks_per_seq = max_blocks_per_seq;
  a.max_context_len = max_context_len;
  a.num_kv_heads = num_kv_heads;
  a.num_blocks = num_blocks;
  a.scale_log2 = scale * 1.4426950408889634f * k_scale;
  a.out_scale = 1.f;
  a.warp_parts = 0;
  a.states_only = 1;
  DecodeArgs own = a;
  own.q = q;
  own.seq_order = seq_order;  // the own-block CTAs in the caller's order
  own.block_tables = c.s_tables;
  own.context_lens = c.s_ctx;
  own.ws_count = reinterpret_cast<int*>(ws + lay.scount_off);
  own.ws_m = sm;
  own.ws_l = const_cast<float*>(c.s_l);
  own.ws_acc = const_cast<float*>(c.s_acc);
  own.num_seqs = num_seqs;
  own.num_q_heads = num_q_heads;
  own.part_blocks = lay.s_part_blocks;
  own.max_parts = lay.s_parts;
  DecodeArgs gpre = a;
  gpre.q = c.gq;
  gpre.block_tables = c.g_tables;
  gpre.context_lens = c.g_ctx;
  gpre.ws_count = reinterpret_cast<int*>(ws + lay.gcount_off);
  gpre.ws_m = gm;
  gpre.ws_l = const_cast<float*>(c.g_l);
  gpre.ws_acc = const_cast<float*>(c.g_acc);
  gpre.num_seqs = num_groups;
  gpre.num_q_heads = num_kv_heads * gg;
  gpre.part_blocks = lay.g_part_blocks;
  gpre.max_parts = lay.g_parts;
  if (single) {
    gpre.q = q;
    gpre.block_tables = block_tables;
    gpre.grp_members = group_members;
    gpre.grp_prefix_blocks = group_prefix_blocks;
    gpre.grp_size = group_size;
    gpre.grp_heads = gh;
    gpre.grp_src_seqs = num_seqs;
    gpre.grp_max_prefix_blocks = max_prefix_blocks;
    if (int e = cuda_status(launch_cascade_decode(gpre, own, head_dim, gh, dtype, cache_dtype, st),
                            "cascade decode launch"))
      return e;
    return cuda_status(launch_cascade_merge(c, head_dim, dtype, st), "cascade merge launch");
  }
  AuxStream* aux = nullptr;
  if (num_groups > 0) {
    if (int e = aux_stream(&aux)) return e;
    if (int e = cuda_status(cudaEventRecord(aux->fork, st), "fork record")) return e;
    if (int e = cuda_status(cudaStreamWaitEvent(aux->stream, aux->fork, 0), "fork wait"))
      return e;
    if (int e = cuda_status(launch_paged_decode(gpre, head_dim, gg, dtype, cache_dtype,
                                                aux->stream),
                            "cascade prefix decode launch"))
      return e;
    if (int e = cuda_status(cudaEventRecord(aux->join, aux->stream), "join record")) return e;
  }
  if (int e = cuda_status(launch_paged_decode(own, head_dim, gh, dtype, cache_dtype, st),
                          "cascade own-block decode launch"))
    return e;
  if (aux) {
    if (int e = cuda_status(cudaStreamWaitEvent(st, aux->join, 0), "join wait")) return e;
  }
  return cuda_status(launch_cascade_merge(c, head_dim, dtype, st), "cascade merge launch");
}

}  // namespace

extern "C" {

int pa_paged_decode_cascade_workspace_size(int num_seqs, int num_q_heads, int num_kv_heads,
                                           int head_dim, int max_context_len,
                                           int max_blocks_per_seq, int block_size, int num_groups,
                                           int group_size, int max_prefix_blocks, size_t* bytes) {
  clear_error();
  if (!bytes) return fail(PA_ERR_INVALID_ARG, "bytes must not be NULL");
  if (block_size != kBlockSize)
    return fail(PA_ERR_UNSUPPORTED, "block_size %d: only %d is supported", block_size,
                kBlockSize);
  CascadeLayout lay;
  if (int st = cascade_layout(num_seqs, num_q_heads, num_kv_heads, head_dim, max_context_len,
                              max_blocks_per_seq, num_groups, group_size, max_prefix_blocks, &lay))
    return st;
  *bytes = lay.bytes;
  return PA_OK;
}

int pa_paged_decode_cascade_plan(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                                 int max_context_len, int max_blocks_per_seq, int block_size,
                                 int num_groups, int group_size, int max_prefix_blocks, int dtype,
                                 int fp8_cache, int* prefix_part_blocks, int* prefix_parts,
                                 int* own_part_blocks, int* own_parts, int* launches) {
  clear_error();
  if (!prefix_part_blocks || !prefix_parts || !own_part_blocks || !own_parts || !launches)
    return fail(PA_ERR_INVALID_ARG, "null output pointer");
  if (block_size != kBlockSize)
    return fail(PA_ERR_UNSUPPORTED, "block_size %d: only %d is supported", block_size,
                kBlockSize);
  if (dtype != PA_F16 && dtype != PA_BF16)
    return fail(PA_ERR_UNSUPPORTED, "dtype %d: expected PA_F16 or PA_BF16", dtype);
  CascadeLayout lay;
  if (int st = cascade_layout(num_seqs, num_q_heads, num_kv_heads, head_dim, max_context_len,
                              max_blocks_per_seq, num_groups, group_size, max_prefix_blocks, &lay))
    return st;
  const int gh = num_q_heads / num_kv_heads;
  const bool single =
      num_groups > 0 &&
      cascade_single_launch(head_dim, gh, group_size * gh, dtype, fp8_cache ? PA_FP8_E4M3 : dtype);
  *prefix_part_blocks = num_groups > 0 ? lay.g_part_blocks : 0;
  *prefix_parts = num_groups > 0 ? lay.g_parts : 0;
  *own_part_blocks = lay.s_part_blocks;
  *own_parts = lay.s_parts;
  // prepare, the decode(s), merge: the two decodes share a launch where the
  // shapes allow, else the prefix decode runs on a second stream
  *launches = num_seqs == 0 ? 0 : (num_groups > 0 && !single) ? 4 : 3;
  return PA_OK;
}

int pa_paged_decode_cascade(void* out, const void* q, const void* k_cache, const void* v_cache,
                            const int32_t* block_tables, int max_blocks_per_seq,
                            const int32_t* context_lens, const int32_t* seq_order,
                            int num_seqs, int max_context_len, int num_q_heads,
                            int num_kv_heads, int head_dim, int block_size, int num_blocks,
                            float scale, const int32_t* group_members,
                            const int32_t* group_prefix_blocks, const int32_t* seq_group,
                            const int32_t* seq_member, int num_groups, int group_size,
                            int max_prefix_blocks, void* workspace, size_t workspace_bytes,
                            int* dev_error, int dtype, void* stream) {
  const NvtxRange nvtx_range("pa_paged_decode_cascade");
  clear_error();
  return paged_decode_cascade_impl(out, q, k_cache, v_cache, block_tables, max_blocks_per_seq,
                                   context_lens, seq_order, num_seqs, max_context_len,
                                   num_q_heads, num_kv_heads, head_dim, block_size, num_blocks,
                                   scale, 1.f, 1.f,
                                   group_members, group_prefix_blocks, seq_group, seq_member,
                                   num_groups, group_size, max_prefix_blocks, workspace,
                                   workspace_bytes, dev_error, dtype, dtype, stream);
}

int pa_paged_decode_cascade_fp8(void* out, const void* q, const void* k_cache,
                                const void* v_cache, const int32_t* block_tables,
                                int max_blocks_per_seq, const int32_t* context_lens,
                                const int32_t* seq_order, int num_seqs, int max_context_len,
                                int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                                int num_blocks, float scale,
                                float k_scale, float v_scale, const int32_t* group_members,
                                const int32_t* group_prefix_blocks, const int32_t* seq_group,
                                const int32_t* seq_member, int num_groups, int group_size,
                                int max_prefix_blocks, void* workspace, size_t workspace_bytes,
                                int* dev_error, int dtype, void* stream) {
  const NvtxRange nvtx_range("pa_paged_decode_cascade_fp8");
  clear_error();
  if (!positive_finite(k_scale) || !positive_finite(v_scale))
    return fail(PA_ERR_INVALID_ARG, "k_scale and v_scale must be finite and positive");
  return paged_decode_cascade_impl(out, q, k_cache, v_cache, block_tables, max_blocks_per_seq,
                                   context_lens, seq_order, num_seqs, max_context_len,
                                   num_q_heads, num_kv_heads, head_dim, block_size, num_blocks,
                                   scale, k_scale, v_scale, group_members, group_prefix_blocks,
                                   seq_group, seq_member, num_groups, group_size, max_prefix_blocks,
                                   workspace, workspace_bytes, dev_error, dtype, PA_FP8_E4M3,
                                   stream);
}

int pa_paged_decode(void* out, const void* q, const void* k_cache, const void* v_cache,
                    const int32_t* block_tables, int max_blocks_per_seq,
                    const int32_t* context_lens, const int32_t* seq_order, int num_seqs,
                    int max_context_len,
                    int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                    int num_blocks, float scale, int partition_tokens, void* workspace,
                    size_t workspace_bytes, int* dev_error, int dtype, void* stream) {
  const NvtxRange nvtx_range("pa_paged_decode");
  clear_error();
  return paged_decode_impl(out, q, k_cache, v_cache, block_tables, max_blocks_per_seq,
                           context_lens, seq_order, num_seqs, max_context_len, num_q_heads,
                           num_kv_heads, head_dim, block_size, num_blocks, scale, 1.f, 1.f,
                           partition_tokens, workspace, workspace_bytes, dev_error, dtype, dtype,
                           stream);
}

int pa_paged_decode_fp8(void* out, const void* q, const void* k_cache, const void* v_cache,
                        const int32_t* block_tables, int max_blocks_per_seq,
                        const int32_t* context_lens, const int32_t* seq_order, int num_seqs,
                        int max_context_len, int num_q_heads, int num_kv_heads, int head_dim,
                        int block_size, int num_blocks, float scale, float k_scale,
                        float v_scale, int partition_tokens, void* workspace,
                        size_t workspace_bytes, int* dev_error, int dtype, void* stream) {
  const NvtxRange nvtx_range("pa_paged_decode_fp8");
  clear_error();
  if (!positive_finite(k_scale) || !positive_finite(v_scale))
    return fail(PA_ERR_INVALID_ARG, "k_scale and v_scale must be finite and positive");
  return paged_decode_impl(out, q, k_cache, v_cache, block_tables, max_blocks_per_seq,
                           context_lens, seq_order, num_seqs, max_context_len, num_q_heads,
                           num_kv_heads, head_dim, block_size, num_blocks, scale, k_scale, v_scale,
                           partition_tokens, workspace, workspace_bytes, dev_error, dtype,
                           PA_FP8_E4M3, stream);
}

int pa_reshape_and_cache_fp8(const void* key, const void* value, int64_t key_token_stride,
                             int64_t value_token_stride, void* k_cache, void* v_cache,
                             const int64_t* slot_mapping, int num_tokens, int num_kv_heads,
                             int head_dim, int block_size, int num_blocks, int src_dtype,
                             float k_scale, float v_scale, int* dev_error, void* stream) {
  const NvtxRange nvtx_range("pa_reshape_and_cache_fp8");
  clear_error();
  if (int st = check_cache_shape(num_kv_heads, head_dim, block_size, num_blocks, src_dtype))
    return st;
  if (!positive_finite(k_scale) || !positive_finite(v_scale))
    return fail(PA_ERR_INVALID_ARG, "k_scale and v_scale must be finite and positive");
  if (num_tokens < 0) return fail(PA_ERR_INVALID_ARG, "num_tokens must be >= 0");
  if (num_tokens == 0) return PA_OK;
  if (!key || !value || !k_cache || !v_cache || !slot_mapping)
    return fail(PA_ERR_INVALID_ARG, "null pointer argument");
  const int64_t row = (int64_t)num_kv_heads * head_dim;
  if (key_token_stride < row || value_token_stride < row || key_token_stride % 8 ||
      value_token_stride % 8)
    return fail(PA_ERR_INVALID_ARG,
                "token strides (%lld, %lld) must be >= num_kv_heads*head_dim (%lld) and a "
                "multiple of 8",
                (long long)key_token_stride, (long long)value_token_stride, (long long)row);
  if (!aligned16(key) || !aligned16(value) || !aligned16(k_cache) || !aligned16(v_cache))
    return fail(PA_ERR_INVALID_ARG, "key, value and cache pointers must be 16-byte aligned");
  return cuda_status(
      launch_reshape_and_cache_fp8(key, value, key_token_stride, value_token_stride, k_cache,
                                   v_cache, slot_mapping, num_tokens, num_kv_heads, head_dim,
                                   num_blocks, src_dtype, k_scale, v_scale, dev_error,
                                   static_cast<cudaStream_t>(stream)),
      "reshape_and_cache_fp8 launch");
}

}  // extern "C"
