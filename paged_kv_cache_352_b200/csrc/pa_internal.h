// Internal declarations shared by libpa's translation units (host side).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "pa.h"

namespace pa {

constexpr int kBlockSize = 16;                 // tokens per cache block
// Default split-KV rule (partition_tokens == 0): partitions of at most
// kMaxPartitionBlocks blocks; shorter ones (down to kMinPartitionBlocks) when the
// batch has fewer than kSplitTargetUnits (sequence, KV head) pairs, so that the
// launch still has about that many CTAs (148 SMs x 3 resident CTAs x ~2.3 waves).
constexpr int kSplitTargetUnits = 1024;
constexpr int kMinPartitionBlocks = 32;
constexpr int kMaxPartitionBlocks = 128;
// With a longest-first seq_order the tail is short enough for longer partitions.
constexpr int kMaxPartitionBlocksOrdered = 256;
constexpr unsigned long long kWaitLimitNs = 1000000000ull;  // bounded on-chip waits: 1 s
constexpr int kMaxCopyPairsPerLaunch = 1024;   // pairs carried in one kernel parameter block

// Names the enclosing library call in profiler timelines (an NVTX range pushed
// on entry and popped on return). Without an attached profiler the calls are
// no-ops behind a function pointer.
struct NvtxRange {
  explicit NvtxRange(const char* name);
  ~NvtxRange();
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

// Launches `kernel` with programmatic stream serialization: it may start while
// the kernel ahead of it in the stream finishes, and waits for that kernel
// (grid_dependency_wait, first thing in every such kernel) before it reads any
// memory. Only the launch latency and the CTAs' start-up overlap.
template <typename... KArgs, typename... Args>
cudaError_t launch_dependent(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                             cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args&&>(args)...);
}

// Records a message for pa_last_error() and returns `code`.
int fail(int code, const char* fmt, ...);
void clear_error();

struct DecodeArgs {
  void* out;
  const void* q;
  const void* k_cache;
  const void* v_cache;
  const int32_t* block_tables;
  const int32_t* context_lens;
  const int32_t* seq_order;  // nullable: CTA z serves sequence seq_order[z]
  float* ws_m;       // [B][Hkv][max_parts][G]  running maximum (base 2) per partition
  float* ws_l;       // [B][Hkv][max_parts][G]  sum of exponentials per partition
  float* ws_acc;     // [B][Hkv][max_parts][G][D]  unnormalised partition outputs
  int* ws_count;     // [B][Hkv]  partitions finished (returned to 0 by the merging CTA)
  int* dev_error;
  int max_blocks_per_seq;
  int max_context_len;
  int num_seqs;
  int num_q_heads;
  int num_kv_heads;
  int num_blocks;
  int part_blocks;   // blocks per split-KV partition
  int max_parts;     // partitions per sequence the grid covers
  float scale_log2;  // softmax scale * log2(e) (* the key scale of an E4M3 cache)
  float out_scale;   // 1, or the value scale of an E4M3 cache
  int warp_parts;    // split mode: one warp per partition + a merge launch (else one CTA)
  int states_only;   // every partition leaves its state in the workspace; nothing writes
                     // `out` and no partitions are merged (a sequence with no blocks
                     // leaves no state): the caller merges them
  // Rows of shared-prefix groups (the cascade's prefix decode, one launch): when
  // grp_members is set, sequence index s names group s. Its table is the row of
  // its leader (member slot 0) in block_tables, its context the group's
  // grp_prefix_blocks[s] full blocks (none when the leader or that count is out
  // of range), and query row r of KV head kvh is head kvh * grp_heads + r %
  // grp_heads of member slot r / grp_heads in q ([grp_src_seqs][Hkv * grp_heads][D];
  // a zero row for an empty slot). Nothing is read that another kernel of the
  // same call writes, so these units do not wait for the kernel ahead.
  const int32_t* grp_members = nullptr;        // [num_seqs][grp_size], -1 pads
  const int32_t* grp_prefix_blocks = nullptr;  // [num_seqs]
  int grp_size = 0;
  int grp_heads = 0;
  int grp_src_seqs = 0;
  int grp_max_prefix_blocks = 0;
  // Failure-detection test hook (pa_test_stall_next_decode); both 0 in normal use.
  // stall_first_block: each warp arms the barrier of its first block without
  // issuing the block's copy, so that wait runs out; wait_limit_ns: the limit of
  // the main loop's waits (0 = kWaitLimitNs).
  unsigned long long wait_limit_ns = 0;
  int stall_first_block = 0;
};

// The wait limit a pending pa_test_stall_next_decode request asked for (0 when
// none); taking it clears the request, so it applies to one decode launch.
unsigned long long take_stall_request();
void set_stall_request(unsigned long long wait_limit_ns);

// Split partitions of at most this many blocks, for batches whose longest
// context spans at least 16 of them, run one warp per partition when that grid
// still has kSplitTargetUnits CTAs (PA_DECODE_SPLIT=cta|warp forces a mode).
constexpr int kWarpPartMaxBlocks = 64;
bool use_warp_parts(int num_seqs, int num_kv_heads, int part_blocks, int max_parts);

struct DecodeLayout {
  int part_blocks;
  int max_parts;
  size_t count_off, ml_off, acc_off, bytes;
};

// Workspace layout for a decode call (bytes == 0 when no sequence can split).
int decode_layout(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                  int max_context_len, int partition_tokens, bool ordered, DecodeLayout* lay);

// The cascade's decode over the groups' prefixes (`pre`, 8 stacked query heads
// per KV head, located through pre.grp_*) and over every sequence's own blocks
// (`own`, g_own query heads) as one launch; cudaErrorNotSupported for shapes
// without that form (cascade_single_launch is false for them), for which the two
// decodes are launched separately.
cudaError_t launch_cascade_decode(const DecodeArgs& pre, const DecodeArgs& own, int head_dim,
                                  int g_own, int dtype, int cache_dtype, cudaStream_t stream);
bool cascade_single_launch(int head_dim, int g_own, int stacked, int dtype, int cache_dtype);

// dtype: query/output type (PA_F16 or PA_BF16); cache_dtype: dtype or PA_FP8_E4M3.
cudaError_t launch_paged_decode(const DecodeArgs& a, int head_dim, int group, int dtype,
                                int cache_dtype, cudaStream_t stream);


cudaError_t launch_reshape_and_cache(const void* key, const void* value, int64_t key_stride,
                                     int64_t value_stride, void* k_cache, void* v_cache,
                                     const int64_t* slot_mapping, int num_tokens,
                                     int num_kv_heads, int head_dim, int num_blocks,
                                     int* dev_error, cudaStream_t stream);

// Quantizing write of 16-bit keys/values into E4M3 caches: code = E4M3(x / scale).
cudaError_t launch_reshape_and_cache_fp8(const void* key, const void* value, int64_t key_stride,
                                         int64_t value_stride, void* k_cache, void* v_cache,
                                         const int64_t* slot_mapping, int num_tokens,
                                         int num_kv_heads, int head_dim, int num_blocks,
                                         int src_dtype, float k_scale, float v_scale,
                                         int* dev_error, cudaStream_t stream);

// Cascade decode of sequences that share leading blocks: the prefix states of
// every group come from one decode over the shared blocks (the members' query
// heads stacked as one KV head's group), the rest of each sequence from its own
// blocks, and a merge combines the two.
struct CascadeArgs {
  const void* q;                       // [B][Hq][D]
  const int32_t* block_tables;         // [B][max_blocks]
  const int32_t* context_lens;         // [B]
  const int32_t* group_members;        // [num_groups][group_size], -1 pads
  const int32_t* group_prefix_blocks;  // [num_groups]
  const int32_t* seq_group;            // [B]: group of s, or -1
  const int32_t* seq_member;           // [B]: slot of s in its group
  void* gq;            // [num_groups][Hkv * group_size * Gh][D] stacked queries (written)
  int32_t* g_tables;   // [num_groups][max_blocks] leader's prefix entries, -1 after (written)
  int32_t* g_ctx;      // [num_groups] prefix tokens used, 0 for a rejected group (written)
  int32_t* s_tables;   // [B][max_blocks] each sequence's blocks after its prefix (written)
  int32_t* s_ctx;      // [B] tokens after the prefix (written)
  int32_t* s_pbase;    // [B] first prefix-state row of s (kvh 0, head 0), -1 if none (written)
  int32_t* s_np;       // [B] prefix partitions of s (written)
  const float* g_m;    // group decode states [num_groups][Hkv][g_parts][Gg] (+ [D] for acc)
  const float* g_l;
  const float* g_acc;
  const float* s_m;    // own-block decode states [B][Hkv][s_parts][Gh] (+ [D] for acc)
  const float* s_l;
  const float* s_acc;
  void* out;           // [B][Hq][D]
  int* dev_error;
  int num_seqs, num_groups, group_size, num_q_heads, num_kv_heads;
  int max_blocks_per_seq, max_prefix_blocks, max_context_len;
  int g_parts, g_part_blocks, s_parts, s_part_blocks;
  float out_scale;
};

cudaError_t launch_cascade_prepare(const CascadeArgs& c, int head_dim, bool stack_queries,
                                   cudaStream_t stream);
cudaError_t launch_cascade_merge(const CascadeArgs& c, int head_dim, int dtype,
                                 cudaStream_t stream);

struct CopyPairs {
  int32_t src[kMaxCopyPairsPerLaunch];
  int32_t dst[kMaxCopyPairsPerLaunch];
};

// Copies block pairs.src[i] of the source pool over block pairs.dst[i] of the
// destination pool (K and V); the pools may be the same (copy-on-write).
cudaError_t launch_copy_pool_blocks(const void* src_k, const void* src_v, void* dst_k,
                                    void* dst_v, const CopyPairs& pairs, int n,
                                    int64_t block_bytes, cudaStream_t stream);

}  // namespace pa
