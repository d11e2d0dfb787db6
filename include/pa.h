/*
 * pa.h — C interface of libpa, a paged KV cache and paged-decode attention for
 * NVIDIA B200 (sm_100a).
 *
 * The method (PagedAttention) keeps every sequence's attention keys and values
 * in fixed-size blocks of 16 tokens taken on demand from a pool allocated once
 * up front; a per-sequence block table maps logical blocks to physical ones, and
 * attention reads the cache through that table. Blocks can be shared between
 * sequences and are copied only when one of them writes (copy-on-write).
 * Sources: "PagedAttention and Continuous Batching" (roadtointelligence.com),
 * section "Pages, from operating systems"; "PagedAttention: The vLLM Paper"
 * (ai.zenoagi.com), sections "The Core Idea", "The OS paging analogy" and
 * "Implementation Essentials"; "vLLM: PagedAttention and continuous batching"
 * (llmstudy.shddai.net), direct answer. The pages define no programming
 * interface; the calls below are this library's.
 *
 * Conventions for every call
 *   - Return value: a pa_status (0 = PA_OK). On failure, pa_last_error() holds a
 *     message for the calling thread until its next libpa call.
 *   - Device calls (pa_reshape_and_cache, pa_copy_blocks, pa_swap_blocks,
 *     pa_paged_decode) take
 *     device pointers owned by the caller, enqueue kernels on the caller's CUDA
 *     stream (`stream` is a cudaStream_t; NULL = legacy default stream), never
 *     synchronise, never allocate device memory, and return after the launch.
 *     Scalar arguments are checked on the host before anything is launched; a
 *     failed check launches nothing. Data-dependent faults (a slot or block id
 *     outside the pool, a context longer than the table) are never trapped on the
 *     device: the offending access is skipped and a bit is OR-ed into *dev_error
 *     when dev_error is non-NULL (a device int the caller zeroes and reads back).
 *   - Supported shapes: block_size 16, head_dim 64 or 128, num_q_heads a
 *     multiple of num_kv_heads with a ratio of 1, 2, 4 or 8, fp16 or bf16 storage.
 *     Other shapes return PA_ERR_UNSUPPORTED.
 *   - Cache layout: two arrays, k_cache and v_cache, each
 *     [num_blocks][num_kv_heads][block_size][head_dim] row-major in the storage
 *     type; slot s is offset s % block_size of block s / block_size. Base
 *     pointers must be 16-byte aligned.
 *   - Host block-manager calls (pa_bm_*) are all-or-nothing: on failure the
 *     manager's state is unchanged. A manager is not thread-safe.
 */
#ifndef PA_H_
#define PA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum pa_status {
  PA_OK = 0,
  PA_ERR_INVALID_ARG = 1,    /* bad pointer, size or value */
  PA_ERR_NO_FREE_BLOCKS = 2, /* the pool cannot cover the request */
  PA_ERR_UNKNOWN_SEQ = 3,    /* sequence id not registered */
  PA_ERR_CUDA = 4,           /* a CUDA runtime call failed */
  PA_ERR_UNSUPPORTED = 5,    /* shape or type outside the supported set */
  PA_ERR_SEQ_EXISTS = 6,     /* sequence id already registered */
  PA_ERR_SEQ_SWAPPED = 7     /* sequence is swapped out (or, for swap-in, is not) */
} pa_status;

/* PA_FP8_E4M3 is a cache element type only: pa_reshape_and_cache_fp8 writes it,
 * pa_paged_decode_fp8 reads it, pa_copy_blocks and pa_swap_blocks move it (one
 * byte per element). Queries, outputs and the 16-bit inputs of the cache write
 * are PA_F16 or PA_BF16. */
typedef enum pa_dtype { PA_F16 = 0, PA_BF16 = 1, PA_FP8_E4M3 = 2 } pa_dtype;

/* Bits OR-ed into *dev_error by device calls. */
#define PA_DEVERR_SLOT_RANGE 1    /* slot >= num_blocks * block_size: token not written */
#define PA_DEVERR_BLOCK_RANGE 2   /* block-table entry outside [0, num_blocks): block skipped */
#define PA_DEVERR_CONTEXT_RANGE 4 /* context_lens[s] < 0, > max_blocks_per_seq*block_size,
                                     or > max_context_len: sequence skipped (zero output) */
#define PA_DEVERR_WAIT_TIMEOUT 8  /* a bounded on-chip wait gave up: output invalid */
#define PA_DEVERR_GROUP 16        /* a cascade group descriptor was rejected (a member that
                                     does not hold the group's prefix blocks, an id out of
                                     range, a member claimed twice): that group's members
                                     were decoded without the shared prefix; outputs stay
                                     correct */

/* Message for the last failed call on this thread ("" if none). */
const char* pa_last_error(void);

/* Library interface version (major * 100 + minor). */
int pa_version(void);

/* ---------------------------------------------------------------------------
 * pa_test_stall_next_decode — test hook for the device-side failure path.
 *
 * The pages tie failure handling to memory running short ("PagedAttention: The
 * vLLM Paper", "Implementation Essentials", preemption); on the device, every
 * on-chip wait of the decode kernels is bounded and gives up with
 * PA_DEVERR_WAIT_TIMEOUT instead of spinning. This call lets a test drive that
 * path without a fault: the next decode kernel launch in the process (by any
 * pa_paged_decode* call; for pa_paged_decode_cascade* the launch that decodes
 * the shared and the own blocks) has each warp arm the barrier of its first block
 * without issuing the block's copy, and lowers the limit of the main loop's
 * waits to wait_limit_ns. That wait runs out, the warp reports
 * PA_DEVERR_WAIT_TIMEOUT, still waits (with the normal 1 s limit) for the
 * copies it did issue, and the kernel returns; that launch's output is invalid.
 * The request applies to one launch and is then cleared.
 *
 *   wait_limit_ns   in [1000, 1e8] (1 us .. 100 ms), else PA_ERR_INVALID_ARG
 *
 * Not for production use: it exists so that tests can check the error path.
 * ------------------------------------------------------------------------- */
int pa_test_stall_next_decode(unsigned long long wait_limit_ns);

/* ---------------------------------------------------------------------------
 * pa_reshape_and_cache — store new tokens' keys and values in their slots.
 *
 * Every generated token's K/V is cached so decode need not recompute it
 * ("PagedAttention: The vLLM Paper", "Background and Motivation"), and blocks
 * are filled as tokens arrive ("PagedAttention and Continuous Batching",
 * "Pages, from operating systems"). For each token t with slot_mapping[t] >= 0:
 *   k_cache[slot / bs][h][slot % bs][:] = key[t][h][:]   for every KV head h,
 * and likewise for value / v_cache. slot_mapping[t] < 0 skips token t.
 *
 *   key, value        device, [num_tokens][num_kv_heads][head_dim] with a token
 *                     stride of key_token_stride / value_token_stride elements
 *                     (>= num_kv_heads*head_dim, a multiple of 8); 16-byte aligned
 *   k_cache, v_cache  device, cache layout above; written in place
 *   slot_mapping      device, int64 [num_tokens]
 *   dev_error         device int or NULL (PA_DEVERR_SLOT_RANGE)
 * Slots must be distinct among the tokens of one call (which write wins is
 * otherwise unspecified). num_tokens == 0 is a no-op.
 * ------------------------------------------------------------------------- */
int pa_reshape_and_cache(const void* key, const void* value, int64_t key_token_stride,
                         int64_t value_token_stride, void* k_cache, void* v_cache,
                         const int64_t* slot_mapping, int num_tokens, int num_kv_heads,
                         int head_dim, int block_size, int num_blocks, int dtype,
                         int* dev_error, void* stream);

/* ---------------------------------------------------------------------------
 * pa_copy_blocks — the copy half of copy-on-write.
 *
 * A block shared by several sequences is copied only when one of them must
 * modify it ("PagedAttention and Continuous Batching", "Pages, from operating
 * systems"; "PagedAttention: The vLLM Paper", "The OS paging analogy", page
 * sharing). For each pair i: block pairs[2i+1] of k_cache and of v_cache
 * becomes a copy of block pairs[2i] (all KV heads, all 16 slots).
 *
 *   pairs   HOST array, int64 [num_pairs][2] = (src, dst); read before return.
 *           Every id in [0, num_blocks); dst ids distinct; no dst equal to any
 *           src of the same call (so the copies are independent). Violations
 *           return PA_ERR_INVALID_ARG and launch nothing.
 * The pairs travel in the kernel's parameter block: no device buffer is needed.
 * num_pairs == 0 is a no-op. dtype PA_FP8_E4M3 copies 8-bit caches.
 * ------------------------------------------------------------------------- */
int pa_copy_blocks(void* k_cache, void* v_cache, const int64_t* pairs, int num_pairs,
                   int num_kv_heads, int head_dim, int block_size, int num_blocks, int dtype,
                   void* stream);

/* ---------------------------------------------------------------------------
 * pa_swap_blocks — move whole blocks between two pools: the device pool and a
 * pool of pinned host memory, for preemption by swapping.
 *
 * When memory runs short a low-priority request's blocks are swapped to CPU
 * memory and brought back later ("PagedAttention: The vLLM Paper",
 * "Implementation Essentials"; "The OS paging analogy", swapping). For each
 * pair i: block pairs[2i+1] of the destination pool (K and V) becomes a copy of
 * block pairs[2i] of the source pool. pa_bm_swap_out / pa_bm_swap_in emit the
 * pairs.
 *
 *   src_k, src_v / dst_k, dst_v   pools in the cache layout above with
 *                 src_num_blocks / dst_num_blocks blocks. Each is device memory
 *                 or pinned host memory the GPU can address (cudaHostAlloc /
 *                 cudaHostRegister); pageable host memory is refused. Source and
 *                 destination must be different pools.
 *   pairs         HOST int64 [num_pairs][2] = (src block, dst block); ids in
 *                 range of their pools and destination ids distinct, else
 *                 PA_ERR_INVALID_ARG and nothing is launched.
 * The copy runs on `stream`; after a swap-out, it must run before the freed
 * device blocks are written again (enqueue it first on the same stream).
 * ------------------------------------------------------------------------- */
int pa_swap_blocks(const void* src_k, const void* src_v, int src_num_blocks, void* dst_k,
                   void* dst_v, int dst_num_blocks, const int64_t* pairs, int num_pairs,
                   int num_kv_heads, int head_dim, int block_size, int dtype, void* stream);

/* ---------------------------------------------------------------------------
 * 8-bit KV cache: pa_reshape_and_cache_fp8 and pa_paged_decode_fp8.
 *
 * Quantizing the KV cache shrinks the bytes a bandwidth-bound decode reads
 * ("PagedAttention: The vLLM Paper", "Impact and Follow-Ups" and "Limitations");
 * the pages fix no format. Format taken: OCP FP8 E4M3 (bias 7, no infinities,
 * largest finite 448, codes 0x7F / 0xFF NaN), one scale per cache tensor.
 * Caches are uint8 arrays in the layout above ([num_blocks][Hkv][16][d], one
 * byte per element); copy and swap them with dtype PA_FP8_E4M3.
 *
 * pa_reshape_and_cache_fp8: as pa_reshape_and_cache, but element x of key
 * (value) is stored as the E4M3 code nearest to float32(x) / k_scale
 * (v_scale), the division rounded to nearest in fp32, ties of the conversion
 * to the even code, magnitudes past 448 saturating to 448, the sign kept.
 * src_dtype is the type of key/value (PA_F16 or PA_BF16). k_scale and v_scale
 * must be finite and positive (else PA_ERR_INVALID_ARG).
 *
 * pa_paged_decode_fp8: as pa_paged_decode over E4M3 caches, attending to the
 * dequantized keys code * k_scale and values code * v_scale; q and out are of
 * type dtype (PA_F16 or PA_BF16). The workspace is sized by
 * pa_paged_decode_workspace_size exactly as for pa_paged_decode.
 * ------------------------------------------------------------------------- */
int pa_reshape_and_cache_fp8(const void* key, const void* value, int64_t key_token_stride,
                             int64_t value_token_stride, void* k_cache, void* v_cache,
                             const int64_t* slot_mapping, int num_tokens, int num_kv_heads,
                             int head_dim, int block_size, int num_blocks, int src_dtype,
                             float k_scale, float v_scale, int* dev_error, void* stream);

int pa_paged_decode_fp8(void* out, const void* q, const void* k_cache, const void* v_cache,
                        const int32_t* block_tables, int max_blocks_per_seq,
                        const int32_t* context_lens, const int32_t* seq_order, int num_seqs,
                        int max_context_len, int num_q_heads, int num_kv_heads, int head_dim,
                        int block_size, int num_blocks, float scale, float k_scale,
                        float v_scale, int partition_tokens, void* workspace,
                        size_t workspace_bytes, int* dev_error, int dtype, void* stream);

/* ---------------------------------------------------------------------------
 * pa_paged_decode — decode-step attention through the block tables.
 *
 * Attention follows the block-table mapping, reading the cache where it lies
 * ("vLLM: PagedAttention and continuous batching", direct answer; "PagedAttention:
 * The vLLM Paper", "The Core Idea", the note under the block-table figure). For
 * sequence s and query head h, with G = num_q_heads / num_kv_heads and
 * g = h / G:
 *   K_s[t] = k_cache[block_tables[s][t / bs]][g][t % bs][:]   t < context_lens[s]
 *   out[s][h] = softmax(scale * K_s q[s][h]) V_s
 * computed in fp32 (online softmax) and rounded to the storage type (nearest
 * even). A zero-length context gives a zero row. Long contexts are cut into
 * partitions of `partition_tokens` tokens processed in parallel and merged by
 * log-sum-exp rescaling inside the same kernel launch (split-KV).
 *
 *   out                device, [num_seqs][num_q_heads][head_dim], storage type
 *   q                  device, [num_seqs][num_q_heads][head_dim], storage type
 *   k_cache, v_cache   device, cache layout above (read only)
 *   block_tables       device, int32 [num_seqs][max_blocks_per_seq], padded with -1
 *   context_lens       device, int32 [num_seqs], tokens per sequence including the
 *                      token written this step
 *   seq_order          device, int32 [num_seqs], a permutation of 0..num_seqs-1
 *                      giving the order in which sequences are scheduled, or
 *                      NULL for 0, 1, 2, ... Listing the sequences longest first
 *                      (pa_longest_first_order) keeps long sequences from
 *                      finishing last and shortens the launch's tail; sequences
 *                      that share blocks are best kept next to each other, so
 *                      the shared blocks are read while still in L2. Results
 *                      do not depend on the order. Entries outside
 *                      [0, num_seqs) are flagged (PA_DEVERR_CONTEXT_RANGE) and
 *                      skipped; a repeated entry leaves some sequence unwritten.
 *   max_context_len    host-known upper bound of context_lens (sizes the grid
 *                      without a device read); longer sequences are flagged
 *   scale              softmax scale, usually 1/sqrt(head_dim)
 *   partition_tokens   a multiple of block_size, or 0 for the library's choice:
 *                      partitions of at most 2048 tokens (4096 when seq_order is
 *                      given), shorter (down to 512) when num_seqs *
 *                      num_kv_heads < 1024, so that the launch still has ~1024
 *                      (sequence, KV head, partition) units
 *   workspace          device scratch of pa_paged_decode_workspace_size() bytes,
 *                      ZERO-FILLED before its first use; every completed call
 *                      leaves it zero-filled again, so it can be reused without
 *                      clearing. Calls that run concurrently need separate
 *                      workspaces. May be NULL when the size is 0. After a call
 *                      that reported PA_DEVERR_WAIT_TIMEOUT, zero it again.
 *   dev_error          device int or NULL
 * Reduction order depends only on logical token positions, so results are
 * bit-identical whatever the physical placement of blocks and whether blocks
 * are shared or duplicated.
 * ------------------------------------------------------------------------- */
/* Workspace bytes pa_paged_decode needs for these sizes (enough with or
 * without a seq_order). */
int pa_paged_decode_workspace_size(int num_seqs, int num_q_heads, int num_kv_heads,
                                   int head_dim, int max_context_len, int block_size,
                                   int partition_tokens, size_t* bytes);

/* The split-KV plan pa_paged_decode (or pa_paged_decode_fp8) would use for these
 * arguments (ordered != 0: a seq_order is passed): blocks per partition, the
 * partitions per sequence the grid covers, and the kernel launches the call
 * makes (1; 2 when short partitions run one warp per partition followed by a
 * merge launch; 0 for an empty batch). The split mode itself is not observable
 * in the results beyond floating-point rounding order. */
int pa_paged_decode_plan(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                         int max_context_len, int block_size, int partition_tokens, int ordered,
                         int* part_blocks, int* max_parts, int* launches);

/* Host helper: order[0..n) = sequence indices by decreasing context_lens (ties
 * by index), the recommended seq_order. Both arrays are host memory. */
int pa_longest_first_order(const int32_t* context_lens, int n, int32_t* order);

/* The plan pa_paged_decode_cascade (fp8_cache == 0) or pa_paged_decode_cascade_fp8
 * (fp8_cache != 0) would follow for these host bounds, which are those of
 * pa_paged_decode_cascade_workspace_size; dtype is the query type (PA_F16 or
 * PA_BF16). Outputs: blocks per partition and partitions of a group's shared
 * prefix (0 and 0 when num_groups is 0), blocks per partition and partitions
 * of a sequence's own blocks, and the kernel launches the call makes: 3
 * (prepare, both decodes in one launch, merge; also with no groups), 4 when the
 * two decodes run on two streams (fewer than 8 stacked query heads per KV
 * head), 0 for an empty batch. Prefixes are split below the decode's
 * partition cap only when groups and sequences together give fewer than about
 * 1024 (group or sequence, KV head) pairs. Host only; nothing is launched.
 * Returns PA_ERR_INVALID_ARG / PA_ERR_UNSUPPORTED for the shapes the cascade
 * refuses. */
int pa_paged_decode_cascade_plan(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                                 int max_context_len, int max_blocks_per_seq, int block_size,
                                 int num_groups, int group_size, int max_prefix_blocks, int dtype,
                                 int fp8_cache, int* prefix_part_blocks, int* prefix_parts,
                                 int* own_part_blocks, int* own_parts, int* launches);

/* Host helper for pa_paged_decode_cascade: order[0..n) = sequence indices by
 * decreasing tokens after their group's prefix (context_lens[i] -
 * block_size * group_prefix_blocks[seq_group[i]] for a sequence in a group,
 * context_lens[i] otherwise; ties by index), the recommended seq_order. All
 * arrays are host memory, as pa_bm_prefix_groups writes them; seq_group and
 * group_prefix_blocks may be NULL when num_groups is 0. */
int pa_cascade_order(const int32_t* context_lens, const int32_t* seq_group,
                     const int32_t* group_prefix_blocks, int num_groups, int n, int32_t* order);

int pa_paged_decode(void* out, const void* q, const void* k_cache, const void* v_cache,
                    const int32_t* block_tables, int max_blocks_per_seq,
                    const int32_t* context_lens, const int32_t* seq_order, int num_seqs,
                    int max_context_len,
                    int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                    int num_blocks, float scale, int partition_tokens, void* workspace,
                    size_t workspace_bytes, int* dev_error, int dtype, void* stream);

/* ---------------------------------------------------------------------------
 * pa_paged_decode_noalloc — pa_paged_decode without a caller-supplied workspace.
 *
 * The paper has no counterpart to this call. It is a convenience of this
 * library for callers that cannot allocate device memory: for example a plugin
 * whose host runtime owns every allocation, or a latency-critical loop that must
 * never reach cudaMalloc, which may synchronise the device.
 *
 * The result is the same as pa_paged_decode with the same arguments. The
 * split-KV scratch comes from one array of PA_NOALLOC_WORKSPACE_BYTES compiled
 * into the library. Every GPU that loads the library holds that array until the
 * process exits.
 *
 * The call allocates nothing:
 *   - The first call on each device looks up the array's device address and
 *     caches it with the id of the device's current context. A call that finds
 *     another context current (after cudaDeviceReset, for example) looks the
 *     address up again, since a new context holds the array elsewhere. Make the
 *     first call on a device, and the first after a reset, with the device
 *     current and before any stream capture on that device.
 *   - The call runs on the current device. out, q, both caches, the tables and
 *     the lengths must be device memory of that device and `stream` one of its
 *     streams; otherwise it returns PA_ERR_INVALID_ARG and launches nothing.
 *   - Each call clears the array's merge counters with an async memset on
 *     `stream`, then launches the decode kernel.
 *   - All calls share the one array, so calls whose kernels overlap on the GPU
 *     race. Issue them on one stream or order them with events.
 *   - A batch whose scratch (pa_paged_decode_workspace_size) exceeds the array
 *     returns PA_ERR_UNSUPPORTED and launches nothing. A larger partition_tokens,
 *     or fewer sequences per call, reduces the scratch needed.
 * ------------------------------------------------------------------------- */
#define PA_NOALLOC_WORKSPACE_BYTES ((size_t)16 << 20) /* 16 MiB */

int pa_paged_decode_noalloc(void* out, const void* q, const void* k_cache, const void* v_cache,
                            const int32_t* block_tables, int max_blocks_per_seq,
                            const int32_t* context_lens, const int32_t* seq_order, int num_seqs,
                            int max_context_len,
                            int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                            int num_blocks, float scale, int partition_tokens, int* dev_error,
                            int dtype, void* stream);

/* ---------------------------------------------------------------------------
 * pa_paged_decode_cascade — paged decode that reads blocks shared by several
 * sequences once.
 *
 * Forks of one prompt hold the same physical blocks for the prompt's full
 * blocks ("PagedAttention and Continuous Batching", "Pages, from operating
 * systems": copy-on-write sharing; "PagedAttention: The vLLM Paper",
 * "Implementation Essentials": prefix sharing). pa_paged_decode reads such a
 * block once per sequence; this call reads it once per group:
 *   1. a prepare kernel checks each group and writes every sequence's table of
 *      the blocks after its prefix (and, for the two-launch form below, the
 *      group's prefix table and its members' stacked query heads);
 *   2. a decode over the groups' prefix blocks (group_size * G query heads per
 *      KV head: the members' heads stacked as one KV head's query group),
 *      leaving its partition states in the workspace;
 *   3. a decode over every sequence's remaining blocks, likewise;
 *   4. a merge of the two sets of softmax states per output row.
 * When group_size * G is 8 and G < 8, steps 2 and 3 are one launch whose
 * prefix CTAs come first and read the leader's table and the members' query
 * rows in place: they start while step 1 runs. Otherwise step 2 runs on a
 * second stream of the library's, beside step 3 on `stream`, forked after
 * step 1 and joined before step 4 by events; the library makes that stream and
 * its two events on a host thread's first such call on a device and keeps them
 * for the life of the process. Either way the call is ordered on `stream` like
 * any other.
 * The result is the decode of pa_paged_decode up to floating-point rounding
 * (the same fp32 arithmetic summed in another order).
 *
 * Arguments as for pa_paged_decode (no partition_tokens: both decodes use the
 * library's default split), plus the group descriptor, in device memory, as
 * pa_bm_prefix_groups writes it:
 *   seq_order            device, int32 [num_seqs], a permutation of
 *                        0..num_seqs-1 giving the order in which the
 *                        remaining-block decode schedules sequences, or NULL
 *                        for 0, 1, 2, ...; pa_cascade_order lists them by
 *                        decreasing length after their prefix, which shortens
 *                        the launch's tail. Results do not depend on the order;
 *                        entries outside [0, num_seqs) are flagged
 *                        (PA_DEVERR_CONTEXT_RANGE) and skipped, and a repeated
 *                        entry leaves some sequence's output undefined.
 *   group_members        int32 [num_groups][group_size], batch indices, -1 pads;
 *                        slot 0 is the group's leader
 *   group_prefix_blocks  int32 [num_groups]: blocks shared by every member
 *   seq_group, seq_member int32 [num_seqs]: each sequence's group and slot, or -1
 *   num_groups, group_size, max_prefix_blocks: host bounds (grid and workspace
 *                        sizing); group_size * (num_q_heads / num_kv_heads) must
 *                        be 1, 2, 4 or 8, max_prefix_blocks >= every prefix
 *   workspace            device, 256-byte aligned, at least
 *                        pa_paged_decode_cascade_workspace_size bytes; fully
 *                        rewritten by each call (no clearing needed)
 * A sequence belongs to a group only if group_members[seq_group[s]][seq_member[s]]
 * names s. A group whose members do not all hold the leader's first prefix
 * blocks as full blocks inside their contexts, or whose descriptor is otherwise
 * inconsistent, is decoded without its prefix (every member over its whole
 * context) and PA_DEVERR_GROUP is set: the outputs stay correct (other bits
 * may be set too, e.g. PA_DEVERR_BLOCK_RANGE when the claimed prefix runs past
 * the leader's table). Host-side errors as for pa_paged_decode.
 * pa_paged_decode_cascade_fp8 decodes E4M3 caches with key and value scales,
 * as pa_paged_decode_fp8.
 * ------------------------------------------------------------------------- */
int pa_paged_decode_cascade_workspace_size(int num_seqs, int num_q_heads, int num_kv_heads,
                                           int head_dim, int max_context_len,
                                           int max_blocks_per_seq, int block_size, int num_groups,
                                           int group_size, int max_prefix_blocks, size_t* bytes);

int pa_paged_decode_cascade(void* out, const void* q, const void* k_cache, const void* v_cache,
                            const int32_t* block_tables, int max_blocks_per_seq,
                            const int32_t* context_lens, const int32_t* seq_order,
                            int num_seqs, int max_context_len, int num_q_heads,
                            int num_kv_heads, int head_dim, int block_size, int num_blocks,
                            float scale, const int32_t* group_members,
                            const int32_t* group_prefix_blocks, const int32_t* seq_group,
                            const int32_t* seq_member, int num_groups, int group_size,
                            int max_prefix_blocks, void* workspace, size_t workspace_bytes,
                            int* dev_error, int dtype, void* stream);

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
                                int* dev_error, int dtype, void* stream);

/* ---------------------------------------------------------------------------
 * Host block manager.
 *
 * The pool is allocated once; blocks are handed out and taken back, and a
 * reference count per block lets sequences share it ("PagedAttention: The vLLM
 * Paper", "Implementation Essentials"); blocks are taken on demand and only the last
 * block of a sequence may be partly filled ("The design yields three immediate
 * wins", item 1); parallel samples share the prompt's blocks (item 3 and
 * "Implementation Essentials", prefix sharing).
 *
 * Rules the pages leave open, fixed here:
 *   - The free list is a stack: initial_free_order[0] is handed out first;
 *     released blocks go on top. NULL initial_free_order = 0, 1, 2, ...
 *   - pa_bm_free_seq releases a sequence's blocks from its last logical block
 *     to its first; a block returns to the free list when its refcount hits 0.
 *   - pa_bm_append_slots: when the first appended token falls in a partly
 *     filled last block whose refcount is > 1, the sequence gets a fresh block,
 *     (old, new) is written to cow_pairs_out and old's refcount drops by one.
 *     The caller must run pa_copy_blocks on those pairs before writing the
 *     appended tokens. At most one pair per call.
 * Slots are block * block_size + offset (the slot_mapping of
 * pa_reshape_and_cache). Sequence ids are arbitrary int64 values.
 * ------------------------------------------------------------------------- */
typedef struct pa_bm pa_bm;

int pa_bm_create(int num_blocks, int block_size, const int32_t* initial_free_order,
                 pa_bm** out);
void pa_bm_destroy(pa_bm* bm);

/* Register seq_id holding num_tokens tokens; their slots go to slots_out[num_tokens]
 * (may be NULL when num_tokens == 0). */
int pa_bm_add_seq(pa_bm* bm, int64_t seq_id, int num_tokens, int64_t* slots_out);

/* child shares every block of parent (refcounts + 1). */
int pa_bm_fork(pa_bm* bm, int64_t parent, int64_t child);

/* Append n tokens to seq_id: slots_out[n]; cow_pairs_out[2] receives at most one
 * (src, dst) pair and *n_cow its count (0 or 1). */
int pa_bm_append_slots(pa_bm* bm, int64_t seq_id, int n, int64_t* slots_out,
                       int64_t* cow_pairs_out, int* n_cow);

int pa_bm_free_seq(pa_bm* bm, int64_t seq_id);

/* Tables of seq_ids[0..n) into out[n][max_blocks], padded with -1;
 * PA_ERR_INVALID_ARG if a table is longer than max_blocks. */
int pa_bm_block_tables(const pa_bm* bm, const int64_t* seq_ids, int n, int32_t* out,
                       int max_blocks);

/* Groups of the batch seq_ids[0..n) that hold the same leading blocks, for
 * pa_paged_decode_cascade. Members are batch indices (rows of the block tables).
 * Rule: sequences with at least one full block are bucketed by their first
 * block id (buckets in order of first appearance, members in batch order); each
 * bucket is cut into runs of group_size; a run of two or more becomes a group
 * whose prefix is the longest run of leading block ids the members all share
 * and all hold full (at most each member's length / block_size). Outputs:
 * group_members[n][group_size] (-1 pads), group_prefix_blocks[n], seq_group[n]
 * (group of each batch index or -1) and seq_member[n] (its slot, -1 if none);
 * *num_groups and *max_prefix_blocks (0 when there is no group). Swapped or
 * unknown sequences are refused and nothing is written. */
int pa_bm_prefix_groups(const pa_bm* bm, const int64_t* seq_ids, int n, int group_size,
                        int32_t* group_members, int32_t* group_prefix_blocks, int32_t* seq_group,
                        int32_t* seq_member, int* num_groups, int* max_prefix_blocks);

/* Swapping. pa_bm_set_host_pool sizes the host pool (host blocks 0..n-1, handed
 * out 0 first; refused while any sequence is swapped out). pa_bm_swap_out moves
 * seq_id's blocks to host blocks: pairs_out[capacity][2] receives one
 * (device block, host block) pair per block in logical order and *n_pairs their
 * count; device refcounts drop by one and blocks reaching zero return to the
 * free list, last logical block first. A block still shared with resident
 * sequences stays on the device for them. pa_bm_swap_in reverses it with
 * (host block, device block) pairs. While swapped, the sequence cannot append,
 * fork or appear in block tables (PA_ERR_SEQ_SWAPPED); pa_bm_free_seq releases
 * its host blocks. Both calls are all-or-nothing (PA_ERR_NO_FREE_BLOCKS when
 * the target pool is short). */
int pa_bm_set_host_pool(pa_bm* bm, int num_host_blocks);
int pa_bm_swap_out(pa_bm* bm, int64_t seq_id, int64_t* pairs_out, int capacity, int* n_pairs);
int pa_bm_swap_in(pa_bm* bm, int64_t seq_id, int64_t* pairs_out, int capacity, int* n_pairs);
/* 1 if swapped out, 0 if resident, -1 for an unknown sequence. */
int pa_bm_is_swapped(const pa_bm* bm, int64_t seq_id);
int pa_bm_num_free_host(const pa_bm* bm);
/* Free host blocks in hand-out order into out[capacity]; returns the count or -1. */
int pa_bm_host_free_list(const pa_bm* bm, int32_t* out, int capacity);

/* Prefix caching across requests: the KV of shared prompt prefixes is kept and
 * reused by later requests, so a hit makes prefill nearly free
 * ("PagedAttention: The vLLM Paper", "Impact and Follow-Ups", item 1).
 * pa_bm_add_seq_cached registers seq_id from its prompt's token_ids. Every full
 * block of the prompt is identified exactly by (physical block of the previous
 * logical block or -1, its block_size token ids); the leading full blocks found
 * in the cache are shared (refcount + 1), the rest get fresh blocks, and the new
 * full blocks join the cache. The partly filled last block is never cached, so
 * no write ever touches a cached block. slots_out[num_tokens] receives every
 * token's slot; *num_cached_tokens = the leading tokens whose keys and values
 * are already in the pool (only the rest need pa_reshape_and_cache).
 * A cached block whose refcount falls to 0 is kept for reuse on a queue, least
 * recently released first, and counts as free; blocks are taken from the free
 * list first, then by evicting the queue's head (with any cached descendants).
 * All-or-nothing like the other calls. */
int pa_bm_add_seq_cached(pa_bm* bm, int64_t seq_id, const int32_t* token_ids, int num_tokens,
                         int64_t* slots_out, int* num_cached_tokens);
/* Read-only look-up for admission decisions: *hit_blocks = the leading full
 * blocks of these prompt tokens found in the cache (what pa_bm_add_seq_cached
 * would share), *revived_blocks = how many of those are held by no sequence
 * (counted in pa_bm_num_free, so sharing them uses up free blocks). */
int pa_bm_cached_prefix(const pa_bm* bm, const int32_t* token_ids, int num_tokens,
                        int* hit_blocks, int* revived_blocks);
int pa_bm_num_cached(const pa_bm* bm);
/* Evictable cached blocks, oldest first, into out[capacity]; returns the count or -1. */
int pa_bm_evictable_list(const pa_bm* bm, int32_t* out, int capacity);

/* Queries. pa_bm_refcount and pa_bm_seq_len return -1 for an unknown block or
 * sequence (and set pa_last_error). pa_bm_num_free counts free blocks plus cached
 * blocks kept for reuse. */
int pa_bm_num_free(const pa_bm* bm);
int pa_bm_refcount(const pa_bm* bm, int32_t block);
int pa_bm_seq_len(const pa_bm* bm, int64_t seq_id);
int pa_bm_num_seqs(const pa_bm* bm);
/* Free blocks in hand-out order into out[capacity]; returns the count written or -1. */
int pa_bm_free_list(const pa_bm* bm, int32_t* out, int capacity);

/* ---------------------------------------------------------------------------
 * Continuous (iteration-level) batching: a scheduler over the block manager and
 * an executor that runs one planned step through the kernels above.
 *
 * Requests join and leave the batch at every decoding step instead of waiting
 * for a whole batch to finish ("PagedAttention and Continuous Batching", "Batch
 * by step, not by request"; "PagedAttention: The vLLM Paper", "Continuous
 * Batching: Request-Level vs. Iteration-Level Scheduling"); when the pool runs
 * short a request is preempted by swapping its blocks to host memory or by
 * dropping them for recomputation ("Implementation Essentials", block manager);
 * parallel samples of one prompt share its blocks (same section, prefix sharing).
 *
 * A request is (request_id >= 0, prompt_len >= 1, output_len >= 1,
 * 1 <= num_samples <= PA_SCHED_MAX_SAMPLES, arrival_step). There is no model:
 * every sample generates exactly output_len tokens, one per step, and the keys,
 * values and queries of the tokens are the caller's inputs. Sample s of request
 * r is block-manager sequence r * PA_SCHED_MAX_SAMPLES + s.
 *
 * pa_sched_step plans one step, in this order (rules the pages leave open):
 *   1. requests that finished in the previous step are freed;
 *   2. running requests, oldest admission first, append one token per sample.
 *      Before a request appends, the blocks its appends take (one per sample
 *      whose last block is full, one per copy-on-write of a shared partly
 *      filled block) are checked against the free count; while short, the
 *      newest running request is preempted (the request itself if it is the
 *      newest). Preemption swaps every sample out when the host pool has room
 *      for a copy of each sample's table, else drops a one-sample request for
 *      recomputation (it rejoins the waiting queue in arrival order, and on
 *      readmission its prompt and generated tokens are written again); a
 *      many-sample request that cannot be swapped makes the step fail;
 *   3. if nothing was preempted in this step: swapped requests resume in
 *      arrival order while the batch (max_num_seqs sequences) and the pool
 *      have room for them and their appends;
 *   4. if nothing was preempted and nothing is swapped out: waiting requests
 *      whose arrival_step has come are admitted in arrival order (arrival_step,
 *      then submission order), stopping at the first that does not fit. The
 *      prompt is registered for sample 0, samples 1.. fork it.
 *   Resumed and admitted requests append in the same step. The decode batch is
 *   every running sample, in running order then sample order, each with its
 *   new token in its context. A request whose samples have generated
 *   output_len tokens finishes with this step.
 *
 * Device order of a step (pa_sched_execute): swap-out pairs (device -> host),
 * swap-in pairs (host -> device), prefill writes (prompts and recomputed
 * tokens of admitted requests), copy-on-write pairs, new-token writes, decode.
 * ------------------------------------------------------------------------- */
#define PA_SCHED_MAX_SAMPLES 64
#define PA_PREEMPT_SWAP 0
#define PA_PREEMPT_RECOMPUTE 1

typedef struct pa_sched pa_sched;

/* Counts of the last planned step. */
typedef struct {
  int64_t step;            /* 0 for the first step */
  int num_finished;        /* requests freed at the start of the step */
  int num_preempted;
  int num_resumed;
  int num_admitted;
  int num_swap_out;        /* (device block, host block) pairs */
  int num_swap_in;         /* (host block, device block) pairs */
  int num_copies;          /* copy-on-write (src, dst) pairs */
  int num_prefill;         /* tokens written before the copies */
  int num_writes;          /* new tokens written after the copies */
  int num_seqs;            /* decode batch */
  int max_blocks_per_seq;  /* widest block table in the batch (>= 1) */
  int max_context_len;
  int64_t total_context;   /* sum of the batch's context lengths (tokens decode reads) */
  int64_t num_cached_tokens;  /* prompt tokens of admitted requests found in the prefix cache */
} pa_sched_plan;

/* num_blocks / block_size / initial_free_order as pa_bm_create. max_num_seqs
 * caps the decode batch (sequences). num_host_blocks sizes the host pool used
 * by swap preemption (0: none). preempt_mode PA_PREEMPT_RECOMPUTE takes no host
 * pool and only one-sample requests. */
int pa_sched_create(int num_blocks, int block_size, const int32_t* initial_free_order,
                    int max_num_seqs, int num_host_blocks, int preempt_mode, pa_sched** out);
void pa_sched_destroy(pa_sched* s);

/* PA_ERR_INVALID_ARG for bad sizes, a duplicate or negative id, or several
 * samples in recompute mode; PA_ERR_NO_FREE_BLOCKS when the request could never
 * fit (num_samples > max_num_seqs, or num_samples * ceil((prompt_len +
 * output_len) / block_size) > num_blocks). */
int pa_sched_submit(pa_sched* s, int64_t request_id, int prompt_len, int output_len,
                    int num_samples, int64_t arrival_step);

/* pa_sched_submit with the prompt's token ids (prompt_tokens[prompt_len], copied):
 * the request is admitted through the block manager's prefix cache
 * (pa_bm_add_seq_cached). Leading full prompt blocks already cached (by earlier
 * requests, or by this one before it was dropped for recomputation) are shared
 * and not written again; the admission check counts the blocks found, less
 * those no sequence holds. A recomputed request re-registers its prompt this
 * way and appends its generated tokens after it ("PagedAttention: The vLLM
 * Paper", "Impact and Follow-Ups", item 1, prefix caching). */
int pa_sched_submit_tokens(pa_sched* s, int64_t request_id, const int32_t* prompt_tokens,
                           int prompt_len, int output_len, int num_samples,
                           int64_t arrival_step);

/* Plans the next step and writes its counts to *plan. PA_ERR_NO_FREE_BLOCKS if
 * a many-sample request could not be preempted (host pool full); the scheduler
 * is then failed and every later step returns that error. */
int pa_sched_step(pa_sched* s, pa_sched_plan* plan);

/* 1 when nothing is pending, waiting, running, swapped or left to free. */
int pa_sched_idle(const pa_sched* s);

/* Detail of the last planned step. Every output pointer may be NULL; arrays
 * are sized by the counts in pa_sched_plan.
 *   requests: finished[num_finished], preempted[num_preempted] with
 *     preempt_modes[num_preempted] (PA_PREEMPT_*), resumed[num_resumed],
 *     admitted[num_admitted] (request ids, in planning order);
 *   pairs: swap_out[num_swap_out][2], swap_in[num_swap_in][2],
 *     copies[num_copies][2];
 *   writes (which = 0: prefill, 1: new tokens): per token its request, sample,
 *     position in the sample's sequence and slot;
 *   batch: per decoded sequence its request, sample and context length, and
 *     block_tables[num_seqs][max_blocks_per_seq] padded with -1. */
int pa_sched_plan_requests(const pa_sched* s, int64_t* finished, int64_t* preempted,
                           int32_t* preempt_modes, int64_t* resumed, int64_t* admitted);
int pa_sched_plan_pairs(const pa_sched* s, int64_t* swap_out, int64_t* swap_in,
                        int64_t* copies);
int pa_sched_plan_writes(const pa_sched* s, int which, int64_t* request, int32_t* sample,
                         int32_t* position, int64_t* slot);
int pa_sched_plan_batch(const pa_sched* s, int64_t* request, int32_t* sample,
                        int32_t* context_lens, int32_t* block_tables);

/* KV occupancy now: *filled = slots holding tokens and *allocated = block_size x device
 * blocks held by resident requests (running, and finished in the last step);
 * a shared block counts once, at the fill of its fullest holder. */
int pa_sched_kv_usage(const pa_sched* s, int64_t* filled, int64_t* allocated);

/* The scheduler's block manager (owned by the scheduler; read-only use). */
const pa_bm* pa_sched_block_manager(const pa_sched* s);

/* Executor. pa_sched_attach allocates, once, the executor's device metadata
 * buffers, a ring of pinned host staging buffers and the decode workspace, for
 * the given head shape and a largest context of max_context_len tokens (on the
 * current device). Planning works without it. */
int pa_sched_attach(pa_sched* s, int num_q_heads, int num_kv_heads, int head_dim, int dtype,
                    int max_context_len);

/* pa_sched_attach over 8-bit caches: the executor writes tokens with
 * pa_reshape_and_cache_fp8 (key/value inputs of type dtype, scales k_scale /
 * v_scale), decodes with pa_paged_decode_fp8 and copies and swaps one-byte
 * pools (PA_FP8_E4M3; the pinned host pool holds codes too). */
int pa_sched_attach_fp8(pa_sched* s, int num_q_heads, int num_kv_heads, int head_dim, int dtype,
                        int max_context_len, float k_scale, float v_scale);

/* Decode of sequences that share leading blocks, inside the executor. Samples
 * forked from one prompt share its full blocks, and so do requests whose
 * prompts were found in the prefix cache ("PagedAttention: The vLLM Paper",
 * "Implementation Essentials", prefix sharing). The executor groups a step's
 * batch with pa_bm_prefix_groups (8 / G members per group, G query heads per KV
 * head; no grouping when G = 8) and, when a group exists, decodes the step with
 * pa_paged_decode_cascade (pa_paged_decode_cascade_fp8 over 8-bit caches),
 * which reads each group's shared blocks once:
 *   PA_SCHED_CASCADE_OFF   never (always pa_paged_decode)
 *   PA_SCHED_CASCADE_ON    whenever the batch has a group
 *   PA_SCHED_CASCADE_AUTO  (default) when the shared blocks it reads once
 *                          instead of once per member from another request
 *                          than the group's first add up to 32 MiB (about the
 *                          cost of its two extra launches). Samples of one
 *                          request are left out: they have equal contexts, so
 *                          the plain decode runs them side by side and L2
 *                          serves their shared prompt once.
 * The results equal the plain decode's up to floating-point rounding order.
 * pa_sched_attach sizes the cascade's workspace once. pa_sched_last_cascade
 * reports the groups the last executed step decoded through the cascade (0 when
 * it used pa_paged_decode) and the block reads that saved. */
#define PA_SCHED_CASCADE_OFF 0
#define PA_SCHED_CASCADE_ON 1
#define PA_SCHED_CASCADE_AUTO 2
int pa_sched_set_cascade(pa_sched* s, int mode);
int pa_sched_last_cascade(const pa_sched* s, int* num_groups, int64_t* shared_blocks);

/* Runs the last planned step on `stream` in device order: pa_swap_blocks for
 * the swap pairs (device pool k_cache/v_cache <-> pinned host pool
 * host_k/host_v, [num_host_blocks][Hkv][16][d]; may be NULL when the plan has
 * no swap pair), pa_reshape_and_cache of prefill_key/prefill_value
 * ([num_prefill][Hkv][d], contiguous, device), pa_copy_blocks, pa_reshape_and_cache
 * of key/value ([num_writes][Hkv][d]), then pa_paged_decode of q
 * ([num_seqs][Hq][d]) into out ([num_seqs][Hq][d]) through the plan's tables,
 * longest context first (or the cascade, above, when sequences share blocks). Row i of each input belongs to write / sequence i of
 * the plan. Block tables, context lengths, slots and the order reach the device
 * through the pinned ring with one host-to-device copy per step; the call
 * waits only for the copy that last used the ring slot. Never synchronises the
 * stream otherwise. dev_error as pa_paged_decode. A step may be executed at
 * most once, and before the next pa_sched_step. */
int pa_sched_execute(pa_sched* s, void* k_cache, void* v_cache, void* host_k, void* host_v,
                     const void* prefill_key, const void* prefill_value, const void* key,
                     const void* value, const void* q, void* out, float scale, int* dev_error,
                     void* stream);

#ifdef __cplusplus
}
#endif

#endif /* PA_H_ */
