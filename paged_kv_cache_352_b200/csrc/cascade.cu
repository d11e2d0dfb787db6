// Cascade decode of sequences that share leading blocks (forks of one prompt).
//
// Sequences forked from one prompt hold the same physical blocks for the
// prompt's full blocks ("PagedAttention and Continuous Batching", "Pages, from
// operating systems": copy-on-write sharing; "PagedAttention: The vLLM Paper",
// "Implementation Essentials": prefix sharing). Attention over those blocks is
// the same computation for every member except for the query, so the members'
// query heads are stacked as one KV head's query group and the shared blocks
// are read once for all of them. A decode over each sequence's remaining blocks
// follows, and the two partial softmax states are merged per output row:
//   M = max(m_prefix, m_own),  out = (2^(m_p - M) acc_p + 2^(m_o - M) acc_o) /
//                                    (2^(m_p - M) l_p + 2^(m_o - M) l_o),
// which is the decode over the whole context up to floating-point rounding.
//
// This file holds the two small kernels around the decode launch(es):
//   cascade_prepare_kernel  validates each group, writes its prefix table and
//                           every sequence's own-block table, and stacks the
//                           members' queries when the prefix decode runs as a
//                           launch of its own (the single-launch form reads
//                           them in place and does not wait for this kernel);
//   cascade_merge_kernel    one warp per output row merges the prefix
//                           partitions and the own-block partitions.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <string.h>

#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {
namespace {

constexpr int kPrepThreads = 256;
constexpr int kMergeWarps = 8;

// Whether sequence s is owned by a group: its (group, slot) entry names it back.
__device__ __forceinline__ bool owned(const CascadeArgs& c, int s, int& g, int& m) {
  g = __ldg(c.seq_group + s);
  m = __ldg(c.seq_member + s);
  if (g < 0 || g >= c.num_groups || m < 0 || m >= c.group_size) return false;
  return __ldg(c.group_members + (size_t)g * c.group_size + m) == s;
}

__device__ __forceinline__ bool ctx_ok(const CascadeArgs& c, int ctx) {
  return ctx >= 0 && ctx <= c.max_blocks_per_seq * kBlockSize && ctx <= c.max_context_len;
}

// Table row of sequence s from block `first` on, padded with -1.
__device__ void write_own_table(const CascadeArgs& c, int s, int first) {
  const int32_t* src = c.block_tables + (size_t)s * c.max_blocks_per_seq;
  int32_t* dst = c.s_tables + (size_t)s * c.max_blocks_per_seq;
  for (int b = threadIdx.x; b < c.max_blocks_per_seq; b += blockDim.x)
    dst[b] = first + b < c.max_blocks_per_seq ? __ldg(src + first + b) : -1;
}

// Three kinds of CTA, by blockIdx.x:
//   [0, num_groups)                 group g: checks it, writes its prefix table, the
//                                   own-block tables of the members it owns and their
//                                   prefix-state rows;
//   [num_groups, + num_seqs)        sequence s when no group owns it: its whole table;
//   [.., + num_groups * copy_ctas)  one query vector per thread of group g's stacked
//                                   queries (none when the prefix decode reads the
//                                   members' rows itself: copy_ctas = 0).
// Every own-block table is written by exactly one CTA. A group CTA loads its
// members' ids, then their lengths, ownership and prefix entries in one round,
// and copies the tables in a third.
template <int D>
__global__ void __launch_bounds__(kPrepThreads) cascade_prepare_kernel(const CascadeArgs c,
                                                                        int gh, int copy_ctas) {
  grid_dependency_wait();  // tables, lengths and queries may come from the kernel ahead
  allow_dependents();      // the decode launch may start; it waits for this kernel
  constexpr int kVec = D / 8;  // 16-byte vectors per query row
  constexpr int kMaxGroup = kPrepThreads / 32;
  const int tid = threadIdx.x;
  const int gg = c.group_size * gh;
  if ((int)blockIdx.x >= c.num_groups + c.num_seqs) {
    // stacked queries: row (g, kvh * Gg + slot * gh + h) = q[member slot][kvh * gh + h]
    const int y = blockIdx.x - c.num_groups - c.num_seqs;
    const int g = y / copy_ctas;
    const int i = (y - g * copy_ctas) * kPrepThreads + tid;
    const int rows = c.num_kv_heads * gg;
    if (i >= rows * kVec) return;
    const int v = i % kVec, r = i / kVec;
    const int kvh = r / gg, rem = r - kvh * gg;
    const int slot = rem / gh, h = rem - slot * gh;
    const int s = __ldg(c.group_members + (size_t)g * c.group_size + slot);
    uint4 val = make_uint4(0u, 0u, 0u, 0u);
    if (s >= 0 && s < c.num_seqs)
      val = __ldg(reinterpret_cast<const uint4*>(c.q) +
                  ((size_t)s * c.num_q_heads + (size_t)kvh * gh + h) * kVec + v);
    reinterpret_cast<uint4*>(c.gq)[((size_t)g * rows) * kVec + i] = val;
    return;
  }
  if ((int)blockIdx.x >= c.num_groups) {
    const int s = blockIdx.x - c.num_groups;
    int g, m;
    if (owned(c, s, g, m)) return;
    int ctx = __ldg(c.context_lens + s);
    if (!ctx_ok(c, ctx)) ctx = 0;  // the decode flags it
    write_own_table(c, s, 0);
    if (tid == 0) {
      c.s_ctx[s] = ctx;
      c.s_pbase[s] = -1;
      c.s_np[s] = 0;
    }
    return;
  }
  const int g = blockIdx.x;
  const int32_t* members = c.group_members + (size_t)g * c.group_size;
  __shared__ int mem[kMaxGroup], mctx[kMaxGroup], mown[kMaxGroup];
  __shared__ int bad, P_sh;
  if (tid < c.group_size) mem[tid] = __ldg(members + tid);
  if (tid == 0) {
    P_sh = __ldg(c.group_prefix_blocks + g);
    bad = 0;
  }
  __syncthreads();
  int P = P_sh;
  const int leader = mem[0];
  const bool shape_ok = P >= 1 && P <= c.max_prefix_blocks && leader >= 0 && leader < c.num_seqs;
  if (tid < c.group_size) {
    const int s = mem[tid];
    int ctx = -1, own = 0;
    if (s >= 0 && s < c.num_seqs) {
      ctx = __ldg(c.context_lens + s);
      if (!ctx_ok(c, ctx)) ctx = -1;
      own = __ldg(c.seq_group + s) == g && __ldg(c.seq_member + s) == tid;
    }
    mctx[tid] = ctx;
    mown[tid] = own;
    // a listed member that the group does not own is reported (another group or
    // its own CTA serves it); its stacked rows are computed and never read
    if (s >= 0 && !own) report(c.dev_error, PA_DEVERR_GROUP);
  }
  int flag = !shape_ok;
  if (shape_ok) {
    // every listed member holds the leader's first P entries
    const int32_t* lt = c.block_tables + (size_t)leader * c.max_blocks_per_seq;
    for (int i = tid; i < c.group_size * P; i += blockDim.x) {
      const int slot = i / P, b = i - slot * P;
      const int s = mem[slot];
      if (s < 0) continue;
      if (s >= c.num_seqs ||
          __ldg(c.block_tables + (size_t)s * c.max_blocks_per_seq + b) != __ldg(lt + b))
        flag = 1;
    }
  }
  if (flag) atomicOr(&bad, 1);
  __syncthreads();
  // ... and holds them as full blocks inside its context
  if (!bad && tid < c.group_size && mem[tid] >= 0 && mctx[tid] < P * kBlockSize)
    atomicOr(&bad, 1);
  __syncthreads();
  if (bad) {
    P = 0;
    if (tid == 0) report(c.dev_error, PA_DEVERR_GROUP);
  }
  if (tid == 0) c.g_ctx[g] = P * kBlockSize;
  {
    const int32_t* lt = c.block_tables + (size_t)(P > 0 ? leader : 0) * c.max_blocks_per_seq;
    int32_t* gt = c.g_tables + (size_t)g * c.max_blocks_per_seq;
    for (int b = tid; b < c.max_blocks_per_seq; b += blockDim.x) gt[b] = b < P ? __ldg(lt + b) : -1;
  }
  // own-block tables and prefix-state rows of the members this group owns:
  // warp w serves slot w
  const int w = tid >> 5, lane = tid & 31;
  if (w < c.group_size && mown[w]) {
    const int s = mem[w];
    const int ctx = mctx[w] < 0 ? 0 : mctx[w];
    const int32_t* src = c.block_tables + (size_t)s * c.max_blocks_per_seq;
    int32_t* dst = c.s_tables + (size_t)s * c.max_blocks_per_seq;
    for (int b = lane; b < c.max_blocks_per_seq; b += 32)
      dst[b] = P + b < c.max_blocks_per_seq ? __ldg(src + P + b) : -1;
    if (lane == 0) {
      c.s_ctx[s] = ctx > P * kBlockSize ? ctx - P * kBlockSize : 0;
      c.s_pbase[s] = P > 0 ? (g * c.num_kv_heads * c.g_parts) * gg + w * gh : -1;
      c.s_np[s] = (P + c.g_part_blocks - 1) / c.g_part_blocks;
    }
  }
}

// One warp per output row (s, h): lane l owns columns 4l .. 4l + 3. The prefix
// partitions (in order), then the own-block partitions (in order), are merged
// four at a time with a running maximum: each set's states are loaded together,
// and the running sums are rescaled when the maximum grows. The order is fixed,
// so results do not depend on timing.
template <typename T, int D>
__global__ void __launch_bounds__(kMergeWarps * 32) cascade_merge_kernel(const CascadeArgs c,
                                                                         int gh) {
  constexpr int kSet = 4;
  const int row = blockIdx.x * kMergeWarps + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= c.num_seqs * c.num_q_heads) return;
  const int s = row / c.num_q_heads;
  const int h = row - s * c.num_q_heads;
  const int kvh = h / gh, hh = h - kvh * gh;
  const int gg = c.group_size * gh;
  // Prepare's rows for this sequence (three independent loads in one round),
  // read before the wait for the decodes. This kernel starts only once every CTA
  // of the decode launch ahead of it has let it start (or exited), and every
  // own-block CTA does so only after its own wait, which returns once prepare
  // has completed and its writes are performed; loads through L2 then see them.
  // (With the decodes on two streams, the launch ahead is the own-block decode,
  // whose CTAs likewise wait first.) Measured on the shared-prefix batch: 88.3 ->
  // 87.0 us per call (8-bit 57.9 -> 57.4 us).
  const int pb = __ldcg(c.s_pbase + s);
  const int np_raw = __ldcg(c.s_np + s);
  const int own_ctx = __ldcg(c.s_ctx + s);
  grid_dependency_wait();  // the partition states come from the decodes
  allow_dependents();
  const int np = pb < 0 ? 0 : np_raw;
  const int ob = (own_ctx + kBlockSize - 1) / kBlockSize;
  const int no = (ob + c.s_part_blocks - 1) / c.s_part_blocks;
  const size_t pbase = pb < 0 ? 0 : (size_t)pb + (size_t)kvh * c.g_parts * gg + hh;
  const size_t obase = ((size_t)s * c.num_kv_heads + kvh) * c.s_parts * gh + hh;
  const bool col = lane * 4 < D;
  float M = -INFINITY, L = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int p0 = 0; p0 < np + no; p0 += kSet) {
    float m[kSet], l[kSet];
    float4 a[kSet];
#pragma unroll
    for (int u = 0; u < kSet; ++u) {
      const int p = p0 + u;
      m[u] = -INFINITY;
      l[u] = 0.f;
      a[u] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (p < np + no) {
        const bool pre = p < np;
        const size_t r = pre ? pbase + (size_t)p * gg : obase + (size_t)(p - np) * gh;
        m[u] = __ldcg((pre ? c.g_m : c.s_m) + r);
        l[u] = __ldcg((pre ? c.g_l : c.s_l) + r);
        if (col) a[u] = __ldcg(reinterpret_cast<const float4*>((pre ? c.g_acc : c.s_acc) + r * D) +
                               lane);
      }
    }
    float Mn = M;
#pragma unroll
    for (int u = 0; u < kSet; ++u) Mn = fmaxf(Mn, m[u]);
    if (Mn == -INFINITY) continue;  // nothing but empty partitions so far
    const float sc = exp2f(M - Mn);  // 0 while M is still -inf
    L *= sc;
    acc.x *= sc;
    acc.y *= sc;
    acc.z *= sc;
    acc.w *= sc;
#pragma unroll
    for (int u = 0; u < kSet; ++u) {
      const float wgt = exp2f(m[u] - Mn);
      L = fmaf(wgt, l[u], L);
      acc.x = fmaf(wgt, a[u].x, acc.x);
      acc.y = fmaf(wgt, a[u].y, acc.y);
      acc.z = fmaf(wgt, a[u].z, acc.z);
      acc.w = fmaf(wgt, a[u].w, acc.w);
    }
    M = Mn;
  }
  if (!col) return;
  const float f = L > 0.f ? c.out_scale / L : 0.f;
  T o[4] = {Storage<T>::from_f32(acc.x * f), Storage<T>::from_f32(acc.y * f),
            Storage<T>::from_f32(acc.z * f), Storage<T>::from_f32(acc.w * f)};
  uint2 packed;
  memcpy(&packed, o, sizeof(packed));
  *reinterpret_cast<uint2*>(reinterpret_cast<T*>(c.out) + (size_t)row * D + 4 * lane) = packed;
}

}  // namespace

cudaError_t launch_cascade_prepare(const CascadeArgs& c, int head_dim, bool stack_queries,
                                   cudaStream_t stream) {
  const int gh = c.num_q_heads / c.num_kv_heads;
  const long long vecs = (long long)c.num_kv_heads * c.group_size * gh * (head_dim / 8);
  const int copy_ctas = stack_queries ? (int)((vecs + kPrepThreads - 1) / kPrepThreads) : 0;
  const long long ctas = (long long)c.num_groups * (1 + copy_ctas) + c.num_seqs;
  if (ctas > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  const dim3 grid((unsigned)ctas);
  if (head_dim != 64 && head_dim != 128) return cudaErrorInvalidValue;
  return launch_dependent(head_dim == 64 ? cascade_prepare_kernel<64> : cascade_prepare_kernel<128>,
                          grid, dim3(kPrepThreads), 0, stream, c, gh, copy_ctas);
}

cudaError_t launch_cascade_merge(const CascadeArgs& c, int head_dim, int dtype,
                                 cudaStream_t stream) {
  const int gh = c.num_q_heads / c.num_kv_heads;
  const long long rows = (long long)c.num_seqs * c.num_q_heads;
  const dim3 grid((unsigned)((rows + kMergeWarps - 1) / kMergeWarps));
  const int threads = kMergeWarps * 32;
  void (*kern)(const CascadeArgs, int) = nullptr;
  if (dtype == PA_F16)
    kern = head_dim == 64 ? cascade_merge_kernel<__half, 64>
           : head_dim == 128 ? cascade_merge_kernel<__half, 128> : nullptr;
  else
    kern = head_dim == 64 ? cascade_merge_kernel<__nv_bfloat16, 64>
           : head_dim == 128 ? cascade_merge_kernel<__nv_bfloat16, 128> : nullptr;
  if (!kern) return cudaErrorInvalidValue;
  return launch_dependent(kern, grid, dim3(threads), 0, stream, c, gh);
}

}  // namespace pa
