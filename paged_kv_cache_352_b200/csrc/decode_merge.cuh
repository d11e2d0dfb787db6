// Second-pass merge of the split-KV partition states (the reduce that follows
// the warp-per-partition decode kernel).
#pragma once

#include <math.h>
#include <string.h>

#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {
namespace {

// Second pass of the warp-per-partition split: one CTA per (sequence, query
// head) merges that row's states in logical order,
//   out = sum_p exp2(m_p - M) acc_p / sum_p exp2(m_p - M) l_p,  M = max_p m_p,
// each thread owning a float4 of columns for the states p = set (mod kSets);
// the sets are added in a fixed order. A state covers the WARPS consecutive
// partitions of one decode CTA (merged on chip), so a sequence of n partitions
// has ceil(n / WARPS) of them.
constexpr int kMergeThreads = 512;

template <typename T, int D, int G, int WARPS>
__global__ void __launch_bounds__(kMergeThreads) merge_partitions_kernel(const DecodeArgs a) {
  grid_dependency_wait();  // the partition states come from the decode kernel
  allow_dependents();
  constexpr int kCols = D / 4;
  constexpr int kSets = kMergeThreads / kCols;
  __shared__ float red[kMergeThreads];
  __shared__ float4 part_sum[kSets][kCols];
  const int kvh = blockIdx.x / G;
  const int g = blockIdx.x - kvh * G;
  const int s = blockIdx.y;
  const int tid = threadIdx.x;
  int ctx = __ldg(a.context_lens + s);
  if (ctx < 0 || ctx > a.max_blocks_per_seq * kBlockSize || ctx > a.max_context_len) ctx = 0;
  const int nblk = (ctx + kBlockSize - 1) / kBlockSize;
  const int nparts = ((nblk + a.part_blocks - 1) / a.part_blocks + WARPS - 1) / WARPS;
  T* out = reinterpret_cast<T*>(a.out) + ((size_t)s * a.num_q_heads + (size_t)kvh * G + g) * D;
  if (nparts == 0) {
    for (int i = tid; i < D; i += blockDim.x) out[i] = Storage<T>::from_f32(0.f);
    return;
  }
  const size_t base = ((size_t)s * a.num_kv_heads + kvh) * a.max_parts * G + g;
  // M, then L, by fixed-order block reductions
  float m = -INFINITY;
  for (int p = tid; p < nparts; p += blockDim.x) m = fmaxf(m, __ldcg(a.ws_m + base + (size_t)p * G));
  red[tid] = m;
  __syncthreads();
  for (int w = kMergeThreads / 2; w > 0; w >>= 1) {
    if (tid < w) red[tid] = fmaxf(red[tid], red[tid + w]);
    __syncthreads();
  }
  const float M = red[0] == -INFINITY ? 0.f : red[0];
  __syncthreads();
  float l = 0.f;
  for (int p = tid; p < nparts; p += blockDim.x)
    l += exp2f(__ldcg(a.ws_m + base + (size_t)p * G) - M) * __ldcg(a.ws_l + base + (size_t)p * G);
  red[tid] = l;
  __syncthreads();
  for (int w = kMergeThreads / 2; w > 0; w >>= 1) {
    if (tid < w) red[tid] += red[tid + w];
    __syncthreads();
  }
  const float L = red[0];
  const int col = tid % kCols;
  const int set = tid / kCols;
  const float4* acc = reinterpret_cast<const float4*>(a.ws_acc) + base * kCols;
  float4 sum[4];
#pragma unroll
  for (int u = 0; u < 4; ++u) sum[u] = make_float4(0.f, 0.f, 0.f, 0.f);
  int p = set;
  for (; p + 3 * kSets < nparts; p += 4 * kSets) {
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int q = p + u * kSets;
      const float w = exp2f(__ldcg(a.ws_m + base + (size_t)q * G) - M);
      const float4 v = __ldcg(acc + (size_t)q * G * kCols + col);
      sum[u].x = fmaf(w, v.x, sum[u].x);
      sum[u].y = fmaf(w, v.y, sum[u].y);
      sum[u].z = fmaf(w, v.z, sum[u].z);
      sum[u].w = fmaf(w, v.w, sum[u].w);
    }
  }
#pragma unroll
  for (int u = 0; u < 4; ++u) {  // at most three partitions of this set are left
    const int q = p + u * kSets;
    if (q < nparts) {
      const float w = exp2f(__ldcg(a.ws_m + base + (size_t)q * G) - M);
      const float4 v = __ldcg(acc + (size_t)q * G * kCols + col);
      sum[u].x = fmaf(w, v.x, sum[u].x);
      sum[u].y = fmaf(w, v.y, sum[u].y);
      sum[u].z = fmaf(w, v.z, sum[u].z);
      sum[u].w = fmaf(w, v.w, sum[u].w);
    }
  }
  float4 t;
  t.x = (sum[0].x + sum[1].x) + (sum[2].x + sum[3].x);
  t.y = (sum[0].y + sum[1].y) + (sum[2].y + sum[3].y);
  t.z = (sum[0].z + sum[1].z) + (sum[2].z + sum[3].z);
  t.w = (sum[0].w + sum[1].w) + (sum[2].w + sum[3].w);
  part_sum[set][col] = t;
  __syncthreads();
  if (set == 0) {
    float4 r = part_sum[0][col];
#pragma unroll
    for (int k = 1; k < kSets; ++k) {
      r.x += part_sum[k][col].x;
      r.y += part_sum[k][col].y;
      r.z += part_sum[k][col].z;
      r.w += part_sum[k][col].w;
    }
    const float f = L > 0.f ? a.out_scale / L : 0.f;
    T o[4] = {Storage<T>::from_f32(r.x * f), Storage<T>::from_f32(r.y * f),
              Storage<T>::from_f32(r.z * f), Storage<T>::from_f32(r.w * f)};
    uint2 packed;
    memcpy(&packed, o, sizeof(packed));
    *reinterpret_cast<uint2*>(out + 4 * col) = packed;
  }
}

}  // namespace
}  // namespace pa
