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
//   out = sum_p exp2(m_p - M) acc_p / sum_p exp2(m_p - M) l_p,  M = max_p m_p.
// A state covers the WARPS consecutive partitions of one decode CTA (merged on
// chip), so a sequence of n partitions has ceil(n / WARPS) of them. Thread
// (set, col) owns a float4 of columns and the states p = set (mod kSets), which
// it merges in one pass with a running maximum, loading kInFlight states per
// round; the kSets partial states then merge in shared memory in set order.
// The result depends only on the number of states.
constexpr int kMergeThreads = 512;

template <typename T, int D, int G, int WARPS>
__global__ void __launch_bounds__(kMergeThreads) merge_partitions_kernel(const DecodeArgs a) {
  grid_dependency_wait();  // the partition states come from the decode kernel
  allow_dependents();
  constexpr int kCols = D / 4;
  constexpr int kSets = kMergeThreads / kCols;
  constexpr int kInFlight = 4;
  __shared__ float set_m[kSets], set_l[kSets];
  __shared__ float4 set_acc[kSets][kCols];
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
  const float4* acc = reinterpret_cast<const float4*>(a.ws_acc) + base * kCols;
  const int col = tid % kCols;
  const int set = tid / kCols;
  float M = -INFINITY, L = 0.f;
  float4 A = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int p0 = set; p0 < nparts; p0 += kInFlight * kSets) {
    float m[kInFlight], l[kInFlight];
    float4 v[kInFlight];
#pragma unroll
    for (int u = 0; u < kInFlight; ++u) {
      const int p = p0 + u * kSets;
      m[u] = -INFINITY;
      l[u] = 0.f;
      v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (p < nparts) {
        m[u] = __ldcg(a.ws_m + base + (size_t)p * G);
        l[u] = __ldcg(a.ws_l + base + (size_t)p * G);
        v[u] = __ldcg(acc + (size_t)p * G * kCols + col);
      }
    }
    float Mn = M;
#pragma unroll
    for (int u = 0; u < kInFlight; ++u) Mn = fmaxf(Mn, m[u]);
    if (Mn == -INFINITY) continue;  // only empty partitions so far
    const float sc = exp2f(M - Mn);  // 0 while M is still -inf
    L *= sc;
    A.x *= sc;
    A.y *= sc;
    A.z *= sc;
    A.w *= sc;
#pragma unroll
    for (int u = 0; u < kInFlight; ++u) {
      const float w = exp2f(m[u] - Mn);
      L = fmaf(w, l[u], L);
      A.x = fmaf(w, v[u].x, A.x);
      A.y = fmaf(w, v[u].y, A.y);
      A.z = fmaf(w, v[u].z, A.z);
      A.w = fmaf(w, v[u].w, A.w);
    }
    M = Mn;
  }
  set_acc[set][col] = A;
  if (col == 0) {
    set_m[set] = M;
    set_l[set] = L;
  }
  __syncthreads();
  if (set != 0) return;
  float Mt = -INFINITY;
#pragma unroll
  for (int k = 0; k < kSets; ++k) Mt = fmaxf(Mt, set_m[k]);
  const float Mref = Mt == -INFINITY ? 0.f : Mt;
  float Lt = 0.f;
  float4 r = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int k = 0; k < kSets; ++k) {
    const float w = exp2f(set_m[k] - Mref);  // 0 for a set that saw no state
    const float4 x = set_acc[k][col];
    Lt = fmaf(w, set_l[k], Lt);
    r.x = fmaf(w, x.x, r.x);
    r.y = fmaf(w, x.y, r.y);
    r.z = fmaf(w, x.z, r.z);
    r.w = fmaf(w, x.w, r.w);
  }
  const float f = Lt > 0.f ? a.out_scale / Lt : 0.f;
  T o[4] = {Storage<T>::from_f32(r.x * f), Storage<T>::from_f32(r.y * f),
            Storage<T>::from_f32(r.z * f), Storage<T>::from_f32(r.w * f)};
  uint2 packed;
  memcpy(&packed, o, sizeof(packed));
  *reinterpret_cast<uint2*>(out + 4 * col) = packed;
}

}  // namespace
}  // namespace pa
