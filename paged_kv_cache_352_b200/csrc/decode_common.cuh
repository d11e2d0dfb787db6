// Shared tail of the paged-decode kernels: merging per-warp softmax states
// into the CTA's result, and the split-KV merge across partitions.
#pragma once

#include <math.h>
#include <string.h>

#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {

// Outputs are multiplied by a.out_scale (the value scale of an E4M3 cache, else 1).
// After the main loop every warp w has left, in shared memory,
//   red_m[w][g], red_l[w][g]   its running max (base 2) and sum of exponentials
//   red_acc[w][g][D]           its unnormalised output rows
// for the G query heads of this CTA's KV head. This merges them by rescaling
// to the common maximum. A sequence with a single partition writes `out`
// directly. Otherwise the CTA stores its partition state in the workspace, and
// the CTA that completes the sequence's last partition merges all partitions
// in logical order and returns the counter to zero. With a.states_only every
// partition stores its state and nothing is merged.
// `wts` (>= nparts * G floats of shared memory) may alias red_*: it is written
// only after they have been read. Every thread of the CTA must call this with
// the same arguments; it ends with a barrier, so shared memory it used can be
// rewritten as soon as it returns.
template <typename T, int D, int G, int WARPS>
__device__ __forceinline__ void finish_partition(const DecodeArgs& a, float* wts,
                                                 const float* red_m, const float* red_l,
                                                 const float* red_acc, int s, int kvh, int part,
                                                 int nparts, T* out_rows) {
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const bool split = nparts > 1 || a.states_only;
  const size_t unit = (size_t)s * a.num_kv_heads + kvh;
  for (int item = threadIdx.x; item < G * D; item += blockDim.x) {
    const int g = item / D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < WARPS; ++w) M = fmaxf(M, red_m[w * G + g]);
    // M is finite unless every block of the partition was skipped as out of range
    const float Mref = M == -INFINITY ? 0.f : M;
    float L = 0.f, A = 0.f;
#pragma unroll
    for (int w = 0; w < WARPS; ++w) {
      const float sc = exp2f(red_m[w * G + g] - Mref);
      L = fmaf(sc, red_l[w * G + g], L);
      A = fmaf(sc, red_acc[(w * G) * D + item], A);
    }
    if (!split) {
      out_rows[item] = Storage<T>::from_f32(L > 0.f ? (A / L) * a.out_scale : 0.f);
    } else {
      const size_t row = (unit * a.max_parts + part) * G + g;
      a.ws_acc[row * D + (item % D)] = A;
      if (item % D == 0) {
        a.ws_m[row] = M;
        a.ws_l[row] = L;
      }
    }
  }
  if (!split || a.states_only) {
    __syncthreads();
    return;
  }

  // ---- split-KV: the last partition to finish merges all of them.
  // The barrier makes every thread's partial-result stores visible to thread 0,
  // whose gpu-scope acq_rel add then publishes them (release is cumulative) and,
  // in the last CTA, acquires the other partitions' results before the barrier
  // hands them to the rest of the CTA. One fence per CTA instead of one per thread.
  __syncthreads();
  __shared__ int is_last;
  if (threadIdx.x == 0) {
    const int prev = atom_add_acq_rel_gpu(a.ws_count + unit, 1);
    is_last = (prev == nparts - 1);
  }
  __syncthreads();
  if (!is_last) return;  // uniform across the CTA; the barrier above ends this call

  // per-(partition, head) weights exp2(m_p - M) / L, staged in shared memory [nparts][G]
  __shared__ float headM[G], headL[G];
  const float* pm = a.ws_m + unit * a.max_parts * G;
  const float* pl = a.ws_l + unit * a.max_parts * G;
  for (int g = warp; g < G; g += WARPS) {
    float M = -INFINITY;
    for (int p = lane; p < nparts; p += 32) M = fmaxf(M, __ldcg(pm + p * G + g));
#pragma unroll
    for (int mask = 16; mask > 0; mask >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, mask));
    if (M == -INFINITY) M = 0.f;
    float L = 0.f;
    for (int p = lane; p < nparts; p += 32)
      L += exp2f(__ldcg(pm + p * G + g) - M) * __ldcg(pl + p * G + g);
#pragma unroll
    for (int mask = 16; mask > 0; mask >>= 1) L += __shfl_xor_sync(0xffffffffu, L, mask);
    if (lane == 0) {
      headM[g] = M;
      headL[g] = L;
    }
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < nparts * G; idx += blockDim.x) {
    const int g = idx % G;
    wts[idx] = headL[g] > 0.f ? exp2f(__ldcg(pm + idx) - headM[g]) / headL[g] : 0.f;
  }
  __syncthreads();
  // Each thread merges four adjacent output columns (one float4 of every
  // partition's state), keeping kMergeInFlight partitions' loads in flight: the
  // merge is bound by load latency, not bandwidth. Accumulator u takes the
  // partitions p = u (mod kMergeInFlight) in increasing order and the
  // accumulators are added in a fixed tree, so the result depends only on the
  // partition count.
  constexpr int kMergeInFlight = 8;
  constexpr int kItems4 = G * D / 4;
  const float4* accp = reinterpret_cast<const float4*>(a.ws_acc + unit * a.max_parts * G * D);
  for (int it = threadIdx.x; it < kItems4; it += blockDim.x) {
    const int g = (it * 4) / D;
    float4 acc[kMergeInFlight];
#pragma unroll
    for (int u = 0; u < kMergeInFlight; ++u) acc[u] = make_float4(0.f, 0.f, 0.f, 0.f);
    int p = 0;
    for (; p + kMergeInFlight <= nparts; p += kMergeInFlight) {
#pragma unroll
      for (int u = 0; u < kMergeInFlight; ++u) {
        const float w = wts[(p + u) * G + g];
        const float4 v = __ldcg(accp + (size_t)(p + u) * kItems4 + it);
        acc[u].x = fmaf(w, v.x, acc[u].x);
        acc[u].y = fmaf(w, v.y, acc[u].y);
        acc[u].z = fmaf(w, v.z, acc[u].z);
        acc[u].w = fmaf(w, v.w, acc[u].w);
      }
    }
#pragma unroll
    for (int u = 0; u < kMergeInFlight; ++u) {
      if (p + u < nparts) {
        const float w = wts[(p + u) * G + g];
        const float4 v = __ldcg(accp + (size_t)(p + u) * kItems4 + it);
        acc[u].x = fmaf(w, v.x, acc[u].x);
        acc[u].y = fmaf(w, v.y, acc[u].y);
        acc[u].z = fmaf(w, v.z, acc[u].z);
        acc[u].w = fmaf(w, v.w, acc[u].w);
      }
    }
#pragma unroll
    for (int step = 1; step < kMergeInFlight; step *= 2) {
#pragma unroll
      for (int u = 0; u < kMergeInFlight; u += 2 * step) {
        acc[u].x += acc[u + step].x;
        acc[u].y += acc[u + step].y;
        acc[u].z += acc[u + step].z;
        acc[u].w += acc[u + step].w;
      }
    }
    T r[4] = {Storage<T>::from_f32(acc[0].x * a.out_scale),
              Storage<T>::from_f32(acc[0].y * a.out_scale),
              Storage<T>::from_f32(acc[0].z * a.out_scale),
              Storage<T>::from_f32(acc[0].w * a.out_scale)};
    uint2 packed;
    memcpy(&packed, r, sizeof(packed));
    *reinterpret_cast<uint2*>(out_rows + 4 * it) = packed;
  }
  if (threadIdx.x == 0) a.ws_count[unit] = 0;
  __syncthreads();
}

}  // namespace pa
