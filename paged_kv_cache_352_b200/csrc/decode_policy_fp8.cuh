// Tensor-core arithmetic policy of the paged-decode kernel over E4M3 caches.
#pragma once

#include <cuda.h>
#include <math.h>
#include <string.h>

#include "decode_policies.cuh"
#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {

// ---------------------------------------------------------------------------
// Tensor cores over an E4M3 cache
// ---------------------------------------------------------------------------

// Fp8TensorPolicy (any G) reads the mma.sync fragments straight from the 8-bit
// tiles; nothing is widened through shared memory.
//
// Every E4M3 code is exact in half precision, so the contraction runs on f16
// operands whatever the query type: a bf16 query row is brought into f16 range
// by a power of two 2^-k (k = 0 unless its largest magnitude is at or above
// 2^15), and 2^k is folded into that row's logit scale.
//
// k-slot permutation. In one mma.m16n8k16 a lane holds the same four k-slots
// (2j, 2j+1, 2j+8, 2j+9, j = lane % 4) in its A and B fragments, so each lane
// may pair those slots with any head dimensions of its own, as long as q and K
// agree: lane j takes, at step kk = 4h + w, dimensions 16(j + 4h) + 4w .. +3.
// One 32-bit word of a key row then gives both B registers (low and high code
// pairs), and the lane reads its 16 or 32 code bytes of a row in 16-byte loads.
//
// Token permutation. S column n of n-tile nt is token (n >> 1) + 4(n & 1) + 8nt,
// so the S accumulator of lane j holds tokens j, j+4, j+8, j+12, which are also
// the P.V k-slots 2j, 2j+1, 2j+8, 2j+9 the lane feeds back as the A operand.
// For V the lane loads those four token rows at its 16 (d = 128) or 8 (d = 64)
// output dimensions and transposes the 4 x 4 byte blocks with byte permutes:
// each resulting word is one dimension's codes for the four tokens, low half
// b0, high half b1.
//
// Output columns: lane group g (lane / 4) is B column n = g; at d = 128 it owns
// dimensions 16 c(g) + nt, c(g) = 4(g & 1) + (g >> 1), at d = 64 dimensions
// 8g + nt. With 128-byte-swizzled tiles (d = 128, 2-D TMA) these choices make
// every K and V load of a warp bank-conflict free; d = 64 tiles arrive by 1-D
// bulk copies.
template <typename T, int D, int G>
struct Fp8TensorPolicy {
  static constexpr int KSTEPS = D / 16;
  static constexpr int NTO = D / 8;    // output n-tiles
  static constexpr int CPT = D / 64;   // 16-byte key chunks a lane reads per row
  static constexpr int kTileBytes = kBS * D;
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr bool kSwizzled = D == 128;
  static constexpr int kAlign = kSwizzled ? 1024 : 128;
  static constexpr int kScratchBytes = 0;
  static constexpr bool kTensorCores = true;
  static constexpr bool kTma2D = kSwizzled;
  static constexpr bool kFp8Cache = true;
  // Four CTAs (16 warps) per SM: the code conversions make this path issue-
  // rather than memory-latency-limited, and the extra warps hide their latency
  // (measured 4 % faster at 8 query heads per KV head than three CTAs).
  static constexpr int kMinCtasPerSm = 4;
  static_assert(D == 64 || D == 128, "unsupported head_dim");

  int g, j;
  uint4 qraw[CPT][2];      // the lane's 16 * CPT query elements of row g (raw T)
  uint32_t qa[KSTEPS][2];  // f16 A fragments (slots 2j,2j+1 and 2j+8,2j+9)
  float m, l, row_scale;
  float o[NTO][2];

  __device__ __forceinline__ void init(int lane) {
    g = lane >> 2;
    j = lane & 3;
  }

  __device__ __forceinline__ void prefetch_q(const DecodeArgs& a, int s, int kvh) {
    const uint4* qrow = reinterpret_cast<const uint4*>(
        reinterpret_cast<const T*>(a.q) + ((size_t)s * a.num_q_heads + (size_t)kvh * G + g) * D);
#pragma unroll
    for (int h = 0; h < CPT; ++h) {
      // elements 16(j + 4h) .. +15 = uint4 words 2(j + 4h), 2(j + 4h) + 1
      qraw[h][0] = g < G ? __ldg(qrow + 2 * (j + 4 * h)) : make_uint4(0u, 0u, 0u, 0u);
      qraw[h][1] = g < G ? __ldg(qrow + 2 * (j + 4 * h) + 1) : make_uint4(0u, 0u, 0u, 0u);
    }
  }

  __device__ __forceinline__ void begin(float scale_log2) {
    float qf[CPT][16];
    float amax = 0.f;
#pragma unroll
    for (int h = 0; h < CPT; ++h) {
      float lo[8], hi[8];
      Storage<T>::to_f32(qraw[h][0], lo);
      Storage<T>::to_f32(qraw[h][1], hi);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        qf[h][e] = lo[e];
        qf[h][8 + e] = hi[e];
        amax = fmaxf(amax, fmaxf(fabsf(lo[e]), fabsf(hi[e])));
      }
    }
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
    // 2^-k brings the row below 2^15 (f16's largest finite value is 65504)
    const int k = amax >= 32768.f ? ilogbf(amax) - 14 : 0;
    const float down = exp2f((float)-k);
    row_scale = scale_log2 * exp2f((float)k);
#pragma unroll
    for (int kk = 0; kk < KSTEPS; ++kk) {
      const int h = kk >> 2, w = kk & 3;
      const __half2 p0 = __floats2half2_rn(qf[h][4 * w] * down, qf[h][4 * w + 1] * down);
      const __half2 p1 = __floats2half2_rn(qf[h][4 * w + 2] * down, qf[h][4 * w + 3] * down);
      memcpy(&qa[kk][0], &p0, 4);
      memcpy(&qa[kk][1], &p1, 4);
    }
    m = -INFINITY;
    l = 0.f;
#pragma unroll
    for (int n = 0; n < NTO; ++n) o[n][0] = o[n][1] = 0.f;
  }

  static __device__ __forceinline__ void issue(const DecodeArgs& a, const CUtensorMap* tm_k,
                                               const CUtensorMap* tm_v, unsigned char* dst,
                                               uint64_t* bar, int phys, int kvh) {
    mbar_arrive_expect_tx(bar, kStageBytes);
    if constexpr (kSwizzled) {
      const int y = (phys * a.num_kv_heads + kvh) * kBS;
      tma_load_2d(dst, tm_k, 0, y, bar);
      tma_load_2d(dst + kTileBytes, tm_v, 0, y, bar);
    } else {
      const size_t off = ((size_t)phys * a.num_kv_heads + kvh) * kTileBytes;
      bulk_copy_g2s(dst, static_cast<const unsigned char*>(a.k_cache) + off, kTileBytes, bar);
      bulk_copy_g2s(dst + kTileBytes, static_cast<const unsigned char*>(a.v_cache) + off,
                    kTileBytes, bar);
    }
  }

  // Byte offset of 16-byte chunk c of row t in a tile.
  static __device__ __forceinline__ int chunk_off(int t, int c) {
    return kSwizzled ? t * D + ((c ^ (t & 7)) << 4) : t * D + (c << 4);
  }

  __device__ __forceinline__ void block(unsigned char* stage, int valid, unsigned char*) {
    const unsigned char* Ks = stage;
    const unsigned char* Vs = stage + kTileBytes;
    // ---- S = Q K^T; B column g of n-tile nt is token (g >> 1) + 4(g & 1) + 8nt
    const int krow = (g >> 1) + 4 * (g & 1);
    uint4 kw[2][CPT];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int h = 0; h < CPT; ++h)
        kw[nt][h] = *reinterpret_cast<const uint4*>(Ks + chunk_off(krow + 8 * nt, j + 4 * h));
    float sacc[2][2];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) sacc[nt][0] = sacc[nt][1] = 0.f;
#pragma unroll
    for (int kk = 0; kk < KSTEPS; ++kk) {
      const int h = kk >> 2, w = kk & 3;
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        const uint32_t word = w == 0 ? kw[nt][h].x : w == 1 ? kw[nt][h].y
                            : w == 2 ? kw[nt][h].z : kw[nt][h].w;
        MmaOps<__half>::run(sacc[nt], qa[kk][0], qa[kk][1], e4m3x2_to_half2_bits(word),
                            e4m3x2_to_half2_bits(word >> 16));
      }
    }
    // ---- online softmax for row g; this lane's columns are tokens j + 4e + 8nt
    float x[2][2];
    float bmax = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const bool ok = g < G && j + 4 * e + 8 * nt < valid;
        x[nt][e] = ok ? sacc[nt][e] * row_scale : -INFINITY;
        bmax = fmaxf(bmax, x[nt][e]);
      }
    bmax = fmaxf(bmax, __shfl_xor_sync(0xffffffffu, bmax, 1));
    bmax = fmaxf(bmax, __shfl_xor_sync(0xffffffffu, bmax, 2));
    const float mnew = fmaxf(m, bmax);
    const float mref = mnew == -INFINITY ? 0.f : mnew;
    const float alpha = exp2f(m - mref);
    m = mnew;
    const float p0 = exp2f(x[0][0] - mref), p1 = exp2f(x[0][1] - mref);
    const float p2 = exp2f(x[1][0] - mref), p3 = exp2f(x[1][1] - mref);
    l = fmaf(l, alpha, (p0 + p1) + (p2 + p3));
    uint32_t pa0, pa2;
    {
      const __half2 h0 = __floats2half2_rn(p0, p1);
      const __half2 h2 = __floats2half2_rn(p2, p3);
      memcpy(&pa0, &h0, 4);
      memcpy(&pa2, &h2, 4);
    }
    // ---- O += P V: rows j, j+4, j+8, j+12 at this lane group's dimensions
    constexpr int VW = D == 128 ? 4 : 2;  // 32-bit words of codes a lane reads per row
    uint32_t vr[4][VW];
#pragma unroll
    for (int mm = 0; mm < 4; ++mm) {
      const int t = j + 4 * mm;
      if constexpr (D == 128) {
        const int c = 4 * (g & 1) + (g >> 1);
        const uint4 v = *reinterpret_cast<const uint4*>(Vs + chunk_off(t, c));
        vr[mm][0] = v.x;
        vr[mm][1] = v.y;
        vr[mm][2] = v.z;
        vr[mm][3] = v.w;
      } else {
        const uint2 v = *reinterpret_cast<const uint2*>(Vs + t * D + 8 * g);
        vr[mm][0] = v.x;
        vr[mm][1] = v.y;
      }
    }
    // rows past the context may hold any codes (NaN included): clear them. Only a
    // sequence's last block is partly filled, and the test is uniform across the warp.
    if (valid < kBS) {
#pragma unroll
      for (int mm = 0; mm < 4; ++mm)
        if (j + 4 * mm >= valid) {
#pragma unroll
          for (int w = 0; w < VW; ++w) vr[mm][w] = 0u;
        }
    }
#pragma unroll
    for (int w = 0; w < VW; ++w) {
      // 4 x 4 byte transpose: y[i] = byte i of rows j, j+4, j+8, j+12
      const uint32_t t0 = __byte_perm(vr[0][w], vr[1][w], 0x5140);
      const uint32_t t1 = __byte_perm(vr[0][w], vr[1][w], 0x7362);
      const uint32_t t2 = __byte_perm(vr[2][w], vr[3][w], 0x5140);
      const uint32_t t3 = __byte_perm(vr[2][w], vr[3][w], 0x7362);
      const uint32_t y[4] = {__byte_perm(t0, t2, 0x5410), __byte_perm(t0, t2, 0x7632),
                             __byte_perm(t1, t3, 0x5410), __byte_perm(t1, t3, 0x7632)};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int nt = 4 * w + i;
        o[nt][0] *= alpha;
        o[nt][1] *= alpha;
        MmaOps<__half>::run(o[nt], pa0, pa2, e4m3x2_to_half2_bits(y[i]),
                            e4m3x2_to_half2_bits(y[i] >> 16));
      }
    }
  }

  __device__ __forceinline__ void to_red(float* red_m, float* red_l, float* red_acc, int warp,
                                         int) {
    float lsum = l + __shfl_xor_sync(0xffffffffu, l, 1);
    lsum += __shfl_xor_sync(0xffffffffu, lsum, 2);
    if (g < G) {
      if (j == 0) {
        red_m[warp * G + g] = m;
        red_l[warp * G + g] = lsum;
      }
      // accumulator columns 2j and 2j+1 of every n-tile
      const int base0 = 16 * j;
      const int base1 = D == 128 ? 64 + 16 * j : 16 * j + 8;
      float* dst = red_acc + (warp * G + g) * D;
#pragma unroll
      for (int n = 0; n < NTO; ++n) {
        dst[base0 + n] = o[n][0];
        dst[base1 + n] = o[n][1];
      }
    }
  }
};

}  // namespace pa
