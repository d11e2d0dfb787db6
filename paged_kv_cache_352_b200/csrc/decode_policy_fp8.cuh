// Tensor-core arithmetic policy of the paged-decode kernel over E4M3 caches.
#pragma once

#include <cuda.h>
#include <math.h>
#include <string.h>

#include "decode_policies.cuh"
#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {

// Four E4M3 codes (one word, low byte first) to two half pairs, exactly: codes
// 0, 1 in `lo` and 2, 3 in `hi`. The word splits into its 16-bit halves by a
// register move, which costs no shift for the upper pair (measured 12 % faster
// on the 8-bit CUDA-core decode than converting `w` and `w >> 16`).
__device__ __forceinline__ void e4m3x4_to_half2x2(uint32_t w, uint32_t& lo, uint32_t& hi) {
  asm("{\n\t.reg .b16 c01, c23;\n\tmov.b32 {c01, c23}, %2;\n\t"
      "cvt.rn.f16x2.e4m3x2 %0, c01;\n\tcvt.rn.f16x2.e4m3x2 %1, c23;\n\t}"
      : "=r"(lo), "=r"(hi)
      : "r"(w));
}

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
// so the S accumulator of lane j holds tokens j, j+4, j+8, j+12 of its head g.
//
// P.V as O^T = V^T P^T. The product runs transposed, with the value tile as the
// A operand (m-tiles of 16 head dimensions, k = tokens) and P^T as B (n = the 8
// query heads): 8 mma per block at d = 128 instead of 16, with no padding rows.
// B's k-slots 2j, 2j+1, 2j+8, 2j+9 are the lane's own tokens j, j+4, j+8, j+12,
// so its p's feed B as they are. For A the lane loads those four token rows at
// its 16 (d = 128) or 8 (d = 64) dimensions, base + 0 .. 15; row g of m-tile t
// is dimension base + 2t and row g + 8 is base + 2t + 1, so one byte permute
// of two rows' words gives a code pair per dimension, converted to the two
// half pairs of a0 / a1 (tokens j, j+4) or a2 / a3 (tokens j+8, j+12). The
// accumulator of m-tile t holds dimensions base + 2t, base + 2t + 1 of heads
// 2j, 2j + 1; their softmax factors come from lanes 4(2j), 4(2j + 1).
//
// Lane groups and dimensions: at d = 128 lane group g (lane / 4) owns dimensions
// 16 c(g) + 0 .. 15, c(g) = 4(g & 1) + (g >> 1), at d = 64 dimensions 8g + 0 .. 7.
// With 128-byte-swizzled tiles (d = 128, 2-D TMA) these choices make every K and
// V load of a warp bank-conflict free; d = 64 tiles arrive by 1-D bulk copies.
// Measured against the former product (P as the 16-row A operand, the value
// bytes transposed 4 x 4 per lane, 16 mma per block): long-context 275.3 ->
// 244.3 us, GQA 100.6 -> 88.6 us per launch over 8-bit caches.
template <typename T, int D, int G>
struct Fp8TensorPolicy {
  static constexpr int KSTEPS = D / 16;
  static constexpr int NTO = D / 8;    // output n-tiles
  static constexpr int MT = D / 16;    // m-tiles of O^T = V^T P^T (16 dimensions each)
  static constexpr int CPT = D / 64;   // 16-byte key chunks a lane reads per row
  static constexpr int kTileBytes = kBS * D;
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr bool kSwizzled = D == 128;
  static constexpr int kAlign = kSwizzled ? 1024 : 128;
  static constexpr int kScratchBytes = 0;
  static constexpr bool kTensorCores = true;
  static constexpr bool kTma2D = kSwizzled;
  static constexpr bool kFp8Cache = true;
  // Four CTAs per SM (128 registers; at most 20 bytes a thread spill). With the
  // transposed P.V product the policy needs about 140 registers; capped at 128,
  // 16 warps per SM measured faster than 12 warps at 142 registers: GQA 88.6 ->
  // 85.0 us, long-context 244.2 -> 242.0 us.
  static constexpr int kMinCtasPerSm = 4;
  static_assert(D == 64 || D == 128, "unsupported head_dim");

  int g, j;
  uint4 qraw[CPT][2];      // the lane's 16 * CPT query elements of row g (raw T)
  uint32_t qa[KSTEPS][2];  // f16 A fragments (slots 2j,2j+1 and 2j+8,2j+9)
  float m, l, row_scale;
  float o[MT][4];  // O^T m-tile mt: dims pi(mt, g), pi(mt, g + 8) x heads 2j, 2j + 1

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

  // The query row this lane holds (rows >= G are padding), and its load from a
  // row the caller located (nullptr: a zero row).
  __device__ __forceinline__ int q_row() const { return g; }
  __device__ __forceinline__ void load_q_row(const T* row) {
    const uint4* qrow = reinterpret_cast<const uint4*>(row);
#pragma unroll
    for (int h = 0; h < CPT; ++h) {
      qraw[h][0] = row ? __ldg(qrow + 2 * (j + 4 * h)) : make_uint4(0u, 0u, 0u, 0u);
      qraw[h][1] = row ? __ldg(qrow + 2 * (j + 4 * h) + 1) : make_uint4(0u, 0u, 0u, 0u);
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
    for (int t = 0; t < MT; ++t) o[t][0] = o[t][1] = o[t][2] = o[t][3] = 0.f;
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
        uint32_t b0, b1;
        e4m3x4_to_half2x2(word, b0, b1);
        MmaOps<__half>::run(sacc[nt], qa[kk][0], qa[kk][1], b0, b1);
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
    float alpha;
    const float mref = lazy_reference(m, bmax, alpha);
    const float p0 = exp2f(x[0][0] - mref), p1 = exp2f(x[0][1] - mref);
    const float p2 = exp2f(x[1][0] - mref), p3 = exp2f(x[1][1] - mref);
    l = fmaf(l, alpha, (p0 + p1) + (p2 + p3));
    if (__any_sync(0xffffffffu, alpha != 1.f)) {
      // this lane's outputs are heads 2j and 2j + 1, whose factors live in
      // lanes 4(2j) and 4(2j + 1)
      const float a0 = __shfl_sync(0xffffffffu, alpha, 8 * j);
      const float a1 = __shfl_sync(0xffffffffu, alpha, 8 * j + 4);
#pragma unroll
      for (int t = 0; t < MT; ++t) {
        o[t][0] *= a0;
        o[t][1] *= a1;
        o[t][2] *= a0;
        o[t][3] *= a1;
      }
    }
    uint32_t pa0, pa2;
    {
      const __half2 h0 = __floats2half2_rn(p0, p1);
      const __half2 h2 = __floats2half2_rn(p2, p3);
      memcpy(&pa0, &h0, 4);
      memcpy(&pa2, &h2, 4);
    }
    // ---- O^T += V^T P^T: A = V^T (m-tile rows are dimensions, k-slots 2j, 2j+1,
    // 2j+8, 2j+9 are tokens j, j+4, j+8, j+12), B = P^T (the lane's own p's:
    // pa0 = tokens j, j+4 and pa2 = j+8, j+12 of head g), N = the 8 heads. Row
    // g of m-tile mt is dimension base + 2mt, row g + 8 is base + 2mt + 1, where
    // the lane's 16 (d = 128) or 8 (d = 64) dimensions start at base.
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
    for (int t = 0; t < MT; ++t) {
      const int w = t >> 1;
      const uint32_t sel = (t & 1) ? 0x7362u : 0x5140u;  // bytes 2(t&1), 2(t&1)+1 of both rows
      uint32_t a0, a1, a2, a3;
      e4m3x4_to_half2x2(__byte_perm(vr[0][w], vr[1][w], sel), a0, a1);
      e4m3x4_to_half2x2(__byte_perm(vr[2][w], vr[3][w], sel), a2, a3);
      asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
          "{%8,%9}, {%0,%1,%2,%3};"
          : "+f"(o[t][0]), "+f"(o[t][1]), "+f"(o[t][2]), "+f"(o[t][3])
          : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(pa0), "r"(pa2));
    }
  }

  __device__ __forceinline__ void to_red(float* red_m, float* red_l, float* red_acc, int warp,
                                         int) {
    float lsum = l + __shfl_xor_sync(0xffffffffu, l, 1);
    lsum += __shfl_xor_sync(0xffffffffu, lsum, 2);
    if (g < G && j == 0) {
      red_m[warp * G + g] = m;
      red_l[warp * G + g] = lsum;
    }
    // O^T elements: dimensions base + 2t (+1) of heads 2j, 2j + 1
    const int base = D == 128 ? 16 * (4 * (g & 1) + (g >> 1)) : 8 * g;
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int h = 2 * j + e;
      if (h < G) {
        float* dst = red_acc + (warp * G + h) * D + base;
#pragma unroll
        for (int t = 0; t < MT; ++t) {
          dst[2 * t] = o[t][e];
          dst[2 * t + 1] = o[t][2 + e];
        }
      }
    }
  }
};

// Fp8TensorPairPolicy: the tensor-core policy over two blocks per loop step. A
// stage holds two blocks of the warp's list (each its K and V tiles); the step
// computes both score tiles (two independent mma chains), updates the running
// maximum, the rescale vote and the sum once for the 32 tokens, and adds both
// blocks' P.V. The arithmetic per token is the block step's; only the softmax
// reference moves once per pair instead of once per block (any reference gives
// the same softmax once the sums and rows agree with it).
template <typename T, int D, int G>
struct Fp8TensorPairPolicy : Fp8TensorPolicy<T, D, G> {
  using Base = Fp8TensorPolicy<T, D, G>;
  static constexpr int kTileBytes = Base::kTileBytes;
  static constexpr int kBlockBytes = Base::kStageBytes;  // one block's K and V tiles
  static constexpr int kStageBytes = 2 * kBlockBytes;    // a pair of blocks
  static constexpr bool kPairs = true;
  // 2 pair stages per warp: 64 KB of ring per 4-warp CTA, three CTAs per SM
  static constexpr int kMinCtasPerSm = 3;

  // The tile copies of one block into dst (the caller arms the barrier).
  static __device__ __forceinline__ void issue_block(const DecodeArgs& a, const CUtensorMap* tm_k,
                                                     const CUtensorMap* tm_v, unsigned char* dst,
                                                     uint64_t* bar, int phys, int kvh) {
    if constexpr (Base::kSwizzled) {
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

  // S = Q K^T of one block (columns: tokens (n >> 1) + 4(n & 1) + 8nt)
  __device__ __forceinline__ void scores(const unsigned char* Ks, float (&sacc)[2][2]) const {
    const int krow = (this->g >> 1) + 4 * (this->g & 1);
    uint4 kw[2][Base::CPT];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int h = 0; h < Base::CPT; ++h)
        kw[nt][h] = *reinterpret_cast<const uint4*>(
            Ks + Base::chunk_off(krow + 8 * nt, this->j + 4 * h));
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) sacc[nt][0] = sacc[nt][1] = 0.f;
#pragma unroll
    for (int kk = 0; kk < Base::KSTEPS; ++kk) {
      const int h = kk >> 2, w = kk & 3;
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        const uint32_t word = w == 0 ? kw[nt][h].x : w == 1 ? kw[nt][h].y
                            : w == 2 ? kw[nt][h].z : kw[nt][h].w;
        uint32_t b0, b1;
        e4m3x4_to_half2x2(word, b0, b1);
        MmaOps<__half>::run(sacc[nt], this->qa[kk][0], this->qa[kk][1], b0, b1);
      }
    }
  }

  // O^T += V^T P^T of one block (as in the block step)
  __device__ __forceinline__ void values(const unsigned char* Vs, int valid, uint32_t pa0,
                                         uint32_t pa2) {
    constexpr int VW = D == 128 ? 4 : 2;
    uint32_t vr[4][VW];
#pragma unroll
    for (int mm = 0; mm < 4; ++mm) {
      const int t = this->j + 4 * mm;
      if constexpr (D == 128) {
        const int c = 4 * (this->g & 1) + (this->g >> 1);
        const uint4 v = *reinterpret_cast<const uint4*>(Vs + Base::chunk_off(t, c));
        vr[mm][0] = v.x;
        vr[mm][1] = v.y;
        vr[mm][2] = v.z;
        vr[mm][3] = v.w;
      } else {
        const uint2 v = *reinterpret_cast<const uint2*>(Vs + t * D + 8 * this->g);
        vr[mm][0] = v.x;
        vr[mm][1] = v.y;
      }
    }
    if (valid < kBS) {
#pragma unroll
      for (int mm = 0; mm < 4; ++mm)
        if (this->j + 4 * mm >= valid) {
#pragma unroll
          for (int w = 0; w < VW; ++w) vr[mm][w] = 0u;
        }
    }
#pragma unroll
    for (int t = 0; t < Base::MT; ++t) {
      const int w = t >> 1;
      const uint32_t sel = (t & 1) ? 0x7362u : 0x5140u;
      uint32_t a0, a1, a2, a3;
      e4m3x4_to_half2x2(__byte_perm(vr[0][w], vr[1][w], sel), a0, a1);
      e4m3x4_to_half2x2(__byte_perm(vr[2][w], vr[3][w], sel), a2, a3);
      asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
          "{%8,%9}, {%0,%1,%2,%3};"
          : "+f"(this->o[t][0]), "+f"(this->o[t][1]), "+f"(this->o[t][2]), "+f"(this->o[t][3])
          : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(pa0), "r"(pa2));
    }
  }

  // Two blocks: stage sa (valid tokens va) and sb (vb; 0 when the pair has one block)
  __device__ __forceinline__ void block2(const unsigned char* sa, int va, const unsigned char* sb,
                                         int vb) {
    float s[2][2][2];  // [block][nt][e]
    scores(sa, s[0]);
    scores(sb, s[1]);
    float bmax = -INFINITY;
#pragma unroll
    for (int b = 0; b < 2; ++b) {
      const int valid = b ? vb : va;
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const bool ok = this->g < G && this->j + 4 * e + 8 * nt < valid;
          s[b][nt][e] = ok ? s[b][nt][e] * this->row_scale : -INFINITY;
          bmax = fmaxf(bmax, s[b][nt][e]);
        }
    }
    bmax = fmaxf(bmax, __shfl_xor_sync(0xffffffffu, bmax, 1));
    bmax = fmaxf(bmax, __shfl_xor_sync(0xffffffffu, bmax, 2));
    float alpha;
    const float mref = lazy_reference(this->m, bmax, alpha);
    float p[2][2][2];
    float psum = 0.f;
#pragma unroll
    for (int b = 0; b < 2; ++b)
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          p[b][nt][e] = exp2f(s[b][nt][e] - mref);
          psum += p[b][nt][e];
        }
    this->l = fmaf(this->l, alpha, psum);
    if (__any_sync(0xffffffffu, alpha != 1.f)) {
      const float a0 = __shfl_sync(0xffffffffu, alpha, 8 * this->j);
      const float a1 = __shfl_sync(0xffffffffu, alpha, 8 * this->j + 4);
#pragma unroll
      for (int t = 0; t < Base::MT; ++t) {
        this->o[t][0] *= a0;
        this->o[t][1] *= a1;
        this->o[t][2] *= a0;
        this->o[t][3] *= a1;
      }
    }
#pragma unroll
    for (int b = 0; b < 2; ++b) {
      uint32_t pa0, pa2;
      const __half2 h0 = __floats2half2_rn(p[b][0][0], p[b][0][1]);
      const __half2 h2 = __floats2half2_rn(p[b][1][0], p[b][1][1]);
      memcpy(&pa0, &h0, 4);
      memcpy(&pa2, &h2, 4);
      values((b ? sb : sa) + kTileBytes, b ? vb : va, pa0, pa2);
    }
  }
};

// ---------------------------------------------------------------------------
// CUDA cores over an E4M3 cache
// ---------------------------------------------------------------------------

// (d0, d1) = (a0 * b0 + d0, a1 * b1 + d1): sm_100's packed fp32 FMA, each half
// rounded exactly as a scalar fmaf.
__device__ __forceinline__ void ffma2(float& d0, float& d1, float a0, float a1, float b0,
                                      float b1) {
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rd, {%0, %1};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rd;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "+f"(d0), "+f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

// (d0, d1) *= (a, a) with sm_100's packed fp32 multiply.
__device__ __forceinline__ void fmul2(float& d0, float& d1, float a) {
  asm("{\n\t.reg .b64 ra, rd;\n\t"
      "mov.b64 ra, {%2, %2};\n\tmov.b64 rd, {%0, %1};\n\t"
      "mul.f32x2 rd, rd, ra;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "+f"(d0), "+f"(d1)
      : "f"(a));
}

// d + a.lo * b.lo + a.hi * b.hi for two packed halves each: sm_100's
// mixed-precision FMA takes half operands and an fp32 addend; a product of two
// halves is exact in fp32, so each step rounds once, as an fp32 fmaf would.
__device__ __forceinline__ float fma_h2_f32(uint32_t a, uint32_t b, float d) {
  asm("{\n\t.reg .f16 al, ah, bl, bh;\n\t"
      "mov.b32 {al, ah}, %1;\n\tmov.b32 {bl, bh}, %2;\n\t"
      "fma.rn.f32.f16 %0, al, bl, %0;\n\tfma.rn.f32.f16 %0, ah, bh, %0;\n\t}"
      : "+f"(d)
      : "r"(a), "r"(b));
  return d;
}

// Fp8CudaCorePolicy (one or two query heads per KV head): a lane holds 16 codes
// (one 16-byte shared-memory load) of a key or value row, so LPT = d/16 lanes
// cover a row, TPW = 32/LPT rows are read per warp pass and TPL = 16/TPW passes
// cover a tile. Codes widen to halves two at a time.
//   keys: q . k with half operands and fp32 accumulation. The query row is held
//     in half precision (an f16 row as it is; a bf16 row times 2^-k, k = 0
//     unless its largest magnitude is at or above 2^15, with 2^k folded into
//     its logit scale), so every product is exact and only the sums round, in
//     fp32, as they would with fp32 operands.
//   values: halves widened to fp32 and accumulated by packed fp32 FMAs.
// Measured against the generic CUDA-core policy over 8-bit tiles (8 codes per
// lane, scalar fp32 FMAs) on the 7B-like MHA batch: 0.099 ms against 0.129 ms
// per launch.
template <typename T, int D, int G>
struct Fp8CudaCorePolicy {
  static constexpr int LPT = D / 16;
  static constexpr int TPW = 32 / LPT;
  static constexpr int TPL = kBS / TPW;
  static constexpr int kTileBytes = kBS * D;
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kAlign = 128;
  static constexpr int kScratchBytes = G * kBS * 4;  // per warp: p values of one tile
  static constexpr bool kTensorCores = false;
  static constexpr bool kTma2D = false;
  static constexpr bool kFp8Cache = true;
  static constexpr int kMinCtasPerSm = 4;  // at most 128 registers a thread
  static_assert(G <= 2, "4 and 8 query heads per KV head use another policy");
  static_assert(D == 64 || D == 128, "unsupported head_dim");
  static_assert(LPT * TPW == 32 && TPL * TPW == kBS, "unsupported head_dim");

  int c, grp, own;
  bool writer;
  uint4 qraw[G][2];    // the lane's 16 query elements of each head (raw T)
  uint32_t qh[G][8];   // those elements as half pairs
  float row_scale[G];  // logit scale of each head's row
  float m[G], l[G], acc[G][16];

  __device__ __forceinline__ void init(int lane) {
    c = lane % LPT;
    grp = lane / LPT;
    own = own_index<TPL>(c);
    writer = c < TPL;
  }

  __device__ __forceinline__ void prefetch_q(const DecodeArgs& a, int s, int kvh) {
    const uint4* qrow = reinterpret_cast<const uint4*>(
        reinterpret_cast<const T*>(a.q) + ((size_t)s * a.num_q_heads + (size_t)kvh * G) * D +
        c * 16);
#pragma unroll
    for (int g = 0; g < G; ++g) {
      qraw[g][0] = __ldg(qrow + g * (D / 8));
      qraw[g][1] = __ldg(qrow + g * (D / 8) + 1);
    }
  }

  __device__ __forceinline__ void begin(float scale_log2) {
#pragma unroll
    for (int g = 0; g < G; ++g) {
      if constexpr (std::is_same<T, __half>::value) {
        const uint32_t w[8] = {qraw[g][0].x, qraw[g][0].y, qraw[g][0].z, qraw[g][0].w,
                               qraw[g][1].x, qraw[g][1].y, qraw[g][1].z, qraw[g][1].w};
#pragma unroll
        for (int e = 0; e < 8; ++e) qh[g][e] = w[e];
        row_scale[g] = scale_log2;
      } else {
        float f[16];
        Storage<T>::to_f32(qraw[g][0], *reinterpret_cast<float(*)[8]>(&f[0]));
        Storage<T>::to_f32(qraw[g][1], *reinterpret_cast<float(*)[8]>(&f[8]));
        float amax = 0.f;
#pragma unroll
        for (int e = 0; e < 16; ++e) amax = fmaxf(amax, fabsf(f[e]));
#pragma unroll
        for (int mask = 1; mask < LPT; mask <<= 1)
          amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, mask));
        const int k = amax >= 32768.f ? ilogbf(amax) - 14 : 0;
        const float down = exp2f((float)-k);
        row_scale[g] = scale_log2 * exp2f((float)k);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const __half2 h = __floats2half2_rn(f[2 * e] * down, f[2 * e + 1] * down);
          memcpy(&qh[g][e], &h, 4);
        }
      }
      m[g] = -INFINITY;
      l[g] = 0.f;
#pragma unroll
      for (int e = 0; e < 16; ++e) acc[g][e] = 0.f;
    }
  }

  static __device__ __forceinline__ void issue(const DecodeArgs& a, const CUtensorMap*,
                                               const CUtensorMap*, unsigned char* dst,
                                               uint64_t* bar, int phys, int kvh) {
    const size_t off = ((size_t)phys * a.num_kv_heads + kvh) * kTileBytes;
    mbar_arrive_expect_tx(bar, kStageBytes);
    bulk_copy_g2s(dst, static_cast<const unsigned char*>(a.k_cache) + off, kTileBytes, bar);
    bulk_copy_g2s(dst + kTileBytes, static_cast<const unsigned char*>(a.v_cache) + off, kTileBytes,
                  bar);
  }

  // 16 codes of a row (4 words) as 8 half pairs, element order kept.
  static __device__ __forceinline__ void widen_h(const uint4& raw, uint32_t (&h)[8]) {
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) e4m3x4_to_half2x2(w[q], h[2 * q], h[2 * q + 1]);
  }

  static __device__ __forceinline__ void widen_f(const uint4& raw, float (&f)[16]) {
    uint32_t h[8];
    widen_h(raw, h);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float2 x = half2_bits_to_float2(h[e]);
      f[2 * e] = x.x;
      f[2 * e + 1] = x.y;
    }
  }

  // One tile: tokens tok0 .. tok0+15 of which `valid` (>= 1) lie inside the context.
  __device__ __forceinline__ void block(unsigned char* stage, int valid, unsigned char* scratch) {
    float* wp = reinterpret_cast<float*>(scratch);
    const unsigned char* Ks = stage;
    const unsigned char* Vs = stage + kTileBytes;
    float part[G][TPL];
#pragma unroll
    for (int i = 0; i < TPL; ++i) {
      const int t = i * TPW + grp;
      const uint4 raw = *reinterpret_cast<const uint4*>(Ks + t * D + c * 16);
      uint32_t h[8];
      widen_h(raw, h);
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float d0 = 0.f, d1 = 0.f;  // two chains for latency
#pragma unroll
        for (int e = 0; e < 8; e += 2) {
          d0 = fma_h2_f32(qh[g][e], h[e], d0);
          d1 = fma_h2_f32(qh[g][e + 1], h[e + 1], d1);
        }
        part[g][i] = d0 + d1;
      }
    }
    const bool own_valid = own * TPW + grp < valid;
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float x = transpose_reduce<TPL, LPT>(part[g], c) * row_scale[g];
      x = own_valid ? x : -INFINITY;
      float bmax = x;
#pragma unroll
      for (int mask = 1; mask < TPL; mask <<= 1)
        bmax = fmaxf(bmax, __shfl_xor_sync(0xffffffffu, bmax, mask));
      const float mnew = fmaxf(m[g], bmax);
      const float mref = mnew == -INFINITY ? 0.f : mnew;
      const float alpha = exp2f(m[g] - mref);
      const float p = exp2f(x - mref);
      m[g] = mnew;
      if (writer) wp[(g * TPW + grp) * TPL + own] = p;
      l[g] *= alpha;
#pragma unroll
      for (int e = 0; e < 16; e += 2) fmul2(acc[g][e], acc[g][e + 1], alpha);
    }
    __syncwarp();
    const bool full = valid >= kBS;
#pragma unroll
    for (int i = 0; i < TPL; ++i) {
      const int t = i * TPW + grp;
      uint4 raw = *reinterpret_cast<const uint4*>(Vs + t * D + c * 16);
      // rows past the context may hold any codes (NaN included): read them as zeros
      if (!full && t >= valid) raw = make_uint4(0u, 0u, 0u, 0u);
      float vf[16];
      widen_f(raw, vf);
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float p = wp[(g * TPW + grp) * TPL + i];
        l[g] += p;
#pragma unroll
        for (int e = 0; e < 16; e += 2) ffma2(acc[g][e], acc[g][e + 1], p, p, vf[e], vf[e + 1]);
      }
    }
  }

  // Merge the warp's token groups, then leave the warp's state in shared memory.
  __device__ __forceinline__ void to_red(float* red_m, float* red_l, float* red_acc, int warp,
                                         int lane) {
#pragma unroll
    for (int mask = LPT; mask < 32; mask <<= 1) {
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float mo = __shfl_xor_sync(0xffffffffu, m[g], mask);
        const float lo = __shfl_xor_sync(0xffffffffu, l[g], mask);
        const float mn = fmaxf(m[g], mo);
        const float mref = mn == -INFINITY ? 0.f : mn;
        const float sa = exp2f(m[g] - mref), sb = exp2f(mo - mref);
        l[g] = l[g] * sa + lo * sb;
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float ao = __shfl_xor_sync(0xffffffffu, acc[g][e], mask);
          acc[g][e] = acc[g][e] * sa + ao * sb;
        }
        m[g] = mn;
      }
    }
    if (lane == 0) {
#pragma unroll
      for (int g = 0; g < G; ++g) {
        red_m[warp * G + g] = m[g];
        red_l[warp * G + g] = l[g];
      }
    }
    if (grp == 0) {
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float4* dst = reinterpret_cast<float4*>(red_acc + (warp * G + g) * D + c * 16);
#pragma unroll
        for (int e = 0; e < 4; ++e)
          dst[e] = make_float4(acc[g][4 * e], acc[g][4 * e + 1], acc[g][4 * e + 2],
                               acc[g][4 * e + 3]);
      }
    }
  }
};

}  // namespace pa
