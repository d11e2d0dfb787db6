// Arithmetic policies of the paged-decode kernel.
//
// Both policies consume one (block, KV head) tile pair per call — the keys and
// values of 16 consecutive tokens of one sequence — and keep a per-lane
// online-softmax state for the G query heads that share the KV head:
//   m  running maximum of the logits (base 2: q is pre-scaled by scale*log2 e)
//   l  running sum of exp2(logit - m)
//   acc / o  running sum of exp2(logit - m) * v
//
// CudaCorePolicy (G = 1, 2): fp32 FMAs. LPT = d/8 lanes cover one token row
// (16 bytes each), TPW = 32/LPT token groups per warp, TPL = 16/TPW tokens per
// lane. Partial q.k dot products are summed across the LPT lanes with a
// transposing butterfly that halves the live values at each exchange. Tiles
// arrive raw ([16][d] row-major) by 1-D bulk copies.
//
// TensorPolicy (G = 4, 8): warp-level mma.sync m16n8k16, fp32 accumulation.
// S = Q K^T takes the query heads as M (padded to 16) and the block's tokens as
// N. P V runs transposed, O^T = V^T P^T: the value tile, loaded transposed by
// ldmatrix, is the A operand (16 head dimensions by the 16 tokens) and P^T the B
// operand (N = 8 heads), whose k-slots are exactly the tokens a lane holds in
// its S accumulator, so the probabilities feed B from registers as they are and
// no accumulator row is padding (half the mma of P as a padded A operand). P
// enters as a 16-bit value plus its rounding residual, keeping ~16 significant
// bits. Tiles arrive by 2-D TMA tensor loads, 128-byte swizzled: token row t,
// 128-byte column half h at h*2048 + t*128, 16-byte chunks XOR-ed by t % 8, so
// ldmatrix fragment loads are bank-conflict free.
#pragma once

#include <cuda.h>
#include <math.h>

#include <type_traits>

#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {

constexpr int kBS = kBlockSize;

// ---------------------------------------------------------------------------
// CUDA cores
// ---------------------------------------------------------------------------

// Butterfly reduction that transposes as it sums. On entry each of the LPT
// lanes of a token group holds N partial sums (one per token). Afterwards each
// lane holds the full sum for token own_index<N>(c) in v[0].
template <int N, int LPT>
__device__ __forceinline__ float transpose_reduce(float (&v)[N], int c) {
  int n = N;
#pragma unroll
  for (int mask = 1; mask < LPT; mask <<= 1) {
    if (n > 1) {
      const bool upper = (c & mask) != 0;
#pragma unroll
      for (int k = 0; k < N / 2; ++k) {
        if (k < n / 2) {
          const float send = upper ? v[k] : v[k + n / 2];
          const float keep = upper ? v[k + n / 2] : v[k];
          v[k] = keep + __shfl_xor_sync(0xffffffffu, send, mask);
        }
      }
      n >>= 1;
    } else {
      v[0] += __shfl_xor_sync(0xffffffffu, v[0], mask);
    }
  }
  return v[0];
}

template <int N>
__device__ __forceinline__ int own_index(int c) {
  int idx = 0;
  int half = N / 2;
#pragma unroll
  for (int bit = 0; (1 << bit) < N; ++bit) {
    if (c & (1 << bit)) idx += half;
    half >>= 1;
  }
  return idx;
}

template <typename T, int D, int G, typename C = T>
struct CudaCorePolicy {
  using E = CacheElem<C>;
  static constexpr int LPT = D / 8;
  static constexpr int TPW = 32 / LPT;
  static constexpr int TPL = kBS / TPW;
  static constexpr int kTileElems = kBS * D;
  static constexpr int kTileBytes = kTileElems * E::kBytes;
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kAlign = 128;
  static constexpr int kScratchBytes = G * kBS * 4;  // per warp: p values of one block
  static constexpr bool kTensorCores = false;
  static constexpr bool kTma2D = false;
  static constexpr bool kFp8Cache = std::is_same<C, E4M3>::value;
  // Three CTAs fit an SM's shared memory with the default 4 x 2 tiles (at most
  // 170 registers a thread); the 4 and 8 query-head variants need more and are
  // left to the compiler (they are not the default path).
  static constexpr int kMinCtasPerSm = G > 2 ? 1 : 3;
  static_assert(LPT * TPW == 32 && TPL * TPW == kBS, "unsupported head_dim");

  int c, grp, own;
  bool writer;
  uint4 qnext[G];
  float qf[G][8];
  float m[G], l[G], acc[G][8];

  __device__ __forceinline__ void init(int lane) {
    c = lane % LPT;
    grp = lane / LPT;
    own = own_index<TPL>(c);
    writer = c < TPL;  // one lane per distinct token writes its p value
  }

  __device__ __forceinline__ void prefetch_q(const DecodeArgs& a, int s, int kvh) {
    const T* qrow =
        reinterpret_cast<const T*>(a.q) + ((size_t)s * a.num_q_heads + (size_t)kvh * G) * D;
#pragma unroll
    for (int g = 0; g < G; ++g) qnext[g] = __ldg(reinterpret_cast<const uint4*>(qrow + g * D + c * 8));
  }

  __device__ __forceinline__ void begin(float scale_log2) {
#pragma unroll
    for (int g = 0; g < G; ++g) {
      Storage<T>::to_f32(qnext[g], qf[g]);
#pragma unroll
      for (int k = 0; k < 8; ++k) qf[g][k] *= scale_log2;
      m[g] = -INFINITY;
      l[g] = 0.f;
#pragma unroll
      for (int k = 0; k < 8; ++k) acc[g][k] = 0.f;
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

  // One block: tokens tok0 .. tok0+15 of which `valid` (>= 1) lie inside the context.
  __device__ __forceinline__ void block(unsigned char* stage, int valid, unsigned char* scratch) {
    using Raw = typename E::Raw;
    float* wp = reinterpret_cast<float*>(scratch);
    const unsigned char* Ks = stage;
    const unsigned char* Vs = stage + kTileBytes;
    float part_dot[G][TPL];
#pragma unroll
    for (int i = 0; i < TPL; ++i) {
      const int t = i * TPW + grp;
      const Raw raw = *reinterpret_cast<const Raw*>(Ks + (t * D + c * 8) * E::kBytes);
      float kf[8];
      E::to_f32(raw, kf);
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float d = qf[g][0] * kf[0];
#pragma unroll
        for (int k = 1; k < 8; ++k) d = fmaf(qf[g][k], kf[k], d);
        part_dot[g][i] = d;
      }
    }
    const bool own_valid = own * TPW + grp < valid;
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float x = transpose_reduce<TPL, LPT>(part_dot[g], c);
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
      for (int k = 0; k < 8; ++k) acc[g][k] *= alpha;
    }
    __syncwarp();
    const bool full = valid >= kBS;
#pragma unroll
    for (int i = 0; i < TPL; ++i) {
      const int t = i * TPW + grp;
      const Raw raw = *reinterpret_cast<const Raw*>(Vs + (t * D + c * 8) * E::kBytes);
      float vf[8];
      E::to_f32(raw, vf);
      if (!full && t >= valid) {
#pragma unroll
        for (int k = 0; k < 8; ++k) vf[k] = 0.f;  // slots past the context may hold anything
      }
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float p = wp[(g * TPW + grp) * TPL + i];
        l[g] += p;
#pragma unroll
        for (int k = 0; k < 8; ++k) acc[g][k] = fmaf(p, vf[k], acc[g][k]);
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
        for (int k = 0; k < 8; ++k) {
          const float ao = __shfl_xor_sync(0xffffffffu, acc[g][k], mask);
          acc[g][k] = acc[g][k] * sa + ao * sb;
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
        float* dst = red_acc + (warp * G + g) * D + c * 8;
#pragma unroll
        for (int k = 0; k < 8; ++k) dst[k] = acc[g][k];
      }
    }
  }
};

// ---------------------------------------------------------------------------
// Tensor cores
// ---------------------------------------------------------------------------

template <typename T>
struct MmaOps;

// d[0..3] += A B for a whole m16n8k16 tile (A rows 0-15 real), f32 accumulate.
template <typename T>
__device__ __forceinline__ void mma_full(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  if constexpr (std::is_same<T, __half>::value) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
  } else {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
  }
}

template <>
struct MmaOps<__half> {
  // d[0..1] += A B for rows 0-7 of the m16n8k16 tile. Rows 8-15 of A are zero
  // padding (at most 8 query heads per KV head), so their accumulators are fed
  // zeros and their results discarded instead of occupying registers.
  static __device__ __forceinline__ void run(float (&d)[2], uint32_t a0, uint32_t a2,
                                             uint32_t b0, uint32_t b1) {
    asm("{\n\t.reg .f32 dead0, dead1;\n\t"
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,dead0,dead1}, {%2,%3,%4,%5}, "
        "{%6,%7}, {%8,%9,%10,%10};\n\t}"
        : "=f"(d[0]), "=f"(d[1])
        : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1), "f"(d[0]), "f"(d[1]), "f"(0.f));
  }
  // (x0, x1) as a packed 16-bit pair `hi` plus the packed rounding residual `lo`
  static __device__ __forceinline__ void split(float x0, float x1, uint32_t& hi, uint32_t& lo) {
    const __half2 h = __floats2half2_rn(x0, x1);
    const float2 r = __half22float2(h);
    const __half2 t = __floats2half2_rn(x0 - r.x, x1 - r.y);
    hi = *reinterpret_cast<const uint32_t*>(&h);
    lo = *reinterpret_cast<const uint32_t*>(&t);
  }
};

template <>
struct MmaOps<__nv_bfloat16> {
  // d[0..1] += A B for rows 0-7 of the m16n8k16 tile. Rows 8-15 of A are zero
  // padding (at most 8 query heads per KV head), so their accumulators are fed
  // zeros and their results discarded instead of occupying registers.
  static __device__ __forceinline__ void run(float (&d)[2], uint32_t a0, uint32_t a2,
                                             uint32_t b0, uint32_t b1) {
    asm("{\n\t.reg .f32 dead0, dead1;\n\t"
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,dead0,dead1}, {%2,%3,%4,%5}, "
        "{%6,%7}, {%8,%9,%10,%10};\n\t}"
        : "=f"(d[0]), "=f"(d[1])
        : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1), "f"(d[0]), "f"(d[1]), "f"(0.f));
  }
  static __device__ __forceinline__ void split(float x0, float x1, uint32_t& hi, uint32_t& lo) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
    const float2 r = __bfloat1622float2(h);
    const __nv_bfloat162 t = __floats2bfloat162_rn(x0 - r.x, x1 - r.y);
    hi = *reinterpret_cast<const uint32_t*>(&h);
    lo = *reinterpret_cast<const uint32_t*>(&t);
  }
};

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1,
                                              uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// 2-D TMA tile load (x = column element, y = row), completion on `bar`.
__device__ __forceinline__ void tma_load_2d(void* smem_dst, const CUtensorMap* map, int x, int y,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3}], [%4];" ::"r"(smem_addr(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_addr(bar))
      : "memory");
}

constexpr int kHalfBytes = kBS * 128;  // one 128-byte column half of a 16-token tile

// Byte offset of 16-byte chunk `chunk` (0 .. d/8-1) of token row `t` in a swizzled tile.
__device__ __forceinline__ uint32_t swz(int t, int chunk) {
  return (uint32_t)((chunk >> 3) * kHalfBytes + t * 128 + (((chunk & 7) ^ (t & 7)) << 4));
}

template <typename T, int D, int G>
struct TensorPolicy {
  static constexpr int HALVES = D / 64;
  static constexpr int kTileBytes = HALVES * kHalfBytes;
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kAlign = 1024;  // 128-byte swizzled TMA destinations
  static constexpr int kScratchBytes = 0;
  static constexpr bool kTensorCores = true;
  static constexpr bool kTma2D = true;
  static constexpr bool kFp8Cache = false;
  static constexpr int kMinCtasPerSm = 3;
  static constexpr int KSTEPS = D / 16;
  static constexpr int MT = D / 16;  // m-tiles of O^T = V^T P^T (16 dimensions each)

  int r, j, mi, ri;
  uint32_t qa[KSTEPS][2];  // A operand of S = Q K^T: row r, columns kk*16 + 2j (+1) and +8
  float m, l;
  // O^T m-tile t: [0] / [1] dimension 16t + r of heads 2j / 2j + 1, [2] / [3]
  // dimension 16t + r + 8 of the same heads
  float o[MT][4];
  float scale_log2;

  __device__ __forceinline__ void init(int lane) {
    r = lane >> 2;  // query head within the group (rows >= G are padding)
    j = lane & 3;
    mi = lane >> 3;  // which 8x8 matrix this lane addresses in ldmatrix.x4
    ri = lane & 7;   // row of that matrix
  }

  __device__ __forceinline__ void prefetch_q(const DecodeArgs& a, int s, int kvh) {
    const uint32_t* qrow = reinterpret_cast<const uint32_t*>(
        reinterpret_cast<const T*>(a.q) + ((size_t)s * a.num_q_heads + (size_t)kvh * G + r) * D);
#pragma unroll
    for (int kk = 0; kk < KSTEPS; ++kk) {
      qa[kk][0] = r < G ? __ldg(qrow + kk * 8 + j) : 0u;
      qa[kk][1] = r < G ? __ldg(qrow + kk * 8 + 4 + j) : 0u;
    }
  }

  // The query row this lane holds (rows >= G are padding), and its load from a
  // row the caller located (nullptr: a zero row).
  __device__ __forceinline__ int q_row() const { return r; }
  __device__ __forceinline__ void load_q_row(const T* row) {
    const uint32_t* qrow = reinterpret_cast<const uint32_t*>(row);
#pragma unroll
    for (int kk = 0; kk < KSTEPS; ++kk) {
      qa[kk][0] = row ? __ldg(qrow + kk * 8 + j) : 0u;
      qa[kk][1] = row ? __ldg(qrow + kk * 8 + 4 + j) : 0u;
    }
  }

  __device__ __forceinline__ void begin(float scale) {
    scale_log2 = scale;
    m = -INFINITY;
    l = 0.f;
#pragma unroll
    for (int t = 0; t < MT; ++t) o[t][0] = o[t][1] = o[t][2] = o[t][3] = 0.f;
  }

  static __device__ __forceinline__ void issue(const DecodeArgs& a, const CUtensorMap* tm_k,
                                               const CUtensorMap* tm_v, unsigned char* dst,
                                               uint64_t* bar, int phys, int kvh) {
    const int y = (phys * a.num_kv_heads + kvh) * kBS;
    mbar_arrive_expect_tx(bar, kStageBytes);
#pragma unroll
    for (int h = 0; h < HALVES; ++h) {
      tma_load_2d(dst + h * kHalfBytes, tm_k, h * 64, y, bar);
      tma_load_2d(dst + kTileBytes + h * kHalfBytes, tm_v, h * 64, y, bar);
    }
  }

  __device__ __forceinline__ void block(unsigned char* stage, int valid, unsigned char*) {
    unsigned char* Vs = stage + kTileBytes;
    if (valid < kBS) {
      // slots past the context may hold anything (even NaN patterns): zero them in V
      for (int idx = (threadIdx.x & 31); idx < (kBS - valid) * (D / 8); idx += 32) {
        const int t = valid + idx / (D / 8);
        *reinterpret_cast<uint4*>(Vs + swz(t, idx % (D / 8))) = make_uint4(0, 0, 0, 0);
      }
      __syncwarp();
    }
    // ---- S = Q K^T (rows: query heads, columns: the block's 16 tokens)
    float sacc[2][2];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) sacc[nt][0] = sacc[nt][1] = 0.f;
    const uint32_t kbase = smem_addr(stage);
#pragma unroll
    for (int kk = 0; kk < KSTEPS; ++kk) {
      const int t = (mi >> 1) * 8 + ri;
      uint32_t b00, b01, b10, b11;
      ldsm_x4(kbase + swz(t, kk * 2 + (mi & 1)), b00, b01, b10, b11);
      MmaOps<T>::run(sacc[0], qa[kk][0], qa[kk][1], b00, b01);
      MmaOps<T>::run(sacc[1], qa[kk][0], qa[kk][1], b10, b11);
    }
    // ---- online softmax for row r (4 of the 16 columns live in this lane)
    float x[2][2];
    float bmax = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const bool ok = r < G && nt * 8 + 2 * j + e < valid;
        x[nt][e] = ok ? sacc[nt][e] * scale_log2 : -INFINITY;
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
    // P^T as the B operand: k-slots 2j, 2j + 1 (and + 8) are this lane's own
    // tokens of row r, so its probabilities feed B as they are
    uint32_t pa0, pa0_lo, pa2, pa2_lo;
    MmaOps<T>::split(p0, p1, pa0, pa0_lo);
    MmaOps<T>::split(p2, p3, pa2, pa2_lo);
    // ---- O^T += V^T P^T: A = V^T (rows: 16 dimensions, k: the block's tokens),
    // loaded transposed by ldmatrix from the [token][dim] tile; N = the 8 heads
    const uint32_t vbase = smem_addr(Vs);
#pragma unroll
    for (int t = 0; t < MT; ++t) {
      uint32_t a0, a1, a2, a3;
      ldsm_x4_trans(vbase + swz((mi >> 1) * 8 + ri, 2 * t + (mi & 1)), a0, a1, a2, a3);
      mma_full<T>(o[t], a0, a1, a2, a3, pa0_lo, pa2_lo);
      mma_full<T>(o[t], a0, a1, a2, a3, pa0, pa2);
    }
  }

  __device__ __forceinline__ void to_red(float* red_m, float* red_l, float* red_acc, int warp,
                                         int) {
    // the 4 lanes of a row each hold 4 of every block's 16 columns
    float lsum = l + __shfl_xor_sync(0xffffffffu, l, 1);
    lsum += __shfl_xor_sync(0xffffffffu, lsum, 2);
    if (r < G && j == 0) {
      red_m[warp * G + r] = m;
      red_l[warp * G + r] = lsum;
    }
    // O^T elements: dimensions 16t + r (+ 8) of heads 2j, 2j + 1
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int h = 2 * j + e;
      if (h < G) {
        float* dst = red_acc + (warp * G + h) * D + r;
#pragma unroll
        for (int t = 0; t < MT; ++t) {
          dst[16 * t] = o[t][e];
          dst[16 * t + 8] = o[t][2 + e];
        }
      }
    }
  }
};

}  // namespace pa
