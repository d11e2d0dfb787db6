// Paged decode with tensor cores, for grouped-query attention (G query heads
// per KV head, G = 2, 4 or 8).
//
// With G query heads reading one KV head, a 16-token block yields a real
// contraction: S = Q K^T is [G x 16] over head_dim, and O += P V is [G x d]
// over 16 tokens. At G = 8 that is 8 flops per byte of K/V, more than the
// fp32 FMA pipe keeps up with at HBM speed, so both products run on the tensor
// cores with warp-level mma.sync m16n8k16 (fp32 accumulation), the query heads
// as the M dimension (padded to 16) and tokens / head_dim as N. The
// FlashAttention-2 register layout lets the S accumulator be reused directly as
// the A operand of P V, so P never leaves registers. The operands of one mma
// share a type, so P (in [0, 1]) enters P V in the storage type: as a rounded
// 16-bit value plus a second mma with its rounding residual, which keeps the
// product accurate to ~2^-16 of P instead of 2^-8 for bf16.
//
// Data movement: as in the CUDA-core kernel each warp owns a ring of stages
// filled by lane 0, but with 2-D TMA tensor loads that land every (block, KV
// head) tile 128-byte swizzled: tile row t (one token, 128-byte column half h)
// sits at h*2048 + t*128 with its 16-byte chunks XOR-ed by t % 8. That makes
// the ldmatrix fragment loads (K as the B operand of S, V transposed as the B
// operand of P V) bank-conflict free, which the raw 256-byte-row layout is not.
//
// The grid, split-KV partitions and merge are those of the CUDA-core kernel
// (finish_partition); the reduction order depends on logical positions only.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <atomic>
#include <mutex>

#include "decode_common.cuh"
#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {
namespace {

constexpr int BS = kBlockSize;
constexpr int kHalfBytes = BS * 128;  // one 128-byte column half of a 16-token tile

template <typename T>
struct Mma;

template <>
struct Mma<__half> {
  static __device__ __forceinline__ void run(float (&d)[4], uint32_t a0, uint32_t a2,
                                             uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1));
  }
  // (x0, x1) as a packed pair `hi` plus the packed rounding residual `lo`
  static __device__ __forceinline__ void split(float x0, float x1, uint32_t& hi, uint32_t& lo) {
    const __half2 h = __floats2half2_rn(x0, x1);
    const float2 r = __half22float2(h);
    const __half2 t = __floats2half2_rn(x0 - r.x, x1 - r.y);
    hi = *reinterpret_cast<const uint32_t*>(&h);
    lo = *reinterpret_cast<const uint32_t*>(&t);
  }
};

template <>
struct Mma<__nv_bfloat16> {
  static __device__ __forceinline__ void run(float (&d)[4], uint32_t a0, uint32_t a2,
                                             uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1));
  }
  // (x0, x1) as a packed pair `hi` plus the packed rounding residual `lo`
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

// Byte offset of 16-byte chunk `chunk` (0 .. d/8-1) of token row `t` in a swizzled tile.
__device__ __forceinline__ uint32_t swz(int t, int chunk) {
  return (uint32_t)((chunk >> 3) * kHalfBytes + t * 128 + (((chunk & 7) ^ (t & 7)) << 4));
}

template <int D, int WARPS, int STAGES, int G>
struct MmaPlan {
  static constexpr int HALVES = D / 64;
  static constexpr int TILE_BYTES = HALVES * kHalfBytes;
  static constexpr int STAGE_BYTES = 2 * TILE_BYTES;
  static constexpr size_t kTiles = size_t(WARPS) * STAGES * STAGE_BYTES;
  static constexpr size_t kBars = size_t(WARPS) * STAGES * sizeof(uint64_t);
  static constexpr size_t kRed = size_t(WARPS) * G * (D + 2) * sizeof(float);
  static constexpr size_t kAlign = 1024;  // 128-byte swizzled TMA destinations
  static constexpr size_t kFixed = kAlign + kTiles + kBars;
  static_assert(kRed <= kTiles, "merge buffers must fit in the tile ring");
};

template <typename T, int D, int G, int WARPS, int STAGES>
__global__ void __launch_bounds__(WARPS * 32)
    paged_decode_mma_kernel(const DecodeArgs a, const __grid_constant__ CUtensorMap tm_k,
                            const __grid_constant__ CUtensorMap tm_v) {
  using Plan = MmaPlan<D, WARPS, STAGES, G>;
  constexpr int KSTEPS = D / 16;
  constexpr int NTO = D / 8;  // output n-tiles of 8 columns
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + Plan::kAlign - 1) & ~(uintptr_t)(Plan::kAlign - 1));

  const int kvh = blockIdx.x;
  const int part = blockIdx.y;
  const int s = blockIdx.z;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int r = lane >> 2;  // query head within the group (rows >= G are padding)
  const int j = lane & 3;

  int ctx = a.context_lens[s];
  if (ctx < 0 || ctx > a.max_blocks_per_seq * BS || ctx > a.max_context_len) {
    if (part == 0 && kvh == 0 && threadIdx.x == 0) report(a.dev_error, PA_DEVERR_CONTEXT_RANGE);
    ctx = 0;
  }
  const int nblk = (ctx + BS - 1) / BS;
  const int nparts = (nblk + a.part_blocks - 1) / a.part_blocks;
  if (part >= (nparts > 0 ? nparts : 1)) return;

  T* out_rows = reinterpret_cast<T*>(a.out) + ((size_t)s * a.num_q_heads + (size_t)kvh * G) * D;
  if (nblk == 0) {
    for (int i = threadIdx.x; i < G * D; i += blockDim.x) out_rows[i] = Storage<T>::from_f32(0.f);
    return;
  }

  const int b_begin = part * a.part_blocks;
  const int b_end = min(nblk, b_begin + a.part_blocks);
  const int nlocal = b_end - b_begin;
  const int my_n = nlocal > warp ? (nlocal - warp + WARPS - 1) / WARPS : 0;

  unsigned char* wtiles = smem + (size_t)warp * STAGES * Plan::STAGE_BYTES;
  uint64_t* wbars = reinterpret_cast<uint64_t*>(smem + Plan::kTiles) + warp * STAGES;
  if (lane == 0) {
#pragma unroll
    for (int st = 0; st < STAGES; ++st) mbar_init(&wbars[st], 1);
    mbar_init_fence();
  }
  __syncwarp();

  const int32_t* table = a.block_tables + (size_t)s * a.max_blocks_per_seq;
  auto issue = [&](int jj) {
    const int b = b_begin + warp + jj * WARPS;
    const int phys = __ldg(table + b);
    uint64_t* bar = &wbars[jj % STAGES];
    if ((unsigned)phys >= (unsigned)a.num_blocks) {
      report(a.dev_error, PA_DEVERR_BLOCK_RANGE);
      mbar_arrive(bar);
      return;
    }
    unsigned char* dst = wtiles + (size_t)(jj % STAGES) * Plan::STAGE_BYTES;
    const int y = (phys * a.num_kv_heads + kvh) * BS;
    mbar_arrive_expect_tx(bar, Plan::STAGE_BYTES);
#pragma unroll
    for (int h = 0; h < Plan::HALVES; ++h) {
      tma_load_2d(dst + h * kHalfBytes, &tm_k, h * 64, y, bar);
      tma_load_2d(dst + Plan::TILE_BYTES + h * kHalfBytes, &tm_v, h * 64, y, bar);
    }
  };
  if (lane == 0) {
    for (int jj = 0; jj < STAGES && jj < my_n; ++jj) issue(jj);
  }
  int issued = my_n < STAGES ? my_n : STAGES;

  // A operand of S = Q K^T: row r of the group, columns kk*16 + 2j (+1) and +8
  uint32_t qa[KSTEPS][2];
  {
    const uint32_t* qrow = reinterpret_cast<const uint32_t*>(
        reinterpret_cast<const T*>(a.q) + ((size_t)s * a.num_q_heads + (size_t)kvh * G + r) * D);
#pragma unroll
    for (int kk = 0; kk < KSTEPS; ++kk) {
      qa[kk][0] = r < G ? __ldg(qrow + kk * 8 + j) : 0u;
      qa[kk][1] = r < G ? __ldg(qrow + kk * 8 + 4 + j) : 0u;
    }
  }

  float m = -INFINITY, l = 0.f;
  float o[NTO][4];
#pragma unroll
  for (int n = 0; n < NTO; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;

  const int mi = lane >> 3;  // which 8x8 matrix this lane addresses in ldmatrix.x4
  const int ri = lane & 7;   // row of that matrix
  bool aborted = false;
  int jj = 0;
  for (; jj < my_n; ++jj) {
    const int st = jj % STAGES;
    if (!mbar_wait_bounded(&wbars[st], (uint32_t)((jj / STAGES) & 1))) {
      if (lane == 0) report(a.dev_error, PA_DEVERR_WAIT_TIMEOUT);
      aborted = true;
      break;
    }
    const int b = b_begin + warp + jj * WARPS;
    const int phys = __ldg(table + b);
    if ((unsigned)phys < (unsigned)a.num_blocks) {
      unsigned char* Ks = wtiles + (size_t)st * Plan::STAGE_BYTES;
      unsigned char* Vs = Ks + Plan::TILE_BYTES;
      const int tok0 = b * BS;
      const int valid = ctx - tok0;  // tokens of this block inside the context (>= 1)
      if (valid < BS) {
        // slots past the context may hold anything (even NaN patterns): zero them in V
        for (int idx = lane; idx < (BS - valid) * (D / 8); idx += 32) {
          const int t = valid + idx / (D / 8);
          *reinterpret_cast<uint4*>(Vs + swz(t, idx % (D / 8))) = make_uint4(0, 0, 0, 0);
        }
        __syncwarp();
      }

      // ---- S = Q K^T (rows: query heads, columns: the block's 16 tokens)
      float sacc[2][4];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) sacc[nt][0] = sacc[nt][1] = sacc[nt][2] = sacc[nt][3] = 0.f;
      const uint32_t kbase = smem_addr(Ks);
#pragma unroll
      for (int kk = 0; kk < KSTEPS; ++kk) {
        const int t = (mi >> 1) * 8 + ri;
        uint32_t b00, b01, b10, b11;
        ldsm_x4(kbase + swz(t, kk * 2 + (mi & 1)), b00, b01, b10, b11);
        Mma<T>::run(sacc[0], qa[kk][0], qa[kk][1], b00, b01);
        Mma<T>::run(sacc[1], qa[kk][0], qa[kk][1], b10, b11);
      }

      // ---- online softmax for row r (4 of the 16 columns live in this lane)
      float x[2][2];
      float bmax = -INFINITY;
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const bool ok = r < G && nt * 8 + 2 * j + e < valid;
          x[nt][e] = ok ? sacc[nt][e] * a.scale_log2 : -INFINITY;
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
      // P enters the tensor cores as a 16-bit pair plus its rounding residual,
      // so P V carries ~16 significant bits of P instead of 8 (bf16) or 11 (fp16).
      uint32_t pa0, pa0_lo, pa2, pa2_lo;
      Mma<T>::split(p0, p1, pa0, pa0_lo);
      Mma<T>::split(p2, p3, pa2, pa2_lo);

      // ---- O += P V (V transposed into the B operand by ldmatrix.trans)
      const uint32_t vbase = smem_addr(Vs);
#pragma unroll
      for (int pp = 0; pp < NTO / 2; ++pp) {
        const int t = (mi & 1) * 8 + ri;
        uint32_t v0, v1, v2, v3;
        ldsm_x4_trans(vbase + swz(t, 2 * pp + (mi >> 1)), v0, v1, v2, v3);
        o[2 * pp][0] *= alpha;
        o[2 * pp][1] *= alpha;
        o[2 * pp + 1][0] *= alpha;
        o[2 * pp + 1][1] *= alpha;
        Mma<T>::run(o[2 * pp], pa0_lo, pa2_lo, v0, v1);
        Mma<T>::run(o[2 * pp + 1], pa0_lo, pa2_lo, v2, v3);
        Mma<T>::run(o[2 * pp], pa0, pa2, v0, v1);
        Mma<T>::run(o[2 * pp + 1], pa0, pa2, v2, v3);
      }
    }
    __syncwarp();
    if (lane == 0 && jj + STAGES < my_n) {
      fence_proxy_async_smem();
      issue(jj + STAGES);
    }
    if (jj + STAGES < my_n) issued = jj + STAGES + 1;
  }
  if (aborted) {
    for (int k = jj; k < issued; ++k)
      mbar_wait_bounded(&wbars[k % STAGES], (uint32_t)((k / STAGES) & 1));
  }

  // row sums: the 4 lanes of a row each hold 4 of every block's 16 columns
  l += __shfl_xor_sync(0xffffffffu, l, 1);
  l += __shfl_xor_sync(0xffffffffu, l, 2);

  __syncthreads();  // every warp is done with its tiles: reuse them for the merge
  float* red_m = reinterpret_cast<float*>(smem);
  float* red_l = red_m + WARPS * G;
  float* red_acc = red_l + WARPS * G;
  if (r < G) {
    if (j == 0) {
      red_m[warp * G + r] = m;
      red_l[warp * G + r] = l;
    }
    float* dst = red_acc + (warp * G + r) * D + 2 * j;
#pragma unroll
    for (int n = 0; n < NTO; ++n) {
      dst[n * 8] = o[n][0];
      dst[n * 8 + 1] = o[n][1];
    }
  }
  __syncthreads();
  finish_partition<T, D, G, WARPS>(a, smem, red_m, red_l, red_acc, s, kvh, part, nparts,
                                   out_rows);
}

constexpr int kWarps = 4;
constexpr int kStages = 3;
constexpr size_t kSmemLimit = 200 * 1024;
constexpr int kMaxDevices = 64;

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      p = nullptr;
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }();
  return fn;
}

// A cache array [num_blocks][Hkv][16][d] viewed as rows of d elements, read in
// 16-row x 64-column boxes with 128-byte swizzling.
cudaError_t make_cache_map(CUtensorMap* map, const void* base, long long rows, int head_dim,
                           int dtype) {
  auto fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  cuuint64_t dims[2] = {(cuuint64_t)head_dim, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)head_dim * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)BS};
  cuuint32_t estr[2] = {1, 1};
  const CUresult res = fn(
      map, dtype == PA_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
      const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
      CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return res == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

template <typename T, int D, int G>
cudaError_t launch_mma_typed(const DecodeArgs& a, int dtype, cudaStream_t stream) {
  using Plan = MmaPlan<D, kWarps, kStages, G>;
  const size_t wts_bytes = Plan::kAlign + (size_t)a.max_parts * G * sizeof(float);
  const size_t smem = Plan::kFixed > wts_bytes ? Plan::kFixed : wts_bytes;
  if (smem > kSmemLimit) return cudaErrorInvalidConfiguration;
  const long long rows = (long long)a.num_blocks * a.num_kv_heads * BS;
  if (rows > 0x7fffffffLL) return cudaErrorInvalidValue;  // TMA row coordinates are int32
  CUtensorMap tk, tv;
  cudaError_t e = make_cache_map(&tk, a.k_cache, rows, D, dtype);
  if (e != cudaSuccess) return e;
  e = make_cache_map(&tv, a.v_cache, rows, D, dtype);
  if (e != cudaSuccess) return e;
  auto kern = paged_decode_mma_kernel<T, D, G, kWarps, kStages>;
  static std::atomic<bool> ready[kMaxDevices];
  int dev = 0;
  e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  if (!ready[dev].load(std::memory_order_acquire)) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemLimit);
    if (e != cudaSuccess) return e;
    ready[dev].store(true, std::memory_order_release);
  }
  dim3 grid(a.num_kv_heads, a.max_parts, a.num_seqs);
  kern<<<grid, kWarps * 32, smem, stream>>>(a, tk, tv);
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t launch_mma_group(const DecodeArgs& a, int group, int dtype, cudaStream_t stream) {
  switch (group) {
    case 2: return launch_mma_typed<T, D, 2>(a, dtype, stream);
    case 4: return launch_mma_typed<T, D, 4>(a, dtype, stream);
    case 8: return launch_mma_typed<T, D, 8>(a, dtype, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

cudaError_t launch_paged_decode_mma(const DecodeArgs& a, int head_dim, int group, int dtype,
                                    cudaStream_t stream) {
  if (dtype == PA_F16) {
    if (head_dim == 64) return launch_mma_group<__half, 64>(a, group, dtype, stream);
    if (head_dim == 128) return launch_mma_group<__half, 128>(a, group, dtype, stream);
  } else {
    if (head_dim == 64) return launch_mma_group<__nv_bfloat16, 64>(a, group, dtype, stream);
    if (head_dim == 128) return launch_mma_group<__nv_bfloat16, 128>(a, group, dtype, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace pa
