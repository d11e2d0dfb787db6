// Paged decode attention (sm_100a): one launch computes
//   out[s][h] = softmax(scale * K_s q[s][h]) V_s
// with K_s / V_s read block by block through the sequence's block table
// ("vLLM: PagedAttention and continuous batching", direct answer;
// "PagedAttention: The vLLM Paper", "The Core Idea", block-table figure note).
//
// Work decomposition
//   grid = (num_kv_heads, max_parts, num_seqs); one CTA per (sequence, KV head,
//   split-KV partition of part_blocks blocks). The CTA serves all G query heads
//   that read this KV head, so each K/V byte is fetched from HBM once.
//
// Data movement
//   A (block, KV head) tile is 16 tokens x head_dim contiguous elements (4 KiB at
//   d=128, fp16/bf16). Each warp owns a private ring of STAGES shared-memory
//   slots; lane 0 fills a slot with two 1-D bulk async copies (K tile, V tile)
//   that complete on the slot's mbarrier. Warp w handles the partition's blocks
//   w, w+WARPS, ... so a CTA keeps WARPS*STAGES tiles of K+V in flight with no
//   cross-warp synchronisation in the main loop.
//
// Arithmetic (fp32, CUDA cores)
//   Lane layout in a warp: LPT = d/8 lanes cover one token row (8 elements =
//   16 bytes each), TPW = 32/LPT token groups per warp, TPL = 16/TPW tokens per
//   lane per block. q.K partial dot products are reduced across the LPT lanes
//   with a transposing butterfly (log2(TPL) exchange steps that halve the number
//   of live values, then plain adds), so a block's 16 logits cost
//   TPL-1+log2(LPT/TPL) shuffles per query head instead of 16*log2(LPT).
//   Online softmax runs in base 2 (q pre-scaled by scale*log2 e). Each token
//   group keeps its own (m, l, acc); groups, warps and partitions merge by
//   rescaling to the common maximum.
//
// Split-KV
//   A sequence with one partition writes `out` directly. Otherwise each CTA
//   writes (m, l, acc) to the workspace, bumps a per-(sequence, KV head) counter,
//   and the CTA that finishes last merges all partitions and resets the counter
//   to zero. The merge walks partitions in logical order, so the result does not
//   depend on which CTA finishes last or where blocks sit physically.
#include <cuda_runtime.h>
#include <math.h>

#include <atomic>
#include <cstdlib>
#include <cstring>

#include "decode_common.cuh"
#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {
namespace {

constexpr int BS = kBlockSize;

template <int D>
struct Geometry {
  static constexpr int LPT = D / 8;     // lanes per token row
  static constexpr int TPW = 32 / LPT;  // token groups per warp
  static constexpr int TPL = BS / TPW;  // tokens per lane per block
  static constexpr int TILE_ELEMS = BS * D;
  static constexpr int TILE_BYTES = TILE_ELEMS * 2;
  static constexpr int STAGE_BYTES = 2 * TILE_BYTES;
  static constexpr int LOG_TPL = TPL == 8 ? 3 : (TPL == 4 ? 2 : (TPL == 2 ? 1 : 0));
  static_assert(LPT * TPW == 32 && TPL * TPW == BS, "unsupported head_dim");
};

template <int WARPS, int STAGES, int D, int G>
struct SmemPlan {
  using Geo = Geometry<D>;
  static constexpr size_t kTiles = size_t(WARPS) * STAGES * Geo::STAGE_BYTES;
  static constexpr size_t kBars = size_t(WARPS) * STAGES * sizeof(uint64_t);
  static constexpr size_t kPbuf = size_t(WARPS) * G * BS * sizeof(float);
  // Cross-warp merge buffers alias the tile ring once the main loop is over.
  static constexpr size_t kRed = size_t(WARPS) * G * (D + 2) * sizeof(float);
  static constexpr size_t kFixed = kTiles + kBars + kPbuf;
  static_assert(kRed <= kTiles, "merge buffers must fit in the tile ring");
};

// Butterfly reduction that transposes as it sums. On entry each of the LPT
// lanes of a token group holds N partial sums (one per token). After the call,
// every lane holds the full sum for token index own_index(c) in v[0].
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

// Token index (within the lane's TPL tokens) whose sum transpose_reduce leaves in a lane.
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

template <typename T, int D, int G, int WARPS, int STAGES>
__global__ void __launch_bounds__(WARPS * 32)
    paged_decode_kernel(const DecodeArgs a) {
  using Geo = Geometry<D>;
  using Plan = SmemPlan<WARPS, STAGES, D, G>;
  constexpr int LPT = Geo::LPT, TPW = Geo::TPW, TPL = Geo::TPL;
  extern __shared__ __align__(128) unsigned char smem[];

  const int kvh = blockIdx.x;
  const int part = blockIdx.y;
  const int s = blockIdx.z;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int c = lane % LPT;    // 16-byte column of the token row
  const int grp = lane / LPT;  // token group within the warp

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

  unsigned char* tiles = smem;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Plan::kTiles);
  float* pbuf = reinterpret_cast<float*>(smem + Plan::kTiles + Plan::kBars);
  unsigned char* wtiles = tiles + (size_t)warp * STAGES * Geo::STAGE_BYTES;
  uint64_t* wbars = bars + warp * STAGES;
  float* wp = pbuf + warp * G * BS;

  if (lane == 0) {
#pragma unroll
    for (int st = 0; st < STAGES; ++st) mbar_init(&wbars[st], 1);
    mbar_init_fence();
  }
  __syncwarp();

  const int32_t* table = a.block_tables + (size_t)s * a.max_blocks_per_seq;
  const T* kbase = reinterpret_cast<const T*>(a.k_cache) + (size_t)kvh * Geo::TILE_ELEMS;
  const T* vbase = reinterpret_cast<const T*>(a.v_cache) + (size_t)kvh * Geo::TILE_ELEMS;
  const size_t block_stride = (size_t)a.num_kv_heads * Geo::TILE_ELEMS;

  // lane 0: start the copies of this warp's j-th block into stage j % STAGES
  auto issue = [&](int j) {
    const int b = b_begin + warp + j * WARPS;
    const int phys = __ldg(table + b);
    uint64_t* bar = &wbars[j % STAGES];
    if ((unsigned)phys >= (unsigned)a.num_blocks) {
      report(a.dev_error, PA_DEVERR_BLOCK_RANGE);
      mbar_arrive(bar);  // complete the phase without data; the block is skipped
      return;
    }
    unsigned char* dst = wtiles + (size_t)(j % STAGES) * Geo::STAGE_BYTES;
    mbar_arrive_expect_tx(bar, Geo::STAGE_BYTES);
    bulk_copy_g2s(dst, kbase + (size_t)phys * block_stride, Geo::TILE_BYTES, bar);
    bulk_copy_g2s(dst + Geo::TILE_BYTES, vbase + (size_t)phys * block_stride, Geo::TILE_BYTES,
                  bar);
  };

  int issued = 0;
  if (lane == 0) {
    for (int j = 0; j < STAGES && j < my_n; ++j) issue(j);
  }
  issued = my_n < STAGES ? my_n : STAGES;

  // this lane's slice of the G query rows, pre-scaled into the base-2 domain
  float qf[G][8];
  {
    const T* qrow = reinterpret_cast<const T*>(a.q) + ((size_t)s * a.num_q_heads + (size_t)kvh * G) * D;
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const uint4 raw = __ldg(reinterpret_cast<const uint4*>(qrow + g * D + c * 8));
      Storage<T>::to_f32(raw, qf[g]);
#pragma unroll
      for (int k = 0; k < 8; ++k) qf[g][k] *= a.scale_log2;
    }
  }

  float m[G], l[G], acc[G][8];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    m[g] = -INFINITY;
    l[g] = 0.f;
#pragma unroll
    for (int k = 0; k < 8; ++k) acc[g][k] = 0.f;
  }

  const int own = own_index<TPL>(c);
  const bool writer = c < TPL;  // one lane per distinct token writes its p value
  bool aborted = false;
  int j = 0;
  for (; j < my_n; ++j) {
    const int st = j % STAGES;
    if (!mbar_wait_bounded(&wbars[st], (uint32_t)((j / STAGES) & 1))) {
      if (lane == 0) report(a.dev_error, PA_DEVERR_WAIT_TIMEOUT);
      aborted = true;
      break;
    }
    const int b = b_begin + warp + j * WARPS;
    const int phys = __ldg(table + b);
    if ((unsigned)phys < (unsigned)a.num_blocks) {
      const T* Ks = reinterpret_cast<const T*>(wtiles + (size_t)st * Geo::STAGE_BYTES);
      const T* Vs = Ks + Geo::TILE_ELEMS;
      const int tok0 = b * BS;

      // ---- logits: partial dot products over this lane's 8 columns
      float part_dot[G][TPL];
#pragma unroll
      for (int i = 0; i < TPL; ++i) {
        const int t = i * TPW + grp;
        const uint4 raw = *reinterpret_cast<const uint4*>(Ks + t * D + c * 8);
        float kf[8];
        Storage<T>::to_f32(raw, kf);
#pragma unroll
        for (int g = 0; g < G; ++g) {
          float acc_dot = qf[g][0] * kf[0];
#pragma unroll
          for (int k = 1; k < 8; ++k) acc_dot = fmaf(qf[g][k], kf[k], acc_dot);
          part_dot[g][i] = acc_dot;
        }
      }
      const bool own_valid = tok0 + own * TPW + grp < ctx;
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

      // ---- P.V over this lane's TPL tokens and 8 columns
      const bool full = tok0 + BS <= ctx;
#pragma unroll
      for (int i = 0; i < TPL; ++i) {
        const int t = i * TPW + grp;
        const uint4 raw = *reinterpret_cast<const uint4*>(Vs + t * D + c * 8);
        float vf[8];
        Storage<T>::to_f32(raw, vf);
        if (!full && tok0 + t >= ctx) {
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
    __syncwarp();
    if (lane == 0 && j + STAGES < my_n) {
      fence_proxy_async_smem();
      issue(j + STAGES);
    }
    if (j + STAGES < my_n) issued = j + STAGES + 1;
  }
  if (aborted) {
    // drain the copies still in flight into this warp's ring before leaving it
    for (int jj = j; jj < issued; ++jj)
      mbar_wait_bounded(&wbars[jj % STAGES], (uint32_t)((jj / STAGES) & 1));
  }

  // ---- merge the token groups of this warp
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

  // ---- merge warps through shared memory (reusing the tile ring)
  __syncthreads();
  float* red_m = reinterpret_cast<float*>(smem);            // [WARPS][G]
  float* red_l = red_m + WARPS * G;                         // [WARPS][G]
  float* red_acc = red_l + WARPS * G;                       // [WARPS][G][D]
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
  __syncthreads();

  finish_partition<T, D, G, WARPS>(a, smem, red_m, red_l, red_acc, s, kvh, part, nparts,
                                   out_rows);
}

constexpr size_t kDecodeSmemLimit = 200 * 1024;
constexpr int kMaxDevices = 64;

template <typename T, int D, int G, int WARPS, int STAGES>
cudaError_t launch_typed(const DecodeArgs& a, cudaStream_t stream) {
  using Plan = SmemPlan<WARPS, STAGES, D, G>;
  const size_t wts_bytes = (size_t)a.max_parts * G * sizeof(float);
  const size_t smem = Plan::kFixed > wts_bytes ? Plan::kFixed : wts_bytes;
  if (smem > kDecodeSmemLimit) return cudaErrorInvalidConfiguration;
  auto kern = paged_decode_kernel<T, D, G, WARPS, STAGES>;
  // The opt-in limit is a ceiling, not a reservation: set it once per device.
  static std::atomic<bool> ready[kMaxDevices];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  if (!ready[dev].load(std::memory_order_acquire)) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kDecodeSmemLimit);
    if (e != cudaSuccess) return e;
    ready[dev].store(true, std::memory_order_release);
  }
  dim3 grid(a.num_kv_heads, a.max_parts, a.num_seqs);
  kern<<<grid, WARPS * 32, smem, stream>>>(a);
  return cudaGetLastError();
}

// Warps per CTA x stages per warp. The default is 4 x 3; PA_DECODE_TILE="WxS"
// selects another built shape for A/B measurements (4x2, 2x3, 2x4, 8x2).
int tile_variant() {
  static const int v = [] {
    const char* e = getenv("PA_DECODE_TILE");
    if (!e) return 0;
    if (!strcmp(e, "4x2")) return 1;
    if (!strcmp(e, "2x3")) return 2;
    if (!strcmp(e, "2x4")) return 3;
    if (!strcmp(e, "8x2")) return 4;
    return 0;
  }();
  return v;
}

template <typename T, int D, int G>
cudaError_t launch_tiles(const DecodeArgs& a, cudaStream_t stream) {
  switch (tile_variant()) {
    case 1: return launch_typed<T, D, G, 4, 2>(a, stream);
    case 2: return launch_typed<T, D, G, 2, 3>(a, stream);
    case 3: return launch_typed<T, D, G, 2, 4>(a, stream);
    case 4: return launch_typed<T, D, G, 8, 2>(a, stream);
    default: return launch_typed<T, D, G, 4, 3>(a, stream);
  }
}

template <typename T, int D>
cudaError_t launch_group(const DecodeArgs& a, int group, cudaStream_t stream) {
  switch (group) {
    case 1: return launch_tiles<T, D, 1>(a, stream);
    case 2: return launch_typed<T, D, 2, 4, 3>(a, stream);
    case 4: return launch_typed<T, D, 4, 4, 3>(a, stream);
    case 8: return launch_typed<T, D, 8, 4, 3>(a, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

// Which arithmetic path serves a query-head group: tensor cores from G = 4 up
// (the q.K / P.V tiles are then real contractions), CUDA cores below.
// PA_DECODE_PATH=cuda_cores or =tensor overrides the choice for A/B measurements.
bool use_tensor_path(int group) {
  static const int forced = [] {
    const char* e = getenv("PA_DECODE_PATH");
    if (e && !strcmp(e, "cuda_cores")) return 0;
    if (e && !strcmp(e, "tensor")) return 1;
    return -1;
  }();
  if (group < 2) return false;
  if (forced >= 0) return forced == 1;
  return group >= 4;
}

cudaError_t launch_paged_decode(const DecodeArgs& a, int head_dim, int group, int dtype,
                                cudaStream_t stream) {
  if (use_tensor_path(group)) return launch_paged_decode_mma(a, head_dim, group, dtype, stream);
  if (dtype == PA_F16) {
    if (head_dim == 64) return launch_group<__half, 64>(a, group, stream);
    if (head_dim == 128) return launch_group<__half, 128>(a, group, stream);
  } else {
    if (head_dim == 64) return launch_group<__nv_bfloat16, 64>(a, group, stream);
    if (head_dim == 128) return launch_group<__nv_bfloat16, 128>(a, group, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace pa
