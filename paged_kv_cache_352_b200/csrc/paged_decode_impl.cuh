// Paged-decode kernel template and its launcher, instantiated once per
// (storage type, head_dim) in paged_decode_<type>_d<dim>.cu, and per
// (query type, head_dim) over E4M3 caches in paged_decode_<type>_d<dim>_e4m3.cu.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <math.h>

#include <atomic>
#include <cstdlib>
#include <cstring>
#include <type_traits>

#include "decode_common.cuh"
#include "decode_merge.cuh"
#include "decode_policies.cuh"
#include "decode_policy_fp8.cuh"
#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {
namespace {

// Register budget hint: each policy names the resident CTAs per SM its kernels
// are compiled for (launch bounds) with 4-warp CTAs, hence the registers a
// thread may use; other CTA sizes keep the same resident threads per SM.
template <class P, int WARPS>
constexpr int min_ctas_hint() {
  return P::kMinCtasPerSm * 4 / WARPS > 0 ? P::kMinCtasPerSm * 4 / WARPS : 1;
}

// One CTA's work: (KV head kvh, partition part) of the sequence that grid row z
// serves. The body of paged_decode_kernel, and of the prefix half of the
// cascade's two-part kernel (kGroupRows: z is a shared-prefix group, whose
// table, context and query rows are located through a.grp_*).
template <class P, typename T, int D, int G, int WARPS, int STAGES, bool kGroupRows = false>
__device__ __forceinline__ void decode_unit(const DecodeArgs& a, const CUtensorMap* tm_k,
                                            const CUtensorMap* tm_v, int kvh, int part, int z) {
  // Every input may come from the kernel ahead in the stream. A group unit reads
  // only the caller's inputs: the kernel ahead of it (the cascade's prepare) has
  // itself waited for everything before it, before letting this launch start.
  if constexpr (!kGroupRows) grid_dependency_wait();
  allow_dependents();
  constexpr size_t kRing = size_t(WARPS) * STAGES * P::kStageBytes;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + P::kAlign - 1) & ~(uintptr_t)(P::kAlign - 1));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int s = a.seq_order ? __ldg(a.seq_order + z) : z;
  if ((unsigned)s >= (unsigned)a.num_seqs) {
    if (part == 0 && kvh == 0 && threadIdx.x == 0) report(a.dev_error, PA_DEVERR_CONTEXT_RANGE);
    return;
  }

  // Independent loads first, so their latencies overlap: the context length,
  // this warp's first 32 block-table entries (lane i holds the entry of the
  // warp's block i; entries past the sequence are padding, never used) and q.
  const int32_t* table;
  int ctx;
  if constexpr (kGroupRows) {
    // the leader's table over the group's full prefix blocks
    int leader = __ldg(a.grp_members + (size_t)s * a.grp_size);
    int pb = __ldg(a.grp_prefix_blocks + s);
    if ((unsigned)leader >= (unsigned)a.grp_src_seqs || pb < 1 || pb > a.grp_max_prefix_blocks ||
        pb * kBS > a.max_context_len) {
      leader = 0;  // a rejected group (its members are decoded without it)
      pb = 0;
    }
    table = a.block_tables + (size_t)leader * a.max_blocks_per_seq;
    ctx = pb * kBS;
  } else {
    table = a.block_tables + (size_t)s * a.max_blocks_per_seq;
    ctx = __ldg(a.context_lens + s);
  }
  const int b_begin = part * a.part_blocks;
  int win_base = 0;  // the window covers this warp's blocks win_base .. win_base + 31
  int win = -1;
  {
    const int idx = b_begin + warp + lane * WARPS;
    if (idx < a.max_blocks_per_seq) win = __ldg(table + idx);
  }
  P pol;
  pol.init(lane);
  if constexpr (kGroupRows) {
    // stacked row r: head r % grp_heads of member slot r / grp_heads
    const int r = pol.q_row();
    const T* row = nullptr;
    if (r < G) {
      const int slot = r / a.grp_heads;
      const int m = __ldg(a.grp_members + (size_t)s * a.grp_size + slot);
      if ((unsigned)m < (unsigned)a.grp_src_seqs)
        row = reinterpret_cast<const T*>(a.q) +
              (((size_t)m * a.num_kv_heads + kvh) * a.grp_heads + (r - slot * a.grp_heads)) * D;
    }
    pol.load_q_row(row);
  } else {
    pol.prefetch_q(a, s, kvh);
  }

  if (ctx < 0 || ctx > a.max_blocks_per_seq * kBS || ctx > a.max_context_len) {
    if (part == 0 && kvh == 0 && threadIdx.x == 0) report(a.dev_error, PA_DEVERR_CONTEXT_RANGE);
    ctx = 0;  // flagged; the sequence yields a zero output
  }
  const int nblk = (ctx + kBS - 1) / kBS;
  const int nparts = (nblk + a.part_blocks - 1) / a.part_blocks;
  if (part >= (nparts > 0 ? nparts : 1)) return;
  T* out_rows = reinterpret_cast<T*>(a.out) + ((size_t)s * a.num_q_heads + (size_t)kvh * G) * D;
  if (nblk == 0) {
    if (!a.states_only)
      for (int i = threadIdx.x; i < G * D; i += blockDim.x) out_rows[i] = Storage<T>::from_f32(0.f);
    return;
  }
  const int nlocal = min(nblk, b_begin + a.part_blocks) - b_begin;
  const int my_n = nlocal > warp ? (nlocal - warp + WARPS - 1) / WARPS : 0;

  unsigned char* wring = smem + (size_t)warp * STAGES * P::kStageBytes;
  uint64_t* wbars = reinterpret_cast<uint64_t*>(smem + kRing) + warp * STAGES;
  int* wvalid = reinterpret_cast<int*>(smem + kRing + WARPS * STAGES * sizeof(uint64_t)) +
                warp * STAGES;
  constexpr size_t kHead = kRing + size_t(WARPS) * STAGES * (sizeof(uint64_t) + sizeof(int));
  unsigned char* scratch =
      smem + ((kHead + 127) & ~size_t(127)) + (size_t)warp * P::kScratchBytes;
  if (lane == 0) {
#pragma unroll
    for (int st = 0; st < STAGES; ++st) mbar_init(&wbars[st], 1);
    mbar_init_fence();
  }
  __syncwarp();

  // Start the copies of this warp's j-th block into stage j % STAGES. Called by
  // every lane (the table entry comes from the window by shuffle); lane 0 copies
  // and records in wvalid whether the stage holds a block to compute.
  auto issue = [&](int j) {
    if (j >= win_base + 32) {
      win_base = j & ~31;
      const int idx = b_begin + warp + (win_base + lane) * WARPS;
      win = win_base + lane < my_n ? __ldg(table + idx) : -1;
    }
    const int phys = __shfl_sync(0xffffffffu, win, j - win_base);
    if (lane == 0) {
      const int st = j % STAGES;
      uint64_t* bar = &wbars[st];
      const bool ok = (unsigned)phys < (unsigned)a.num_blocks;
      wvalid[st] = ok;  // published to the consumers by the arrive below
      if (a.stall_first_block && j == 0) {
        mbar_arrive_expect_tx(bar, 16);  // test hook: bytes that no copy will bring
      } else if (!ok) {
        report(a.dev_error, PA_DEVERR_BLOCK_RANGE);
        mbar_arrive(bar);  // complete the phase without data; the block is skipped
      } else {
        P::issue(a, tm_k, tm_v, wring + (size_t)st * P::kStageBytes, bar, phys, kvh);
      }
    }
  };
  for (int j = 0; j < STAGES && j < my_n; ++j) issue(j);
  int issued = my_n < STAGES ? my_n : STAGES;
  pol.begin(a.scale_log2);

  // test hook: the first stage was armed without a copy; its wait runs out
  bool aborted = a.stall_first_block && my_n > 0 &&
                 !mbar_wait_bounded(&wbars[0], 0u, a.wait_limit_ns);
  if (aborted && lane == 0) report(a.dev_error, PA_DEVERR_WAIT_TIMEOUT);
  int j = 0;
  for (; !aborted && j < my_n; ++j) {
    const int st = j % STAGES;
    if (!mbar_wait_bounded(&wbars[st], (uint32_t)((j / STAGES) & 1))) {
      if (lane == 0) report(a.dev_error, PA_DEVERR_WAIT_TIMEOUT);
      aborted = true;
      break;
    }
    const int b = b_begin + warp + j * WARPS;
    if (wvalid[st]) pol.block(wring + (size_t)st * P::kStageBytes, ctx - b * kBS, scratch);
    __syncwarp();
    if (j + STAGES < my_n) {
      if (lane == 0) fence_proxy_async_smem();  // this stage's reads precede its next copy
      issue(j + STAGES);
      issued = j + STAGES + 1;
    }
  }
  if (aborted) {
    // drain the copies still in flight into this warp's ring before leaving it
    // (a stage the test hook armed without a copy has none)
    for (int k = j; k < issued; ++k)
      if (!(a.stall_first_block && k == 0))
        mbar_wait_bounded(&wbars[k % STAGES], (uint32_t)((k / STAGES) & 1));
  }

  // merge the warps through shared memory, reusing the tile ring
  __syncthreads();
  float* red_m = reinterpret_cast<float*>(smem);  // [WARPS][G]
  float* red_l = red_m + WARPS * G;                // [WARPS][G]
  float* red_acc = red_l + WARPS * G;              // [WARPS][G][D]
  pol.to_red(red_m, red_l, red_acc, warp, lane);
  __syncthreads();
  finish_partition<T, D, G, WARPS>(a, red_m, red_m, red_l, red_acc, s, kvh, part, nparts,
                                   out_rows);
}

template <class P, typename T, int D, int G, int WARPS, int STAGES>
__global__ void __launch_bounds__(WARPS * 32, (min_ctas_hint<P, WARPS>()))
    paged_decode_kernel(const DecodeArgs a, const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v) {
  decode_unit<P, T, D, G, WARPS, STAGES>(a, &tm_k, &tm_v, blockIdx.x, blockIdx.y, blockIdx.z);
}

// One CTA's work with one KV head per warp: warp w serves KV head kvh0 + w of
// partition `part` of the sequence grid row z serves, streams the whole
// partition through its own ring and leaves its state (m, l, unnormalised rows)
// in the workspace: a states-only decode whose warps never wait for each
// other. The warps of a CTA read the same table entries and have the same
// number of blocks. Used for the cascade's own blocks: short runs of blocks per
// (sequence, KV head), WARPS of them per CTA instead of one.
template <class P, typename T, int D, int G, int WARPS, int STAGES>
__device__ __forceinline__ void decode_heads_unit(const DecodeArgs& a, const CUtensorMap* tm_k,
                                                  const CUtensorMap* tm_v, int kvh0, int part,
                                                  int z) {
  grid_dependency_wait();
  allow_dependents();
  constexpr size_t kRing = size_t(WARPS) * STAGES * P::kStageBytes;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + P::kAlign - 1) & ~(uintptr_t)(P::kAlign - 1));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int kvh = kvh0 + warp;
  const int s = a.seq_order ? __ldg(a.seq_order + z) : z;
  if ((unsigned)s >= (unsigned)a.num_seqs) {
    if (part == 0 && kvh0 == 0 && threadIdx.x == 0) report(a.dev_error, PA_DEVERR_CONTEXT_RANGE);
    return;
  }
  if (kvh >= a.num_kv_heads) return;  // the whole warp; no barrier spans warps here
  const int32_t* table = a.block_tables + (size_t)s * a.max_blocks_per_seq;
  const int b_begin = part * a.part_blocks;
  int ctx = __ldg(a.context_lens + s);
  int win = -1;  // lane i holds the table entry of the warp's block win_base + i
  {
    const int idx = b_begin + lane;
    if (lane < a.part_blocks && idx < a.max_blocks_per_seq) win = __ldg(table + idx);
  }
  P pol;
  pol.init(lane);
  pol.prefetch_q(a, s, kvh);
  if (ctx < 0 || ctx > a.max_blocks_per_seq * kBS || ctx > a.max_context_len) {
    if (part == 0 && kvh == 0 && lane == 0) report(a.dev_error, PA_DEVERR_CONTEXT_RANGE);
    ctx = 0;
  }
  const int nblk = (ctx + kBS - 1) / kBS;
  const int nparts = (nblk + a.part_blocks - 1) / a.part_blocks;
  if (part >= nparts) return;  // a sequence with no blocks leaves no state
  const int my_n = min(nblk, b_begin + a.part_blocks) - b_begin;

  unsigned char* wring = smem + (size_t)warp * STAGES * P::kStageBytes;
  uint64_t* wbars = reinterpret_cast<uint64_t*>(smem + kRing) + warp * STAGES;
  int* wvalid = reinterpret_cast<int*>(smem + kRing + WARPS * STAGES * sizeof(uint64_t)) +
                warp * STAGES;
  constexpr size_t kHead = kRing + size_t(WARPS) * STAGES * (sizeof(uint64_t) + sizeof(int));
  unsigned char* scratch =
      smem + ((kHead + 127) & ~size_t(127)) + (size_t)warp * P::kScratchBytes;
  if (lane == 0) {
#pragma unroll
    for (int st = 0; st < STAGES; ++st) mbar_init(&wbars[st], 1);
    mbar_init_fence();
  }
  __syncwarp();

  int win_base = 0;
  auto issue = [&](int j) {
    if (j >= win_base + 32) {
      win_base = j & ~31;
      win = win_base + lane < my_n ? __ldg(table + b_begin + win_base + lane) : -1;
    }
    const int phys = __shfl_sync(0xffffffffu, win, j - win_base);
    if (lane == 0) {
      const int st = j % STAGES;
      uint64_t* bar = &wbars[st];
      const bool ok = (unsigned)phys < (unsigned)a.num_blocks;
      wvalid[st] = ok;
      if (a.stall_first_block && j == 0) {
        mbar_arrive_expect_tx(bar, 16);  // test hook: bytes that no copy will bring
      } else if (!ok) {
        report(a.dev_error, PA_DEVERR_BLOCK_RANGE);
        mbar_arrive(bar);
      } else {
        P::issue(a, tm_k, tm_v, wring + (size_t)st * P::kStageBytes, bar, phys, kvh);
      }
    }
  };
  for (int j = 0; j < STAGES && j < my_n; ++j) issue(j);
  int issued = my_n < STAGES ? my_n : STAGES;
  pol.begin(a.scale_log2);

  bool aborted = a.stall_first_block && my_n > 0 &&
                 !mbar_wait_bounded(&wbars[0], 0u, a.wait_limit_ns);
  if (aborted && lane == 0) report(a.dev_error, PA_DEVERR_WAIT_TIMEOUT);
  int j = 0;
  for (; !aborted && j < my_n; ++j) {
    const int st = j % STAGES;
    if (!mbar_wait_bounded(&wbars[st], (uint32_t)((j / STAGES) & 1))) {
      if (lane == 0) report(a.dev_error, PA_DEVERR_WAIT_TIMEOUT);
      aborted = true;
      break;
    }
    if (wvalid[st])
      pol.block(wring + (size_t)st * P::kStageBytes, ctx - (b_begin + j) * kBS, scratch);
    __syncwarp();
    if (j + STAGES < my_n) {
      if (lane == 0) fence_proxy_async_smem();
      issue(j + STAGES);
      issued = j + STAGES + 1;
    }
  }
  if (aborted) {
    for (int k = j; k < issued; ++k)
      if (!(a.stall_first_block && k == 0))
        mbar_wait_bounded(&wbars[k % STAGES], (uint32_t)((k / STAGES) & 1));
  }
  // the partition's state straight from registers: rows [G] of m, l and [G][D] of acc
  const size_t row = (((size_t)s * a.num_kv_heads + kvh) * a.max_parts + part) * G;
  pol.to_red(a.ws_m + row, a.ws_l + row, a.ws_acc + row * D, 0, lane);
}

template <class P1, class P2, int WARPS>
constexpr int min_ctas_hint2() {
  return min_ctas_hint<P1, WARPS>() < min_ctas_hint<P2, WARPS>() ? min_ctas_hint<P1, WARPS>()
                                                                 : min_ctas_hint<P2, WARPS>();
}

// The cascade's two decodes in one launch: CTAs [0, n1) serve `a1` (the
// groups' shared prefixes, members' query heads stacked, read through the group
// descriptors; one CTA per KV head and partition, its warps on alternate blocks) and the rest serve `a2` (every
// sequence's own blocks, states only; one warp per KV head, WARPS KV heads per
// CTA), each CTA index split into (KV head or head group, partition, sequence)
// with the first fastest. The long prefix partitions are scheduled first and
// the short own-block CTAs fill the SMs behind them, so the launch has one tail
// instead of two.
template <class P1, int G1, class P2, int G2, typename T, int D, int WARPS, int STAGES>
__global__ void __launch_bounds__(WARPS * 32, (min_ctas_hint2<P1, P2, WARPS>()))
    cascade_decode_kernel(const DecodeArgs a1, const DecodeArgs a2,
                          const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v) {
  const int hkv = a1.num_kv_heads;
  const int hg = (hkv + WARPS - 1) / WARPS;  // KV-head groups of the own-block half
  const int n1 = hkv * a1.max_parts * a1.num_seqs;
  int i = blockIdx.x;
  if (i < n1) {
    decode_unit<P1, T, D, G1, WARPS, STAGES, true>(a1, &tm_k, &tm_v, i % hkv,
                                                   (i / hkv) % a1.max_parts,
                                                   i / (hkv * a1.max_parts));
  } else {
    i -= n1;
    decode_heads_unit<P2, T, D, G2, WARPS, STAGES>(a2, &tm_k, &tm_v, (i % hg) * WARPS,
                                                   (i / hg) % a2.max_parts,
                                                   i / (hg * a2.max_parts));
  }
}

// Whether a policy computes two blocks per loop step (P::kPairs, P::block2).
template <class P, class = void>
struct has_pairs : std::false_type {};
template <class P>
struct has_pairs<P, std::void_t<decltype(P::kPairs)>> : std::bool_constant<P::kPairs> {};

// Split-KV with one warp per partition, for short partitions (at most
// kWarpPartMaxBlocks blocks): warp w of CTA (kvh, y, z) streams partition
// y * WARPS + w of sequence seq_order[z] through its own ring and leaves that
// partition's state (m, l, unnormalised rows) in the workspace; no warp waits
// for another. merge_partitions_kernel then writes every output. Compared with
// one CTA per partition, each pipeline ramp and state write is amortised over
// WARPS times more blocks, and no CTA-wide merge runs per partition. A policy
// with kPairs takes two blocks per loop step (one ring stage and one barrier
// for both, one P::block2 call).
template <class P, typename T, int D, int G, int WARPS, int STAGES>
__global__ void __launch_bounds__(WARPS * 32, (min_ctas_hint<P, WARPS>()))
    paged_decode_warp_parts_kernel(const DecodeArgs a, const __grid_constant__ CUtensorMap tm_k,
                                   const __grid_constant__ CUtensorMap tm_v) {
  grid_dependency_wait();
  allow_dependents();
  constexpr size_t kRing = size_t(WARPS) * STAGES * P::kStageBytes;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + P::kAlign - 1) & ~(uintptr_t)(P::kAlign - 1));
  const int kvh = blockIdx.x;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int part = blockIdx.y * WARPS + warp;
  const int s = a.seq_order ? __ldg(a.seq_order + blockIdx.z) : (int)blockIdx.z;
  if ((unsigned)s >= (unsigned)a.num_seqs) {
    if (blockIdx.y == 0 && kvh == 0 && threadIdx.x == 0) report(a.dev_error, PA_DEVERR_CONTEXT_RANGE);
    return;
  }
  const int32_t* table = a.block_tables + (size_t)s * a.max_blocks_per_seq;
  const int b_begin = part * a.part_blocks;
  int ctx = __ldg(a.context_lens + s);
  int win = -1;  // lane i holds the table entry of the warp's block win_base + i
  {
    const int idx = b_begin + lane;
    if (lane < a.part_blocks && idx < a.max_blocks_per_seq) win = __ldg(table + idx);
  }
  P pol;
  pol.init(lane);
  pol.prefetch_q(a, s, kvh);
  if (ctx < 0 || ctx > a.max_blocks_per_seq * kBS || ctx > a.max_context_len) {
    if (part == 0 && kvh == 0 && lane == 0) report(a.dev_error, PA_DEVERR_CONTEXT_RANGE);
    ctx = 0;
  }
  const int nblk = (ctx + kBS - 1) / kBS;
  const int nparts = (nblk + a.part_blocks - 1) / a.part_blocks;
  if ((int)blockIdx.y * WARPS >= nparts) return;  // the whole CTA
  // a warp past the sequence's last partition streams nothing but joins the merge
  const int my_n = part < nparts ? min(nblk, b_begin + a.part_blocks) - b_begin : 0;

  unsigned char* wring = smem + (size_t)warp * STAGES * P::kStageBytes;
  uint64_t* wbars = reinterpret_cast<uint64_t*>(smem + kRing) + warp * STAGES;
  int* wvalid = reinterpret_cast<int*>(smem + kRing + WARPS * STAGES * sizeof(uint64_t)) +
                warp * STAGES;
  constexpr size_t kHead = kRing + size_t(WARPS) * STAGES * (sizeof(uint64_t) + sizeof(int));
  unsigned char* scratch =
      smem + ((kHead + 127) & ~size_t(127)) + (size_t)warp * P::kScratchBytes;
  if (lane == 0) {
#pragma unroll
    for (int st = 0; st < STAGES; ++st) mbar_init(&wbars[st], 1);
    mbar_init_fence();
  }
  __syncwarp();

  int win_base = 0;
  bool aborted;
  int j = 0;  // loop steps taken (blocks, or pairs of blocks)
  int issued;
  if constexpr (!has_pairs<P>::value) {
    auto issue = [&](int j) {
      if (j >= win_base + 32) {
        win_base = j & ~31;
        win = win_base + lane < my_n ? __ldg(table + b_begin + win_base + lane) : -1;
      }
      const int phys = __shfl_sync(0xffffffffu, win, j - win_base);
      if (lane == 0) {
        const int st = j % STAGES;
        uint64_t* bar = &wbars[st];
        const bool ok = (unsigned)phys < (unsigned)a.num_blocks;
        wvalid[st] = ok;
        if (a.stall_first_block && j == 0) {
          mbar_arrive_expect_tx(bar, 16);  // test hook: bytes that no copy will bring
        } else if (!ok) {
          report(a.dev_error, PA_DEVERR_BLOCK_RANGE);
          mbar_arrive(bar);
        } else {
          P::issue(a, &tm_k, &tm_v, wring + (size_t)st * P::kStageBytes, bar, phys, kvh);
        }
      }
    };
    for (int k = 0; k < STAGES && k < my_n; ++k) issue(k);
    issued = my_n < STAGES ? my_n : STAGES;
    pol.begin(a.scale_log2);

    aborted = a.stall_first_block && my_n > 0 &&
              !mbar_wait_bounded(&wbars[0], 0u, a.wait_limit_ns);
    if (aborted && lane == 0) report(a.dev_error, PA_DEVERR_WAIT_TIMEOUT);
    for (; !aborted && j < my_n; ++j) {
      const int st = j % STAGES;
      if (!mbar_wait_bounded(&wbars[st], (uint32_t)((j / STAGES) & 1))) {
        if (lane == 0) report(a.dev_error, PA_DEVERR_WAIT_TIMEOUT);
        aborted = true;
        break;
      }
      if (wvalid[st])
        pol.block(wring + (size_t)st * P::kStageBytes, ctx - (b_begin + j) * kBS, scratch);
      __syncwarp();
      if (j + STAGES < my_n) {
        if (lane == 0) fence_proxy_async_smem();
        issue(j + STAGES);
        issued = j + STAGES + 1;
      }
    }
  } else {
    // Two blocks per step: stage jp % STAGES holds blocks 2jp and 2jp + 1 of this
    // warp, behind one barrier; wvalid bit 0 / 1 says block 2jp / 2jp + 1 was copied.
    const int my_pairs = (my_n + 1) / 2;
    auto issue = [&](int jp) {
      const int j0 = 2 * jp;
      if (j0 >= win_base + 32) {
        win_base = j0 & ~31;
        win = win_base + lane < my_n ? __ldg(table + b_begin + win_base + lane) : -1;
      }
      // j0 - win_base is even and below 32, so both entries are in the window
      const int phys0 = __shfl_sync(0xffffffffu, win, j0 - win_base);
      const int phys1 = __shfl_sync(0xffffffffu, win, j0 + 1 - win_base);
      if (lane == 0) {
        const int st = jp % STAGES;
        uint64_t* bar = &wbars[st];
        unsigned char* dst = wring + (size_t)st * P::kStageBytes;
        const bool has1 = j0 + 1 < my_n;
        const bool ok0 = (unsigned)phys0 < (unsigned)a.num_blocks;
        const bool ok1 = has1 && (unsigned)phys1 < (unsigned)a.num_blocks;
        wvalid[st] = (ok0 ? 1 : 0) | (ok1 ? 2 : 0);
        if (!ok0 || (has1 && !ok1)) report(a.dev_error, PA_DEVERR_BLOCK_RANGE);
        if (a.stall_first_block && jp == 0) {
          mbar_arrive_expect_tx(bar, 16);  // test hook: bytes that no copy will bring
        } else if (!ok0 && !ok1) {
          mbar_arrive(bar);  // complete the phase without data; the pair is skipped
        } else {
          mbar_arrive_expect_tx(bar, (ok0 ? P::kBlockBytes : 0) + (ok1 ? P::kBlockBytes : 0));
          if (ok0) P::issue_block(a, &tm_k, &tm_v, dst, bar, phys0, kvh);
          if (ok1) P::issue_block(a, &tm_k, &tm_v, dst + P::kBlockBytes, bar, phys1, kvh);
        }
      }
    };
    for (int jp = 0; jp < STAGES && jp < my_pairs; ++jp) issue(jp);
    issued = my_pairs < STAGES ? my_pairs : STAGES;
    pol.begin(a.scale_log2);

    aborted = a.stall_first_block && my_pairs > 0 &&
              !mbar_wait_bounded(&wbars[0], 0u, a.wait_limit_ns);
    if (aborted && lane == 0) report(a.dev_error, PA_DEVERR_WAIT_TIMEOUT);
    for (; !aborted && j < my_pairs; ++j) {
      const int st = j % STAGES;
      if (!mbar_wait_bounded(&wbars[st], (uint32_t)((j / STAGES) & 1))) {
        if (lane == 0) report(a.dev_error, PA_DEVERR_WAIT_TIMEOUT);
        aborted = true;
        break;
      }
      const int v = wvalid[st];
      if (v) {
        unsigned char* sa = wring + (size_t)st * P::kStageBytes;
        const int b0 = b_begin + 2 * j;
        // a block that was not copied enters with no valid tokens (masked, its
        // value rows cleared) and the other block's tiles as a readable stand-in
        const int va = (v & 1) ? ctx - b0 * kBS : 0;
        const int vb = (v & 2) ? ctx - (b0 + 1) * kBS : 0;
        pol.block2((v & 1) ? sa : sa + P::kBlockBytes, va, (v & 2) ? sa + P::kBlockBytes : sa,
                   vb);
      }
      __syncwarp();
      if (j + STAGES < my_pairs) {
        if (lane == 0) fence_proxy_async_smem();
        issue(j + STAGES);
        issued = j + STAGES + 1;
      }
    }
  }
  if (aborted) {
    for (int k = j; k < issued; ++k)
      if (!(a.stall_first_block && k == 0))
        mbar_wait_bounded(&wbars[k % STAGES], (uint32_t)((k / STAGES) & 1));
  }
  // The CTA's WARPS consecutive partitions merge on chip (through shared memory,
  // reusing the tile ring) into one state row, row blockIdx.y of the sequence's
  // rows: the merge kernel then reads WARPS times fewer states.
  __syncthreads();
  float* red_m = reinterpret_cast<float*>(smem);  // [WARPS][G]
  float* red_l = red_m + WARPS * G;                // [WARPS][G]
  float* red_acc = red_l + WARPS * G;              // [WARPS][G][D]
  pol.to_red(red_m, red_l, red_acc, warp, lane);
  __syncthreads();
  const size_t row0 = (((size_t)s * a.num_kv_heads + kvh) * a.max_parts + blockIdx.y) * G;
  for (int item = threadIdx.x; item < G * D; item += blockDim.x) {
    const int g = item / D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < WARPS; ++w) M = fmaxf(M, red_m[w * G + g]);
    const float Mref = M == -INFINITY ? 0.f : M;
    float L = 0.f, A = 0.f;
#pragma unroll
    for (int w = 0; w < WARPS; ++w) {
      const float sc = exp2f(red_m[w * G + g] - Mref);
      L = fmaf(sc, red_l[w * G + g], L);
      A = fmaf(sc, red_acc[(w * G) * D + item], A);
    }
    a.ws_acc[(row0 + g) * D + (item % D)] = A;
    if (item % D == 0) {
      a.ws_m[row0 + g] = M;
      a.ws_l[row0 + g] = L;
    }
  }
}

constexpr size_t kSmemLimit = 200 * 1024;
constexpr int kMaxDevices = 64;

template <class P, int WARPS, int STAGES, int G, int D>
size_t smem_bytes(int max_parts) {
  // The warp-merge buffers and the split-KV weights reuse the tile ring once
  // the main loop is over.
  const size_t ring = size_t(WARPS) * STAGES * P::kStageBytes;
  const size_t red = size_t(WARPS) * G * (D + 2) * sizeof(float);
  const size_t wts = (size_t)max_parts * G * sizeof(float);
  size_t reuse = red > wts ? red : wts;
  if (reuse < ring) reuse = ring;
  return P::kAlign + reuse + size_t(WARPS) * STAGES * (sizeof(uint64_t) + sizeof(int)) + 128 +
         size_t(WARPS) * P::kScratchBytes;
}

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
  cuuint32_t box[2] = {64, (cuuint32_t)kBS};
  cuuint32_t estr[2] = {1, 1};
  const CUresult res = fn(
      map, dtype == PA_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
      const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
      CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return res == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// An E4M3 cache viewed as rows of head_dim (= 128) bytes, read in 16-row boxes
// of whole rows with 128-byte swizzling.
cudaError_t make_fp8_cache_map(CUtensorMap* map, const void* base, long long rows,
                               int head_dim) {
  auto fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  cuuint64_t dims[2] = {(cuuint64_t)head_dim, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)head_dim};
  cuuint32_t box[2] = {(cuuint32_t)head_dim, (cuuint32_t)kBS};
  cuuint32_t estr[2] = {1, 1};
  const CUresult res = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims,
                          strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return res == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

template <class P, typename T, int D, int G, int WARPS, int STAGES>
cudaError_t launch_kernel(const DecodeArgs& a, int dtype, cudaStream_t stream) {
  const size_t smem = smem_bytes<P, WARPS, STAGES, G, D>(a.max_parts);
  if (smem > kSmemLimit) return cudaErrorInvalidConfiguration;
  auto kern = paged_decode_kernel<P, T, D, G, WARPS, STAGES>;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  // The opt-in limit is a ceiling, not a reservation: set it once per device.
  static std::atomic<bool> ready[kMaxDevices];
  if (!ready[dev].load(std::memory_order_acquire)) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemLimit);
    if (e != cudaSuccess) return e;
    ready[dev].store(true, std::memory_order_release);
  }
  CUtensorMap tk, tv;
  memset(&tk, 0, sizeof(tk));
  memset(&tv, 0, sizeof(tv));
  if (P::kTma2D) {
    const long long rows = (long long)a.num_blocks * a.num_kv_heads * kBS;
    if (rows > 0x7fffffffLL) return cudaErrorInvalidValue;  // TMA row coordinates are int32
    if constexpr (P::kFp8Cache) {
      e = make_fp8_cache_map(&tk, a.k_cache, rows, D);
      if (e != cudaSuccess) return e;
      e = make_fp8_cache_map(&tv, a.v_cache, rows, D);
    } else {
      e = make_cache_map(&tk, a.k_cache, rows, D, dtype);
      if (e != cudaSuccess) return e;
      e = make_cache_map(&tv, a.v_cache, rows, D, dtype);
    }
    if (e != cudaSuccess) return e;
  }
  if (a.warp_parts) {
    auto wkern = paged_decode_warp_parts_kernel<P, T, D, G, WARPS, STAGES>;
    static std::atomic<bool> wready[kMaxDevices];
    if (!wready[dev].load(std::memory_order_acquire)) {
      e = cudaFuncSetAttribute(wkern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)kSmemLimit);
      if (e != cudaSuccess) return e;
      wready[dev].store(true, std::memory_order_release);
    }
    dim3 wgrid(a.num_kv_heads, (a.max_parts + WARPS - 1) / WARPS, a.num_seqs);
    e = launch_dependent(wkern, wgrid, dim3(WARPS * 32), smem, stream, a, tk, tv);
    if (e != cudaSuccess || a.states_only) return e;
    dim3 mgrid(a.num_kv_heads * G, a.num_seqs);
    return launch_dependent(merge_partitions_kernel<T, D, G, WARPS>, mgrid, dim3(kMergeThreads),
                            0, stream, a);
  }
  dim3 grid(a.num_kv_heads, a.max_parts, a.num_seqs);
  return launch_dependent(kern, grid, dim3(WARPS * 32), smem, stream, a, tk, tv);
}

// The warp-per-partition split with a two-block policy, then the merge launch.
template <class P, typename T, int D, int G, int WARPS, int STAGES>
cudaError_t launch_pair_parts(const DecodeArgs& a, int dtype, cudaStream_t stream) {
  const size_t smem = smem_bytes<P, WARPS, STAGES, G, D>(a.max_parts);
  if (smem > kSmemLimit) return cudaErrorInvalidConfiguration;
  auto kern = paged_decode_warp_parts_kernel<P, T, D, G, WARPS, STAGES>;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  static std::atomic<bool> ready[kMaxDevices];
  if (!ready[dev].load(std::memory_order_acquire)) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemLimit);
    if (e != cudaSuccess) return e;
    ready[dev].store(true, std::memory_order_release);
  }
  CUtensorMap tk, tv;
  memset(&tk, 0, sizeof(tk));
  memset(&tv, 0, sizeof(tv));
  if (P::kTma2D) {
    const long long rows = (long long)a.num_blocks * a.num_kv_heads * kBS;
    if (rows > 0x7fffffffLL) return cudaErrorInvalidValue;  // TMA row coordinates are int32
    e = make_fp8_cache_map(&tk, a.k_cache, rows, D);
    if (e != cudaSuccess) return e;
    e = make_fp8_cache_map(&tv, a.v_cache, rows, D);
    if (e != cudaSuccess) return e;
  }
  dim3 wgrid(a.num_kv_heads, (a.max_parts + WARPS - 1) / WARPS, a.num_seqs);
  e = launch_dependent(kern, wgrid, dim3(WARPS * 32), smem, stream, a, tk, tv);
  if (e != cudaSuccess || a.states_only) return e;
  dim3 mgrid(a.num_kv_heads * G, a.num_seqs);
  return launch_dependent(merge_partitions_kernel<T, D, G, WARPS>, mgrid, dim3(kMergeThreads), 0,
                          stream, a);
}

// The cascade's two decodes as one launch of cascade_decode_kernel: 4 x 2
// tiles, 4 x 3 over E4M3 caches (a stage holds half the bytes; 62.5 -> 62.2 us
// on the shared-prefix batch, 4 x 4 slower at 68.3 us).
template <class P1, int G1, class P2, int G2, typename T, int D>
cudaError_t launch_dual(const DecodeArgs& a1, const DecodeArgs& a2, int dtype,
                        cudaStream_t stream) {
  constexpr int WARPS = 4, STAGES = P1::kFp8Cache ? 3 : 2;
  const size_t s1 = smem_bytes<P1, WARPS, STAGES, G1, D>(a1.max_parts);
  const size_t s2 = smem_bytes<P2, WARPS, STAGES, G2, D>(a2.max_parts);
  const size_t smem = s1 > s2 ? s1 : s2;
  if (smem > kSmemLimit) return cudaErrorInvalidConfiguration;
  const long long n1 = (long long)a1.num_kv_heads * a1.max_parts * a1.num_seqs;
  const long long n2 =
      (long long)((a2.num_kv_heads + WARPS - 1) / WARPS) * a2.max_parts * a2.num_seqs;
  if (a1.num_kv_heads != a2.num_kv_heads || n1 + n2 > 0x7fffffffLL) return cudaErrorInvalidValue;
  if (n1 + n2 == 0) return cudaSuccess;
  auto kern = cascade_decode_kernel<P1, G1, P2, G2, T, D, WARPS, STAGES>;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  static std::atomic<bool> ready[kMaxDevices];
  if (!ready[dev].load(std::memory_order_acquire)) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemLimit);
    if (e != cudaSuccess) return e;
    ready[dev].store(true, std::memory_order_release);
  }
  CUtensorMap tk, tv;
  memset(&tk, 0, sizeof(tk));
  memset(&tv, 0, sizeof(tv));
  if (P1::kTma2D || P2::kTma2D) {
    static_assert(P1::kFp8Cache == P2::kFp8Cache, "one cache type");
    const long long rows = (long long)a1.num_blocks * a1.num_kv_heads * kBS;
    if (rows > 0x7fffffffLL) return cudaErrorInvalidValue;  // TMA row coordinates are int32
    if constexpr (P1::kFp8Cache) {
      e = make_fp8_cache_map(&tk, a1.k_cache, rows, D);
      if (e != cudaSuccess) return e;
      e = make_fp8_cache_map(&tv, a1.v_cache, rows, D);
    } else {
      e = make_cache_map(&tk, a1.k_cache, rows, D, dtype);
      if (e != cudaSuccess) return e;
      e = make_cache_map(&tv, a1.v_cache, rows, D, dtype);
    }
    if (e != cudaSuccess) return e;
  }
  return launch_dependent(kern, dim3((unsigned)(n1 + n2)), dim3(WARPS * 32), smem, stream, a1, a2,
                          tk, tv);
}

// Warps per CTA x stages per warp. Over 16-bit caches 4 x 2 (64 KiB of K/V in
// flight per CTA at head_dim 128, three CTAs per SM) measured best or within 2%
// of best on every workload. Over E4M3 caches a stage holds half the bytes and
// 4 x 3 measured faster than 4 x 2 (7B-like MHA 99.1 -> 97.7 us, GQA 32/8 85.2 ->
// 84.9 us per launch; 8 x 2 and 2 x 3 slower). PA_DECODE_TILE="WxS" selects
// another built shape for A/B measurements (4x2, 4x3, 8x2, 2x3).
int tile_variant() {
  static const int v = [] {
    const char* e = getenv("PA_DECODE_TILE");
    if (!e) return 0;
    if (!strcmp(e, "4x3")) return 1;
    if (!strcmp(e, "8x2")) return 2;
    if (!strcmp(e, "2x3")) return 3;
    if (!strcmp(e, "4x2")) return 4;
    return 0;
  }();
  return v;
}

template <class P, typename T, int D, int G>
cudaError_t launch_tiles(const DecodeArgs& a, int dtype, cudaStream_t stream) {
  switch (tile_variant()) {
    case 1: return launch_kernel<P, T, D, G, 4, 3>(a, dtype, stream);
    case 2: return launch_kernel<P, T, D, G, 8, 2>(a, dtype, stream);
    case 3: return launch_kernel<P, T, D, G, 2, 3>(a, dtype, stream);
    case 4: return launch_kernel<P, T, D, G, 4, 2>(a, dtype, stream);
    default:
      if constexpr (P::kFp8Cache) return launch_kernel<P, T, D, G, 4, 3>(a, dtype, stream);
      else return launch_kernel<P, T, D, G, 4, 2>(a, dtype, stream);
  }
}

// Which arithmetic path serves a query-head group: tensor cores from G = 4 up
// (the q.K and P.V tiles are then real contractions), CUDA cores below.
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

// Over E4M3 caches 4 and 8 query heads per KV head run on tensor cores, which
// take each converted code pair straight into an mma fragment; 1 and 2 run on
// CUDA cores (Fp8CudaCorePolicy). PA_DECODE_PATH overrides the choice here too
// (for any group).
bool use_tensor_path_e4m3(int group) {
  static const int forced = [] {
    const char* e = getenv("PA_DECODE_PATH");
    if (e && !strcmp(e, "cuda_cores")) return 0;
    if (e && !strcmp(e, "tensor")) return 1;
    return -1;
  }();
  if (forced >= 0) return forced == 1;
  return group >= 4;
}

template <typename T, int D, int G, typename C>
cudaError_t launch_g(const DecodeArgs& a, int dtype, cudaStream_t stream) {
  if constexpr (std::is_same<C, E4M3>::value) {
    if constexpr (G == 8) {
      // warp-per-partition split over 8 query heads per KV head: two blocks per
      // loop step (long-context 8-bit batch 237.6 -> 227.2 us); PA_DECODE_TILE
      // keeps the one-block kernel for A/B measurements
      if (a.warp_parts && use_tensor_path_e4m3(G) && tile_variant() == 0)
        return launch_pair_parts<Fp8TensorPairPolicy<T, D, G>, T, D, G, 4, 2>(a, dtype, stream);
    }
    if (use_tensor_path_e4m3(G))
      return launch_tiles<Fp8TensorPolicy<T, D, G>, T, D, G>(a, dtype, stream);
    if constexpr (G <= 2) {
      return launch_tiles<Fp8CudaCorePolicy<T, D, G>, T, D, G>(a, dtype, stream);
    } else {
      // 4 and 8 query heads reach the CUDA cores only when PA_DECODE_PATH
      // forces them; the generic policy keeps their register use lower
      return launch_tiles<CudaCorePolicy<T, D, G, C>, T, D, G>(a, dtype, stream);
    }
  } else {
    if (use_tensor_path(G)) return launch_tiles<TensorPolicy<T, D, G>, T, D, G>(a, dtype, stream);
    return launch_tiles<CudaCorePolicy<T, D, G, C>, T, D, G>(a, dtype, stream);
  }
}

template <typename T, int D, typename C>
cudaError_t launch_group(const DecodeArgs& a, int group, int dtype, cudaStream_t stream) {
  switch (group) {
    case 1:
      if constexpr (std::is_same<C, E4M3>::value) return launch_g<T, D, 1, C>(a, dtype, stream);
      return launch_tiles<CudaCorePolicy<T, D, 1, C>, T, D, 1>(a, dtype, stream);
    case 2: return launch_g<T, D, 2, C>(a, dtype, stream);
    case 4: return launch_g<T, D, 4, C>(a, dtype, stream);
    case 8: return launch_g<T, D, 8, C>(a, dtype, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

// The cascade's decodes in one launch: the groups' prefixes with 8 stacked
// query heads (`pre`, tensor cores) and the own blocks with g_own query heads
// per KV head (`own`, the policy paged_decode would pick), over a cache of T
// (C = T) or of E4M3 codes (C = E4M3). cudaErrorNotSupported when that shape
// has no single-launch form (or a PA_DECODE_PATH override is set): the caller
// then launches the two decodes.
template <typename T, int D, typename C = T>
cudaError_t launch_cascade_typed(const DecodeArgs& pre, const DecodeArgs& own, int g_own,
                                 int dtype, cudaStream_t stream) {
  if (getenv("PA_DECODE_PATH")) return cudaErrorNotSupported;
  if constexpr (std::is_same<C, E4M3>::value) {
    using Pre = Fp8TensorPolicy<T, D, 8>;
    switch (g_own) {
      case 1:
        return launch_dual<Pre, 8, Fp8CudaCorePolicy<T, D, 1>, 1, T, D>(pre, own, dtype, stream);
      case 2:
        return launch_dual<Pre, 8, Fp8CudaCorePolicy<T, D, 2>, 2, T, D>(pre, own, dtype, stream);
      case 4:
        return launch_dual<Pre, 8, Fp8TensorPolicy<T, D, 4>, 4, T, D>(pre, own, dtype, stream);
      default: return cudaErrorNotSupported;
    }
  } else {
    using Pre = TensorPolicy<T, D, 8>;
    switch (g_own) {
      case 1:
        return launch_dual<Pre, 8, CudaCorePolicy<T, D, 1, T>, 1, T, D>(pre, own, dtype, stream);
      case 2:
        return launch_dual<Pre, 8, CudaCorePolicy<T, D, 2, T>, 2, T, D>(pre, own, dtype, stream);
      case 4:
        return launch_dual<Pre, 8, TensorPolicy<T, D, 4>, 4, T, D>(pre, own, dtype, stream);
      default: return cudaErrorNotSupported;
    }
  }
}

// Launches the decode kernel for one query/output type T, head_dim and cache
// element type C (T itself, or E4M3).
template <typename T, int D, typename C = T>
cudaError_t launch_decode_typed(const DecodeArgs& a, int group, int dtype,
                                cudaStream_t stream) {
  return launch_group<T, D, C>(a, group, dtype, stream);
}

}  // namespace pa
