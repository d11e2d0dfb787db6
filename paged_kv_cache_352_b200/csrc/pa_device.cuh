// Device-side building blocks shared by libpa's kernels (sm_100a only).
//
// mbarrier + 1-D bulk async copy (the TMA bulk path) for staging 4 KiB cache
// tiles into shared memory, a bounded wait that gives up after a time limit
// instead of spinning forever, and conversions between the 16-bit storage types
// and fp32.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <stdint.h>
#include <string.h>

#include "pa_internal.h"

namespace pa {

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "libpa kernels are written for sm_100a only"
#endif

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
               : "memory");
}

// Makes barrier initialisation visible to the async (TMA) proxy.
__device__ __forceinline__ void mbar_init_fence() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return done != 0;
}

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Waits for the barrier phase with the given parity; returns false when the
// phase has not completed within `limit_ns` (0: kWaitLimitNs), and the caller
// reports the timeout.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity,
                                                  uint64_t limit_ns = 0) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t limit = limit_ns ? limit_ns : kWaitLimitNs;
  const uint64_t t0 = global_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (global_ns() - t0 > limit) return false;
  }
}

// Orders this thread's earlier generic-proxy shared-memory accesses before
// later async-proxy (TMA) accesses to the same memory.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// 1-D bulk copy global -> shared, completion counted in bytes on `bar`.
// Addresses 16-byte aligned, size a multiple of 16 (checked by the host).
__device__ __forceinline__ void bulk_copy_g2s(void* smem_dst, const void* gmem_src,
                                              uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_addr(smem_dst)),
      "l"(gmem_src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

// ---- 16-bit storage <-> fp32 -------------------------------------------------

template <typename T>
struct Storage;

template <>
struct Storage<__half> {
  // 8 packed halves -> 8 floats
  static __device__ __forceinline__ void to_f32(const uint4& u, float (&f)[8]) {
    const __half2* h = reinterpret_cast<const __half2*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 x = __half22float2(h[i]);
      f[2 * i] = x.x;
      f[2 * i + 1] = x.y;
    }
  }
  static __device__ __forceinline__ __half from_f32(float x) { return __float2half_rn(x); }
};

template <>
struct Storage<__nv_bfloat16> {
  static __device__ __forceinline__ void to_f32(const uint4& u, float (&f)[8]) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      f[2 * i] = __uint_as_float(w[i] << 16);
      f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
  static __device__ __forceinline__ __nv_bfloat16 from_f32(float x) {
    return __float2bfloat16_rn(x);
  }
};

// Tag type of an 8-bit E4M3 cache (OCP FP8, no infinities; saturating stores).
struct E4M3 {};

// Element of a K/V cache: C is the query/output type T for 16-bit caches or E4M3.
// Raw is the load unit holding 8 elements; to_f32 widens them exactly.
template <typename C>
struct CacheElem {
  static constexpr int kBytes = 2;
  using Raw = uint4;
  static __device__ __forceinline__ void to_f32(const Raw& u, float (&f)[8]) {
    Storage<C>::to_f32(u, f);
  }
};

// Two E4M3 codes (low byte first) to two halves; exact (every code is a half).
__device__ __forceinline__ uint32_t e4m3x2_to_half2_bits(uint32_t pair16) {
  const __half2_raw h =
      __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(pair16 & 0xffffu), __NV_E4M3);
  return static_cast<uint32_t>(h.x) | (static_cast<uint32_t>(h.y) << 16);
}

__device__ __forceinline__ float2 half2_bits_to_float2(uint32_t h) {
  __half2 v;
  memcpy(&v, &h, sizeof(v));
  return __half22float2(v);
}

template <>
struct CacheElem<E4M3> {
  static constexpr int kBytes = 1;
  using Raw = uint2;
  static __device__ __forceinline__ void to_f32(const Raw& u, float (&f)[8]) {
    const uint32_t w[2] = {u.x, u.y};
#pragma unroll
    for (int i = 0; i < 2; ++i) {
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const float2 x = half2_bits_to_float2(e4m3x2_to_half2_bits(w[i] >> (16 * k)));
        f[4 * i + 2 * k] = x.x;
        f[4 * i + 2 * k + 1] = x.y;
      }
    }
  }
};

// Two floats to two E4M3 codes (`lo` in the low byte), nearest even, saturating.
__device__ __forceinline__ uint32_t f32x2_to_e4m3x2(float lo, float hi) {
  return static_cast<uint32_t>(
      __nv_cvt_float2_to_fp8x2(make_float2(lo, hi), __NV_SATFINITE, __NV_E4M3));
}

// Online-softmax reference of one row, updated lazily: the reference (base 2)
// moves up only when the block's largest logit passes it by more than
// kLazyRescaleLog2, so every exponential stays at most 2^kLazyRescaleLog2 and
// most blocks keep the reference, when the caller's rescale of its accumulators
// can be skipped. Any reference gives the same softmax once the accumulators
// and the sum agree with it. Returns the reference for this block's exponentials
// (0 while every logit so far is -inf); alpha is the factor to bring the
// accumulators to it, exactly 1 when the reference did not move (and while
// nothing has accumulated).
constexpr float kLazyRescaleLog2 = 8.f;

__device__ __forceinline__ float lazy_reference(float& m, float bmax, float& alpha) {
  const float mnew = bmax > m + kLazyRescaleLog2 ? bmax : m;
  const float mref = mnew == -INFINITY ? 0.f : mnew;
  alpha = m == -INFINITY ? 1.f : exp2f(m - mref);
  m = mnew;
  return mref;
}

// gpu-scope fetch-and-add with acquire + release semantics.
__device__ __forceinline__ int atom_add_acq_rel_gpu(int* addr, int v) {
  int old;
  asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(addr), "r"(v)
               : "memory");
  return old;
}

// Programmatic dependent launch. A kernel launched with programmatic stream
// serialization (launch_dependent) may start while the kernel ahead of it in
// the stream is still running; grid_dependency_wait() returns once that kernel
// has completed and its memory operations are visible, and is a no-op in an
// ordinary launch. allow_dependents() lets the next kernel in the stream launch
// early (it still waits for this one before reading anything).
__device__ __forceinline__ void grid_dependency_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

__device__ __forceinline__ void allow_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ void report(int* dev_error, int bit) {
  if (dev_error != nullptr) atomicOr(dev_error, bit);
}

}  // namespace pa
