// pa_common.cuh -- shared device helpers of libpagedattn (sm_100a): PTX wrappers for mbarriers
// and bulk async copies, bf16/fp8 unpacking, the per-device error word.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace pa {

constexpr int kBlock = 16;  // tokens per physical block

// Bit set in the per-device error word when a kernel meets an out-of-range value.
enum : unsigned {
  kErrBlockId = 1u,      // block table entry outside [0, num_blocks)
  kErrSlot = 2u,         // slot outside [0, num_blocks*16)
  kErrLength = 4u,       // context length beyond the table row or max_context_len
  kErrTimeout = 8u,      // a bounded wait gave up
};

// Per-device error word (one copy per device that loads the library).  The library is built
// as one translation unit (api.cu includes every kernel header), so this is its only definition.
__device__ unsigned g_error_word = 0;

__device__ __forceinline__ void flag_error(unsigned bits) { atomicOr(&g_error_word, bits); }

// ----------------------------------------------------------------------------- smem / mbarrier
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait for phase `parity` of an mbarrier.  Each try_wait already suspends for a
// hardware-chosen interval; after `kMaxTries` failed tries the wait gives up, flags
// kErrTimeout and returns false so the caller can unwind instead of hanging.
constexpr uint32_t kMaxTries = 1u << 22;
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity) {
  for (uint32_t i = 0; i < kMaxTries; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  flag_error(kErrTimeout);
  return false;
}

// ----------------------------------------------------------------------------- bulk copies
// L2 policy: streamed once, evict first.
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

// 1-D bulk async copy global -> this CTA's shared memory, completing `bytes` on `bar`.
// dst and src 16-byte aligned, bytes a multiple of 16.  No multicast.
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar,
                                         uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1], %2, [%3], %4;" ::"r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// ----------------------------------------------------------------------------- unpacking
// bf16x2 word -> two floats (exact: a bf16 is the top half of a binary32).
__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Two E4M3 codes (low 16 bits of w, element 0 in the low byte) -> two floats (exact).
__device__ __forceinline__ float2 e4m3x2_to_float2(uint16_t w) {
  __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(w), __NV_E4M3);
  return __half22float2(*reinterpret_cast<__half2 *>(&h));
}

template <typename T>
__device__ __forceinline__ T ld_nc(const T *p) {
  return __ldg(p);
}

}  // namespace pa
