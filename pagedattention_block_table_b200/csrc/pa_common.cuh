// pa_common.cuh -- shared device helpers of libpagedattn (sm_100a): PTX wrappers for mbarriers
// and bulk async copies, bf16/fp8 unpacking, the per-device error word.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

namespace pa {

// Kernels walk the cache in units of 16 tokens (one 16-row run of a (block, KV head) tile); a
// physical block holds 16 or 32 tokens, i.e. one or two units.
constexpr int kBlock = 16;

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

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// Bounded wait for phase `parity` of an mbarrier.  The waits in this library are for this CTA's own
// copies and MMAs (microseconds); after kWaitLimitNs of wall time the wait gives up, flags
// kErrTimeout and returns false so the caller can unwind instead of hanging.
constexpr uint64_t kWaitLimitNs = 200ull * 1000 * 1000;
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 255u) == 0 && global_ns() - t0 > kWaitLimitNs) break;
  }
  flag_error(kErrTimeout);
  return false;
}

// One thread waits on a barrier that nothing will ever complete: the bounded wait above must give up,
// flag kErrTimeout and return (pa_selftest_bounded_wait).
__global__ void bounded_wait_selftest_kernel() {
  __shared__ uint64_t bar;
  mbar_init(&bar, 1);
  fence_mbar_init();
  (void)mbar_wait(&bar, 0);
}

// ----------------------------------------------------------------------------- bulk copies
// L2 policy: streamed once, evict first.
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

// 1-D bulk async copy global -> this CTA's shared memory, completing `bytes` on `bar`.
// dst and src 16-byte aligned, bytes a multiple of 16.  The destination is this CTA's own shared memory.
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

// Packed pairs of fp32 (sm_100 f32x2 arithmetic: two lanes per instruction).
__device__ __forceinline__ uint64_t f2pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ float2 f2unpack(uint64_t r) {
  float2 v;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(v.x), "=f"(v.y) : "l"(r));
  return v;
}
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t fmul2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t f2add(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
// bf16x2 word -> packed fp32 pair (element 0 low).
__device__ __forceinline__ uint64_t bf16x2_to_f2(uint32_t w) { return f2pack(bf16lo(w), bf16hi(w)); }

// Four E4M3 codes (element 0 in the low byte of w) -> f16 pairs (0,1) and (2,3), exact: the hardware
// e4m3x2 -> f16x2 conversion on each 16-bit half of w (one instruction per pair, no repacking).
__device__ __forceinline__ void e4m3x4_to_h2x2(uint32_t w, uint32_t &p01, uint32_t &p23) {
  asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %2;\n\t"
      "cvt.rn.f16x2.e4m3x2 %0, lo;\n\tcvt.rn.f16x2.e4m3x2 %1, hi;\n\t}"
      : "=r"(p01), "=r"(p23)
      : "r"(w));
}
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&v);
}

// Four one-byte codes (element 0 in the low byte) -> two f16 pairs (0,1) and (2,3), exact.  KT 1: OCP
// E4M3 through the hardware e4m3x2 -> f16x2 conversion.  KT 2: signed INT8: each byte, biased to unsigned,
// becomes the low byte of the f16 1024 + b (byte permute), and 1024 + 128 is subtracted (packed).
template <int KT>
__device__ __forceinline__ void bytes4_to_h2(uint32_t w, uint32_t &p01, uint32_t &p23) {
  if constexpr (KT == 1) {
    e4m3x4_to_h2x2(w, p01, p23);
  } else {
    const uint32_t u = w ^ 0x80808080u;
    const uint32_t bias = 0x64806480u;   // (1152, 1152) in f16
    const uint32_t x01 = __byte_perm(u, 0x64646464u, 0x4140), x23 = __byte_perm(u, 0x64646464u, 0x4342);
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(p01) : "r"(x01), "r"(bias));
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(p23) : "r"(x23), "r"(bias));
  }
}

// f16 pair (element 0 low) -> packed fp32 pair, exact.
__device__ __forceinline__ uint64_t h2_to_f2(uint32_t h) {
  uint64_t r;
  asm("{\n\t.reg .b16 lo, hi;\n\t.reg .f32 a, b;\n\tmov.b32 {lo, hi}, %1;\n\t"
      "cvt.f32.f16 a, lo;\n\tcvt.f32.f16 b, hi;\n\tmov.b64 %0, {a, b};\n\t}"
      : "=l"(r)
      : "r"(h));
  return r;
}

// Four one-byte KV codes (element 0 in the low byte) -> two packed fp32 pairs (0,1) and (2,3), exact.
// KT 1: OCP E4M3 through the hardware e4m3x2 -> f16x2 conversion, then f16 -> f32.  KT 2: signed INT8: each byte,
// biased to unsigned, is placed in the mantissa of 2^23 (byte permute), and 2^23 + 128 is then
// subtracted (packed), which is exact for every value.
template <int KT>
__device__ __forceinline__ void bytes4_to_f2(uint32_t w, uint64_t &p01, uint64_t &p23) {
  if constexpr (KT == 1) {
    uint32_t h01, h23;
    e4m3x4_to_h2x2(w, h01, h23);
    p01 = h2_to_f2(h01);
    p23 = h2_to_f2(h23);
  } else {
    const uint32_t u = w ^ 0x80808080u;
    const float f0 = __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7650));
    const float f1 = __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7651));
    const float f2 = __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7652));
    const float f3 = __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7653));
    const uint64_t bias = f2pack(8388736.f, 8388736.f);  // 2^23 + 128
    uint64_t d0, d1;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d0) : "l"(f2pack(f0, f1)), "l"(bias));
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d1) : "l"(f2pack(f2, f3)), "l"(bias));
    p01 = d0;
    p23 = d1;
  }
}

// Programmatic dependent launch: a kernel launched with programmatic stream serialisation may be
// scheduled while the previous kernel on the stream is still running.  Every kernel of this library
// calls griddep_wait() first, before reading any input (any of them may be that kernel's output), so
// what PDL buys is the launch latency: the CTAs are resident and start the moment it completes.
// griddep_launch() lets the next kernel be scheduled early in turn.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Launch with programmatic stream serialisation (see griddep_wait).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

}  // namespace pa
