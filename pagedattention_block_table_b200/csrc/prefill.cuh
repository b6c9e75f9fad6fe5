// prefill.cuh -- paged causal prefill on the tcgen05 tensor cores (sm_100a).
//
// What it computes (vLLM overview page, "Continuous Batching": prefill chunks share the batch with
// decoding requests; Core Concepts page §3.2: the chunk's K/V sit in the paged cache, read through
// the block table): for chunk c with history H_c and C_c new tokens, query row i (position H_c + i)
// of head h attends to positions t <= H_c + i of KV head h / G:
//     out[i][h] = softmax_t(scale * q[i][h] . K[t]) V[t].
//
// Design.  A CTA serves one KV head's query-head group: its rows stack the G query heads of each
// position (row r = position r / G, head r % G), so every K/V byte fetched serves G heads.  It holds
// two 128-row query tiles, A and B, that take turns ("ping-pong"): while one warpgroup runs the
// softmax of its tile, the tensor core computes the other tile's products.
//   warps 0-3  softmax of tile A, one row per thread = one TMEM lane   warps 4-7  the same for tile B
//   warp 8     issues every tcgen05.mma (one elected lane)              warp 9     issues the TMA loads
// Keys come in tiles of 128 (8 units of 16 tokens).  K and V tiles take turns in one ring of shared
// memory slots (K0, V0, K1, V1, ...), filled by TMA with one 16-row x 64-element box per unit and per
// 64-element plane of head_dim, in the UMMA 128-byte-swizzled layout (tensor map over the cache seen
// as [num_blocks*Hkv*block_size][head_dim]; each CTA loads its own copy).
// TMEM (512 columns): S_A, S_B (128 columns each), O_A, O_B (head_dim columns each).
// Per key tile j and query tile X:
//   S_X = Q_X K_j^T        M=128, N=128, both operands in shared memory, fp32 into TMEM
//   softmax warps          read S_X, base-2 online softmax, write P_X (bf16 pairs) back into the first
//                          64 columns of S_X with tcgen05.st
//   O_X += P_X V_j         A operand (P) read from TMEM, V from shared memory, fp32 accumulator in TMEM
// The tensor core runs O_A(j), S_A(j+1), O_B(j), S_B(j+1), ... in issue order, so S_X(j+1) overwrites
// the columns P_X(j) occupies only after O_X(j) has read them.  p is taken relative to a per-row
// reference max; only when a tile's max exceeds it by more than 2^8 does the row move the reference
// and rescale its O row in TMEM (tcgen05.ld/st) and its sum l.  O and l always share the reference,
// so out = O / l is exact whichever reference was used.
//
// One-byte caches (FP8 E4M3 or INT8 codes with a scale per KV head, head_dim 128; vLLM "Quantized KV
// Cache" page).  The products run in f16 (kind::f16 with f16 operands): TMA brings each unit's codes
// (16 rows x 128 bytes) into a two-item staging ring, warps 10-11 convert them into f16 tiles of the
// same swizzled layout in the K/V ring (exact for every code: E4M3 and INT8 values are f16 values), and
// the MMA and softmax warps run unchanged.  Each Q row is scaled by a power of two into f16 range
// (exact for its elements down to 2^-22 of its largest), P is written as f16 (it is at most 2^8), the
// K scale and the power of two fold into the row's softmax scale and the V scale into 1 / l.
#pragma once
#include <algorithm>
#include <functional>
#include <queue>
#include <type_traits>
#include <vector>

#include "pa_common.cuh"

#ifndef PA_PREFILL_SPLIT_REGS
#define PA_PREFILL_SPLIT_REGS 1
#endif

namespace pa {

// ----------------------------------------------------------------------------- tcgen05 / TMA wrappers
__device__ __forceinline__ void tmem_alloc(uint32_t *dst_smem, uint32_t ncols) {  // whole warp
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {  // whole warp
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// D[tmem] (+)= A[smem desc] * B[smem desc], bf16 inputs, fp32 accumulate; issued by one thread.
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive on `bar` once every tcgen05.mma this thread issued before has completed.
__device__ __forceinline__ void mma_commit(uint64_t *bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// This thread's TMEM lane, 32 consecutive fp32 columns starting at taddr's column.  The load and its
// wait are one asm statement, so no use of the registers can be scheduled before the wait.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// 128 consecutive 32-bit columns of this thread's TMEM lane (two loads, one wait, one asm statement).
__device__ __forceinline__ void tmem_ld128(uint32_t taddr, uint32_t (&r)[128]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x64.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, "
      "%32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, "
      "%48, %49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63}, [%128];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x64.b32 "
      "{%64, %65, %66, %67, %68, %69, %70, %71, %72, %73, %74, %75, %76, %77, %78, %79, "
      "%80, %81, %82, %83, %84, %85, %86, %87, %88, %89, %90, %91, %92, %93, %94, %95, "
      "%96, %97, %98, %99, %100, %101, %102, %103, %104, %105, %106, %107, %108, %109, %110, %111, "
      "%112, %113, %114, %115, %116, %117, %118, %119, %120, %121, %122, %123, %124, %125, %126, %127}, [%129];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]),
        "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]),
        "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]),
        "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]),
        "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63]),
        "=r"(r[64]), "=r"(r[65]), "=r"(r[66]), "=r"(r[67]), "=r"(r[68]), "=r"(r[69]), "=r"(r[70]), "=r"(r[71]),
        "=r"(r[72]), "=r"(r[73]), "=r"(r[74]), "=r"(r[75]), "=r"(r[76]), "=r"(r[77]), "=r"(r[78]), "=r"(r[79]),
        "=r"(r[80]), "=r"(r[81]), "=r"(r[82]), "=r"(r[83]), "=r"(r[84]), "=r"(r[85]), "=r"(r[86]), "=r"(r[87]),
        "=r"(r[88]), "=r"(r[89]), "=r"(r[90]), "=r"(r[91]), "=r"(r[92]), "=r"(r[93]), "=r"(r[94]), "=r"(r[95]),
        "=r"(r[96]), "=r"(r[97]), "=r"(r[98]), "=r"(r[99]), "=r"(r[100]), "=r"(r[101]), "=r"(r[102]),
        "=r"(r[103]), "=r"(r[104]), "=r"(r[105]), "=r"(r[106]), "=r"(r[107]), "=r"(r[108]), "=r"(r[109]),
        "=r"(r[110]), "=r"(r[111]), "=r"(r[112]), "=r"(r[113]), "=r"(r[114]), "=r"(r[115]), "=r"(r[116]),
        "=r"(r[117]), "=r"(r[118]), "=r"(r[119]), "=r"(r[120]), "=r"(r[121]), "=r"(r[122]), "=r"(r[123]),
        "=r"(r[124]), "=r"(r[125]), "=r"(r[126]), "=r"(r[127])
      : "r"(taddr), "r"(taddr + 64)
      : "memory");
}

// Store 32 fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])), "r"(__float_as_uint(v[3])),
      "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])), "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])),
      "r"(__float_as_uint(v[8])), "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])), "r"(__float_as_uint(v[15])),
      "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])), "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])),
      "r"(__float_as_uint(v[20])), "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
      "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])), "r"(__float_as_uint(v[27])),
      "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])), "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
      : "memory");
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// D[tmem] (+)= A[tmem] * B[smem desc]: A (M rows = TMEM lanes, K packed two bf16 per column) from
// tensor memory, bf16 inputs, fp32 accumulate; issued by one thread.
__device__ __forceinline__ void mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}


// Groups of K-steps issued from one asm statement.  The issuing thread dispatches one product at a time,
// so whatever it executes between two products adds to every product's time: a clock64 timeline showed
// 104-132 cycles per 128x128x16 product when each step computed its shared-memory descriptors in C++
// (and the PV loop ran with a runtime trip count), against 72-76 for products issued back to back.  Here
// only immediate adds to the two descriptors sit between products.  The start-address field of a
// descriptor holds (address >> 4) in 14 bits; shared-memory addresses stay below 2^18 bytes, so the adds
// never carry out of it.
//
// NK steps of D (+)= A*B, both operands in shared memory (K-major, 128-byte swizzle): step kk reads 32 bytes
// at column (kk % 4) of plane (kk / 4) of each operand; APL / BPL are the plane strides in 16-byte units.
// The first step overwrites D (the S products start a new tile).
template <int NK, int APL, int BPL>
__device__ __forceinline__ void mma_ss_group(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc) {
  static_assert(NK == 4 || NK == 8, "steps per group");
#define PA_MMA_SS(P) "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, " P ";\n\t"
#define PA_STEP2 "add.s64 %1, %1, 2;\n\tadd.s64 %2, %2, 2;\n\t"
  if constexpr (NK == 8) {
    asm volatile(
        "{\n\t.reg .pred f, t;\n\tsetp.ne.b32 f, %3, %3;\n\tsetp.eq.b32 t, %3, %3;\n\t"
        PA_MMA_SS("f") PA_STEP2 PA_MMA_SS("t") PA_STEP2 PA_MMA_SS("t") PA_STEP2 PA_MMA_SS("t")
        "add.s64 %1, %1, %4;\n\tadd.s64 %2, %2, %5;\n\t"
        PA_MMA_SS("t") PA_STEP2 PA_MMA_SS("t") PA_STEP2 PA_MMA_SS("t") PA_STEP2 PA_MMA_SS("t") "}"
        : "+r"(d_tmem), "+l"(a_desc), "+l"(b_desc)
        : "r"(idesc), "n"(APL - 6), "n"(BPL - 6)
        : "memory");
  } else {
    asm volatile(
        "{\n\t.reg .pred f, t;\n\tsetp.ne.b32 f, %3, %3;\n\tsetp.eq.b32 t, %3, %3;\n\t"
        PA_MMA_SS("f") PA_STEP2 PA_MMA_SS("t") PA_STEP2 PA_MMA_SS("t") PA_STEP2 PA_MMA_SS("t") "}"
        : "+r"(d_tmem), "+l"(a_desc), "+l"(b_desc)
        : "r"(idesc)
        : "memory");
  }
#undef PA_STEP2
#undef PA_MMA_SS
}

// Eight steps of D += A*B with A in TMEM (8 columns = 16 bf16 per lane and step) and B in shared memory
// (MN-major, 16 rows = 2048 bytes per step); the first step accumulates only when acc0 != 0.
__device__ __forceinline__ void mma_ts_group8(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                              uint32_t acc0) {
#define PA_MMA_TS(P) "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, " P ";\n\t"
#define PA_STEPV "add.u32 %1, %1, 8;\n\tadd.s64 %2, %2, 128;\n\t"
  asm volatile(
      "{\n\t.reg .pred f, t;\n\tsetp.ne.b32 f, %4, 0;\n\tsetp.eq.b32 t, %4, %4;\n\t"
      PA_MMA_TS("f") PA_STEPV PA_MMA_TS("t") PA_STEPV PA_MMA_TS("t") PA_STEPV PA_MMA_TS("t") PA_STEPV
      PA_MMA_TS("t") PA_STEPV PA_MMA_TS("t") PA_STEPV PA_MMA_TS("t") PA_STEPV PA_MMA_TS("t") "}"
      : "+r"(d_tmem), "+r"(a_tmem), "+l"(b_desc)
      : "r"(idesc), "r"(acc0)
      : "memory");
#undef PA_STEPV
#undef PA_MMA_TS
}

// Store 16 consecutive 32-bit columns of this thread's TMEM lane (no wait).
__device__ __forceinline__ void tmem_st16u_nowait(uint32_t taddr, const uint32_t *v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),
      "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// 2-D tiled TMA load global -> shared, completing on `bar`.  x is the innermost coordinate.
__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int x, int y, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::
          "r"(smem_u32(dst)),
      "l"(map), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

// UMMA shared-memory descriptor of a 128-byte-swizzled operand (Blackwell format: start, leading and
// stride byte offsets in 16-byte units, version 1, layout type 2 = SWIZZLE_128B).  The operand's
// swizzle atoms (8 rows x 128 bytes) start on 1024-byte boundaries.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  d |= static_cast<uint64_t>(2) << 61;
  return d;
}

// Instruction descriptor for kind::f16 with bf16 A and B, fp32 D, A K-major; B K-major or MN-major.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((b_mn_major ? 1u : 0u) << 16) |
         (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}
// The same with f16 A and B (format fields 0).
__host__ __device__ constexpr uint32_t idesc_f16(int M, int N, bool b_mn_major) {
  return (1u << 4) | ((b_mn_major ? 1u : 0u) << 16) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&v);
}

// ----------------------------------------------------------------------------- the kernel
struct PrefillParams {
  __nv_bfloat16 *out;
  const __nv_bfloat16 *q;
  const int32_t *cu_q_lens;
  const int32_t *block_tables;
  const int32_t *context_lens;
  int64_t num_blocks;
  int block_size;       // 16 or 32 tokens per physical block
  int max_blocks_per_seq;
  int num_q_heads;
  int num_kv_heads;
  int group;            // Hq / Hkv
  int hpr;              // query heads stacked per position in a tile (G if 128 % G == 0, else 1)
  int max_context_len;
  int num_chunks;
  float qscale;         // scale * log2(e)
  const float *k_scale; // one-byte caches: per-KV-head scales of the codes (else unused)
  const float *v_scale;
  float *ws_o;          // planned launches with split key ranges: partial O rows [slot][x][256][D]
  float *ws_ml;         // and their (reference max, sum) [slot][x][256][2]
};

constexpr int kOrderedChunks = 64;   // chunks the prefill grid orders by context length
constexpr int kPlanItems = 1024;     // work items of a planned launch (kernel-parameter list)
constexpr int kPlanChunks = 1024;    // chunks a planned launch can carry

// A planned launch (the caller passed the lengths on the host too): grid row y serves work item y, in
// the order a longest-processing-time-first schedule gives.  An item is a query-tile pair of a chunk
// and a range of its key tiles: a CTA whose key range is long next to the launch's average is cut into
// pieces of `per` key tiles that run as separate CTAs and leave partial (O, max, sum) rows in the
// workspace; prefill_combine_kernel merges them.
//   item[y][0] = chunk | pair << 16   (pair 0 = the chunk's last query-tile pair, which sees the most keys)
//   item[y][1] = piece | pieces << 8 | per << 16
//   slot[y]    = workspace slot of the piece's partials (pieces > 1)
//   pairs[c]   = query-tile pairs the plan launched for chunk c (a longer chunk on the device is flagged)
template <bool PLANNED>
struct PrefillPlan {
  int32_t item[PLANNED ? kPlanItems : 1][2];
  int32_t slot[PLANNED ? kPlanItems : 1];
  int32_t pairs[PLANNED ? kPlanChunks : 1];
};
// The split items of a plan, for the combine: item[i][0] = chunk | pair << 16; item[i][1] = pieces | first
// slot << 8.
struct PrefillCombineList {
  int32_t item[kPlanItems][2];
};

// KT: cache element type (0 bf16, 1 FP8 E4M3, 2 INT8; one-byte types at head_dim 128 only)
template <int D, int KT = 0>
struct PrefillCfg {
  static constexpr int BM = 128;                  // rows per query tile (= TMEM lanes)
  static constexpr int BN = 128;                  // keys per key tile (8 units of 16 tokens)
  static constexpr int DH = D / 64;               // 64-element (128-byte) planes of a head_dim row
  static constexpr int Q_PLANE = BM * 128;        // 16 KB
  static constexpr int Q_BYTES = DH * Q_PLANE;
  static constexpr int KV_PLANE = BN * 128;       // 16 KB
  static constexpr int SLOT_BYTES = DH * KV_PLANE;  // one K or V tile
  // ring of K/V tiles (K and V alternate); one-byte caches give a slot to the staging ring of codes
  static constexpr int NSLOT = KT != 0 ? 4 : (D == 128 ? 5 : 8);
  static constexpr int NU8 = KT != 0 ? 2 : 0;     // staging ring of one-byte K or V tiles
  static constexpr int U8_BYTES = BN * 128;       // 16 KB: 128 keys x 128 one-byte codes
  static constexpr int OFF_QA = 0;
  static constexpr int OFF_QB = OFF_QA + Q_BYTES;
  static constexpr int OFF_KV = OFF_QB + Q_BYTES;
  static constexpr int OFF_U8 = OFF_KV + NSLOT * SLOT_BYTES;
  static constexpr int OFF_BAR = OFF_U8 + NU8 * U8_BYTES;
  static constexpr int NBAR = 32;
  static constexpr int SMEM = OFF_BAR + NBAR * 8 + 16 + 1024;  // + slack to align the base to 1024
  static constexpr uint32_t TMEM_COLS = 512;
  // TMEM columns: S of tile X at 128X (P_X in its first 64 columns); O of tile X at 256 + D*X
  __host__ __device__ static constexpr uint32_t s_col(int X) { return 128u * X; }
  __host__ __device__ static constexpr uint32_t o_col(int X) { return 256u + static_cast<uint32_t>(D) * X; }
#if PA_PREFILL_SPLIT_REGS
  // three warpgroups: softmax A, softmax B, and one holding the MMA and TMA warps (plus two warps that
  // convert one-byte codes, idle over a bf16 cache) that hands registers to the softmax warpgroups with
  // setmaxnreg
  static constexpr int THREADS = 384;
  static constexpr int REGS_LAUNCH = 168;         // 65536 / 384, rounded down to a multiple of 8
  static constexpr int REGS_SOFTMAX = 216;
  static constexpr int REGS_PRODUCER = 72;        // the rest of the launch allocation (one-byte converters)
  static_assert(2 * 128 * REGS_SOFTMAX + 128 * REGS_PRODUCER <= THREADS * REGS_LAUNCH, "register split");
#else
  static constexpr int THREADS = KT != 0 ? 384 : 320;
#endif
  static_assert(D == 64 || D == 128, "head_dim");
  static_assert(KT == 0 || D == 128, "one-byte caches at head_dim 128");
  static_assert(SMEM <= 227 * 1024, "shared memory");
};

// mbarrier slots: kFull/kEmpty per ring slot; kSFull, kPFull per query tile
enum : int {
  kFull = 0,
  kEmpty = kFull + 8,
  kSFull = kEmpty + 8,
  kPFull = kSFull + 2,
  kQReady = kPFull + 2,
  kDone = kQReady + 1,
  kU8Full = kDone + 1,   // one-byte staging ring: codes landed / codes converted
  kU8Empty = kU8Full + 2,
  kNumBars = kU8Empty + 2
};

// Three-input max / min (sm_100).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
__device__ __forceinline__ float fmin3(float a, float b, float c) {
  float d;
  asm("min.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

template <int D, int KT, bool PLANNED>
__global__ void __launch_bounds__(PrefillCfg<D, KT>::THREADS, 1)
    paged_prefill_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                         const PrefillParams P, const __grid_constant__ PrefillPlan<PLANNED> W) {
  using C = PrefillCfg<D, KT>;
  static_assert(kNumBars <= C::NBAR && C::NSLOT <= 8 && C::NU8 <= 2, "barrier slots");
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int hg0 = blockIdx.x * P.hpr;                 // first query head of this CTA's rows
  const int g = hg0 / P.group;                        // their KV head
  const int ppt = C::BM / P.hpr;                      // positions per query tile
  // any input may come from the kernel before this one on the stream (launched with PDL)
  griddep_wait();
  griddep_launch();

  // Longest work first (CTAs are dispatched in index order).  Planned launch: grid row y is work item y.
  // Otherwise chunk rank blockIdx.z serves the chunk with the rank-th longest context (ties by index),
  // and within a chunk blockIdx.y counts query-tile pairs down from the last one, which sees the most
  // keys (up to kOrderedChunks chunks; beyond that, blockIdx.z is the chunk).
  int c = blockIdx.z, pair = blockIdx.y, piece = 0, pieces = 1, per = 0, slot = 0;
  if constexpr (PLANNED) {
    const int32_t w0 = W.item[blockIdx.y][0], w1 = W.item[blockIdx.y][1];
    c = w0 & 0xffff;
    pair = (w0 >> 16) & 0xffff;
    piece = w1 & 0xff;
    pieces = (w1 >> 8) & 0xff;
    per = (w1 >> 16) & 0xffff;
    slot = W.slot[blockIdx.y];
    if (c >= P.num_chunks || pieces < 1 || (pieces > 1 && per < 1)) {
      if (tid == 0 && blockIdx.x == 0) flag_error(kErrLength);
      return;
    }
  } else if (P.num_chunks <= kOrderedChunks) {
    int *s_chunk = reinterpret_cast<int *>(smem + C::OFF_BAR + C::NBAR * 8 + 8);
    if (tid < P.num_chunks) {
      const int mine = P.context_lens[tid];
      int rank = 0;
      for (int k = 0; k < P.num_chunks; ++k) {
        const int other = P.context_lens[k];
        rank += (other > mine || (other == mine && k < tid)) ? 1 : 0;
      }
      if (rank == static_cast<int>(blockIdx.z)) *s_chunk = tid;
    }
    __syncthreads();
    c = *s_chunk;
  }
  const int q0 = P.cu_q_lens[c];
  const int Cn = P.cu_q_lens[c + 1] - q0;
  const int ctx = P.context_lens[c];
  const int H = ctx - Cn;
  if (Cn < 0 || H < 0 || ctx > min(P.max_blocks_per_seq * P.block_size, P.max_context_len)) {
    if (tid == 0 && blockIdx.x == 0 && blockIdx.y == 0) flag_error(kErrLength);
    return;
  }
  const int nx = (Cn + 2 * ppt - 1) / (2 * ppt);      // CTAs (pairs of query tiles) of this chunk
  if (!PLANNED && nx > static_cast<int>(gridDim.y)) { // chunk longer than the max_q_len launched for
    if (tid == 0 && blockIdx.x == 0 && blockIdx.y == 0) flag_error(kErrLength);
    return;
  }
  if constexpr (PLANNED) {
    // the device chunk needs query-tile pairs the plan did not launch (host lengths shorter than the
    // device's): reported like a chunk longer than max_q_len, and those rows are not written
    if (nx > W.pairs[c] && pair == 0 && piece == 0) {
      if (tid == 0 && blockIdx.x == 0) flag_error(kErrLength);
    }
  }
  if (pair >= nx) return;                             // (planned: the plan's chunk was longer)
  const int p0 = (nx - 1 - pair) * 2 * ppt;           // first position of tile A
  const int p_end = min(Cn, p0 + 2 * ppt);
  const int kv_len = H + p_end;                       // keys visible to some row of this CTA
  const int all_tiles = (kv_len + C::BN - 1) / C::BN;
  // this CTA's key tiles [tl0, tl0 + ntiles): all of them, or one piece (the last piece always runs to
  // the end, so the keys are covered whatever lengths the plan was made for)
  int tl0 = 0, tl1 = all_tiles;
  if (pieces > 1) {
    tl0 = min(piece * per, all_tiles);
    tl1 = piece == pieces - 1 ? all_tiles : min(all_tiles, tl0 + per);
  }
  const int ntiles = tl1 - tl0;
  // rows of this CTA in the workspace (split items): [slot][blockIdx.x][256 rows]
  const int64_t ws_row0 = ((int64_t)slot * gridDim.x + blockIdx.x) * 256;
  if (ntiles <= 0) {
    // an empty piece (the chunk is shorter than the plan's): its rows contribute nothing to the merge
    if (pieces > 1 && tid < 256) {
      P.ws_ml[(ws_row0 + tid) * 2] = -INFINITY;
      P.ws_ml[(ws_row0 + tid) * 2 + 1] = 0.f;
    }
    return;
  }
  // 16-key steps of the last tile that hold a visible key (the PV product stops there; a piece that
  // ends before the CTA's last tile has only full tiles)
  const int last_k16 = tl1 == all_tiles ? (kv_len - (all_tiles - 1) * C::BN + 15) / 16 : C::BN / 16;

  // the producer lanes' block-table entries of the first two key tiles, read before the CTA's set-up so
  // that their latency overlaps it (the first K tile's copy waits on them; checked where they are used).
  // bf16 caches only: on the mixed step it moved bf16 from 902 to 913 TFLOP/s and FP8 from 894 to 880.
  int pre_e0 = 0, pre_e1 = 0;
  const bool pre_read = KT == 0;
  if (pre_read && warp == 9) {
    constexpr int UPT = C::BN / kBlock, NPL = KT != 0 ? 1 : C::DH;
    const int w_lane = lane / (UPT * NPL), bb = (lane / NPL) % UPT;
    const int ush = P.block_size == 32 ? 1 : 0;
    const int32_t *trow = P.block_tables + (int64_t)c * P.max_blocks_per_seq;
    const int u0 = tl0 * UPT + bb, u1 = u0 + UPT;
    if (w_lane < 2 && u0 * kBlock < kv_len) pre_e0 = __ldg(trow + (u0 >> ush));
    if (w_lane < 2 && 1 < ntiles && u1 * kBlock < kv_len) pre_e1 = __ldg(trow + (u1 >> ush));
  }

  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + C::NBAR);
  if (warp == 8) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  if (tid == 0) {
    for (int i = 0; i < C::NSLOT; ++i) {
      mbar_init(&bars[kFull + i], KT != 0 ? 64 : 1);   // one-byte: the 64 converting threads
      mbar_init(&bars[kEmpty + i], 1);
    }
    for (int i = 0; i < C::NU8; ++i) {
      mbar_init(&bars[kU8Full + i], 1);
      mbar_init(&bars[kU8Empty + i], 64);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars[kSFull + i], 1);
      mbar_init(&bars[kPFull + i], 128);
    }
    mbar_init(&bars[kQReady], 256);
    mbar_init(&bars[kDone], 1);
    fence_mbar_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  bool timeout = false;
  // ring item i (K of tile i/2 when i is even, V when odd) sits in slot i % NSLOT; its use count is i / NSLOT
  auto slot_of = [&](int i) { return smem + C::OFF_KV + (i % C::NSLOT) * C::SLOT_BYTES; };

  if (warp < 8) {
    // ===================================================================== softmax warpgroups
#if PA_PREFILL_SPLIT_REGS
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(C::REGS_SOFTMAX));
#endif
    const int X = warp >> 2;                          // 0: tile A, 1: tile B
    const int r = tid & 127;                          // row = TMEM lane
    const int pos_i = p0 + X * ppt + r / P.hpr;       // position within the chunk
    const int h = hg0 + r % P.hpr;
    const bool row_ok = pos_i < Cn;
    const int pos = row_ok ? H + pos_i : kv_len - 1;  // padding rows behave like the last row
    uint8_t *sQ = smem + (X ? C::OFF_QB : C::OFF_QA);
    float qs = P.qscale;
    // Q row into the K-major 128-byte-swizzled tile (chunk ch of row r at ch ^ (r % 8))
    if constexpr (KT != 0) {
      // f16 row scaled by 2^e so that its largest magnitude lies in [2^8, 2^9); 2^-e and the K scale
      // join the row's softmax scale
      uint8_t *rowp = sQ + r * 128;
      uint4 w[D / 8];
      float amax = 0.f;
#pragma unroll
      for (int ch = 0; ch < D / 8; ++ch) {
        w[ch] = row_ok ? reinterpret_cast<const uint4 *>(P.q + ((int64_t)(q0 + pos_i) * P.num_q_heads + h) * D)[ch]
                       : make_uint4(0, 0, 0, 0);
        const uint32_t ww[4] = {w[ch].x, w[ch].y, w[ch].z, w[ch].w};
#pragma unroll
        for (int t = 0; t < 4; ++t) amax = fmax3(amax, fabsf(bf16lo(ww[t])), fabsf(bf16hi(ww[t])));
      }
      int ex = amax > 0.f ? static_cast<int>((__float_as_uint(amax) >> 23) & 0xff) - 127 : 0;
      ex = ex < -118 ? -118 : (ex > 126 ? 126 : ex);
      const float up = __uint_as_float(static_cast<uint32_t>(127 + 8 - ex) << 23);   // 2^(8 - ex)
      qs = __uint_as_float(static_cast<uint32_t>(127 + ex - 8) << 23) * (P.qscale * P.k_scale[g]);
#pragma unroll
      for (int ch = 0; ch < D / 8; ++ch) {
        const uint32_t ww[4] = {w[ch].x, w[ch].y, w[ch].z, w[ch].w};
        uint32_t hw[4];
#pragma unroll
        for (int t = 0; t < 4; ++t) hw[t] = pack_f16x2(bf16lo(ww[t]) * up, bf16hi(ww[t]) * up);
        *reinterpret_cast<uint4 *>(rowp + (ch >> 3) * C::Q_PLANE + (((ch & 7) ^ (r & 7)) << 4)) =
            make_uint4(hw[0], hw[1], hw[2], hw[3]);
      }
      fence_async_smem();
      mbar_arrive(&bars[kQReady]);
    } else {
      // all of the row's loads are issued before any store: a store between them would order each load
      // behind the previous store (the compiler cannot tell the global row from shared memory), and the
      // row would take one memory latency per 16 bytes
      uint8_t *rowp = sQ + r * 128;
      uint4 w[D / 8];
      const uint4 *src =
          reinterpret_cast<const uint4 *>(P.q + ((int64_t)(q0 + (row_ok ? pos_i : 0)) * P.num_q_heads + h) * D);
#pragma unroll
      for (int ch = 0; ch < D / 8; ++ch) w[ch] = row_ok ? __ldg(src + ch) : make_uint4(0, 0, 0, 0);
#pragma unroll
      for (int ch = 0; ch < D / 8; ++ch)
        *reinterpret_cast<uint4 *>(rowp + (ch >> 3) * C::Q_PLANE + (((ch & 7) ^ (r & 7)) << 4)) = w[ch];
      fence_async_smem();
      mbar_arrive(&bars[kQReady]);
    }
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t s_addr = tmem + lane_base + C::s_col(X);
    const uint32_t o_addr = tmem + lane_base + C::o_col(X);
    constexpr float kRescale = 8.f;
    float m_ref = -INFINITY, l_run = 0.f;
    for (int j = 0; j < ntiles; ++j) {
      const int kbase = (tl0 + j) * C::BN;
      const bool diag = kbase + C::BN - 1 > pos;       // some key of this tile is past the row
      // the passes below store P with warp-collective tcgen05.st, so the choice of pass is made per warp:
      // the masking pass when any row of the warp has a key past its position (it masks nothing for the
      // other rows).  Decided before S is ready, off the tile's critical path.
      const bool wdiag = __any_sync(0xffffffffu, diag);
      // every wait's outcome is made warp-uniform: the tcgen05.ld/st below are warp-collective.
      // S_X(j) complete also means O_X(j-1) complete (issued before it, tracked by the same commit).
      if (!__all_sync(0xffffffffu, mbar_wait(&bars[kSFull + X], j & 1))) { timeout = true; break; }
      tc_fence_after();
      uint32_t sr[C::BN];
      tmem_ld128(s_addr, sr);
      // last key tile: V rows of keys no row may see, up to the last 16-key step the PV product reads,
      // are zeroed (tile A's threads, one row each) once the V tile has landed, so that 0 * (whatever
      // the cache holds past the context) never reaches the MMA
      // (one-byte caches: the converting warps write those rows as zeros)
      if (KT == 0 && X == 0 && j == ntiles - 1 && kbase + r >= kv_len && r < last_k16 * 16) {
        const int it = 2 * j + 1;
        if (mbar_wait(&bars[kFull + it % C::NSLOT], (it / C::NSLOT) & 1)) {
          uint8_t *vt = slot_of(it);
#pragma unroll
          for (int hh = 0; hh < C::DH; ++hh)
#pragma unroll
            for (int ch = 0; ch < 8; ++ch)
              *reinterpret_cast<uint4 *>(vt + hh * C::KV_PLANE + r * 128 + ch * 16) = make_uint4(0, 0, 0, 0);
          fence_async_smem();
        }
      }
      if (m_ref == -INFINITY) {
        // first tile of the row: the reference is the tile's scaled max (masked keys do not take part)
        float mt_ = -INFINITY;
        if (!diag) {
          // max of s * qscale: the max of s for a positive scale, the min for a negative one
          // (three-input max/min: two new keys per instruction, four independent chains)
          const float s0 = __uint_as_float(sr[0]), s1 = __uint_as_float(sr[1]), s2 = __uint_as_float(sr[2]),
                      s3 = __uint_as_float(sr[3]), s4 = __uint_as_float(sr[4]), s5 = __uint_as_float(sr[5]),
                      s6 = __uint_as_float(sr[6]), s7 = __uint_as_float(sr[7]);
          if (qs >= 0.f) {
            float e0 = fmaxf(s0, s1), e1 = fmaxf(s2, s3), e2 = fmaxf(s4, s5), e3 = fmaxf(s6, s7);
#pragma unroll
            for (int k = 8; k < C::BN; k += 8) {
              e0 = fmax3(e0, __uint_as_float(sr[k]), __uint_as_float(sr[k + 1]));
              e1 = fmax3(e1, __uint_as_float(sr[k + 2]), __uint_as_float(sr[k + 3]));
              e2 = fmax3(e2, __uint_as_float(sr[k + 4]), __uint_as_float(sr[k + 5]));
              e3 = fmax3(e3, __uint_as_float(sr[k + 6]), __uint_as_float(sr[k + 7]));
            }
            mt_ = fmax3(fmaxf(e0, e1), e2, e3) * qs;
          } else {
            float e0 = fminf(s0, s1), e1 = fminf(s2, s3), e2 = fminf(s4, s5), e3 = fminf(s6, s7);
#pragma unroll
            for (int k = 8; k < C::BN; k += 8) {
              e0 = fmin3(e0, __uint_as_float(sr[k]), __uint_as_float(sr[k + 1]));
              e1 = fmin3(e1, __uint_as_float(sr[k + 2]), __uint_as_float(sr[k + 3]));
              e2 = fmin3(e2, __uint_as_float(sr[k + 4]), __uint_as_float(sr[k + 5]));
              e3 = fmin3(e3, __uint_as_float(sr[k + 6]), __uint_as_float(sr[k + 7]));
            }
            mt_ = fmin3(fminf(e0, e1), e2, e3) * qs;
          }
        } else {
#pragma unroll
          for (int k = 0; k < C::BN; ++k)
            if (kbase + k <= pos) mt_ = fmaxf(mt_, __uint_as_float(sr[k]) * qs);
        }
        m_ref = mt_;
      }
      // p = 2^(s * qscale - m_ref) for the tile's keys into the first 64 columns of S (bf16 pairs), with the
      // largest exponent; keys past the row's position get p = 0.  Masking is compiled only into the pass
      // of diagonal tiles.
      float sum = 0.f;
      auto pass = [&](auto diag_c) {
        constexpr bool kDiag = decltype(diag_c)::value;
        // two independent max chains, P stored in quarters of 32 keys: the last store and the last max
        // are short when the pass ends
        float mx = -INFINITY, my = -INFINITY;
        uint64_t ls2 = 0ull;
        const uint64_t qs2 = f2pack(qs, qs), nm2 = f2pack(-m_ref, -m_ref);
#pragma unroll
        for (int qq = 0; qq < 4; ++qq) {
          uint32_t pk[16];
#pragma unroll
          for (int k2 = 0; k2 < 16; ++k2) {
            const int k = qq * 32 + 2 * k2;
            float2 x = f2unpack(ffma2(f2pack(__uint_as_float(sr[k]), __uint_as_float(sr[k + 1])), qs2, nm2));
            if (kDiag) {
              if (kbase + k > pos) x.x = -INFINITY;
              if (kbase + k + 1 > pos) x.y = -INFINITY;
            }
            if (k2 & 1)
              my = fmax3(my, x.x, x.y);
            else
              mx = fmax3(mx, x.x, x.y);
            const float a = ex2(x.x);
            const float b = ex2(x.y);
            ls2 = f2add(ls2, f2pack(a, b));
            pk[k2] = KT != 0 ? pack_f16x2(a, b) : pack_bf16x2(a, b);
          }
          tmem_st16u_nowait(s_addr + qq * 16, pk);
        }
        mx = fmaxf(mx, my);
        const float2 lsv = f2unpack(ls2);
        sum = lsv.x + lsv.y;
        return mx;
      };
      const float mx = wdiag ? pass(std::true_type{}) : pass(std::false_type{});
      // The reference moves only when the tile's max exceeds it by more than 2^8: then P is recomputed
      // against the new one (p of such a tile may even have overflowed), O and l are rescaled below.  The
      // recompute rewrites P (warp-collective tcgen05.st), so the whole warp takes it when any row does; a
      // row that keeps its reference rewrites the same values.
      const bool bump = mx > kRescale;
      const bool any_bump = __any_sync(0xffffffffu, bump);
      float alpha = 1.f;
      if (any_bump) {
        if (bump) {
          const float m_new = m_ref + mx;
          alpha = exp2f(m_ref - m_new);
          m_ref = m_new;
        }
        tmem_wait_st();
        (void)(wdiag ? pass(std::true_type{}) : pass(std::false_type{}));
      }
      if (any_bump && j > 0) {
        // rescale this row's O to the new reference (O_X(j-1) is complete; O_X(j) waits for P_X(j))
#pragma unroll 1
        for (int cc = 0; cc < D / 32; ++cc) {
          float ov[32];
          tmem_ld32(o_addr + cc * 32, ov);
#pragma unroll
          for (int k = 0; k < 32; ++k) ov[k] *= alpha;
          tmem_st32(o_addr + cc * 32, ov);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bars[kPFull + X]);
      l_run = l_run * alpha + sum;
    }
    // ---- epilogue: out = O / l once the last PV is done; a piece of a split key range leaves its
    // unnormalised O row and (reference, sum) for the merge instead
    if (pieces > 1) {
      if (!timeout && __all_sync(0xffffffffu, mbar_wait(&bars[kDone], 0))) {
        tc_fence_after();
        const int64_t wrow = ws_row0 + X * 128 + r;
        float4 *dst = reinterpret_cast<float4 *>(P.ws_o + wrow * D);
#pragma unroll 1
        for (int cc = 0; cc < D / 32; ++cc) {
          float ov[32];
          tmem_ld32(o_addr + cc * 32, ov);
          if (row_ok) {
#pragma unroll
            for (int q4 = 0; q4 < 8; ++q4)
              dst[cc * 8 + q4] = make_float4(ov[4 * q4], ov[4 * q4 + 1], ov[4 * q4 + 2], ov[4 * q4 + 3]);
          }
        }
        if (row_ok) *reinterpret_cast<float2 *>(P.ws_ml + wrow * 2) = make_float2(m_ref, l_run);
      }
    } else if (!timeout && __all_sync(0xffffffffu, mbar_wait(&bars[kDone], 0))) {
      tc_fence_after();
      const float inv = l_run > 0.f ? (KT != 0 ? P.v_scale[g] : 1.f) / l_run : 0.f;
      uint4 *dst = reinterpret_cast<uint4 *>(P.out + ((int64_t)(q0 + (row_ok ? pos_i : 0)) * P.num_q_heads + h) * D);
#pragma unroll 1
      for (int cc = 0; cc < D / 32; ++cc) {
        float ov[32];
        tmem_ld32(o_addr + cc * 32, ov);
        if (row_ok) {
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4)
            dst[cc * 4 + q4] = make_uint4(pack_bf16x2(ov[8 * q4] * inv, ov[8 * q4 + 1] * inv),
                                          pack_bf16x2(ov[8 * q4 + 2] * inv, ov[8 * q4 + 3] * inv),
                                          pack_bf16x2(ov[8 * q4 + 4] * inv, ov[8 * q4 + 5] * inv),
                                          pack_bf16x2(ov[8 * q4 + 6] * inv, ov[8 * q4 + 7] * inv));
        }
      }
    }
  } else {
#if PA_PREFILL_SPLIT_REGS
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(C::REGS_PRODUCER));
#endif
  if (warp == 8) {
    // ===================================================================== MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = KT != 0 ? idesc_f16(128, C::BN, false) : idesc_bf16(128, C::BN, false);
      constexpr uint32_t idO = KT != 0 ? idesc_f16(128, D, true) : idesc_bf16(128, D, true);
      const uint32_t qa = smem_u32(smem + C::OFF_QA), qb = smem_u32(smem + C::OFF_QB);
      auto ready = [&](int i) {
        const bool r = mbar_wait(&bars[kFull + i % C::NSLOT], (i / C::NSLOT) & 1);
        tc_fence_after();
        return r;
      };
      auto release = [&](int i) { mma_commit(&bars[kEmpty + i % C::NSLOT]); };
      const uint64_t qdesc[2] = {sw128_desc(qa, 16, 1024), sw128_desc(qb, 16, 1024)};
      auto issue_s = [&](int X, int j) {
        mma_ss_group<D / 16, C::Q_PLANE / 16, C::KV_PLANE / 16>(
            tmem + C::s_col(X), qdesc[X], sw128_desc(smem_u32(slot_of(2 * j)), 16, 1024), idS);
        mma_commit(&bars[kSFull + X]);
      };
      auto issue_o = [&](int X, int j) {
        const uint32_t vt = smem_u32(slot_of(2 * j + 1));
        const int nk = j == ntiles - 1 ? last_k16 : C::BN / 16;
        if (nk == C::BN / 16) {
          mma_ts_group8(tmem + C::o_col(X), tmem + C::s_col(X), sw128_desc(vt, C::KV_PLANE, 1024), idO,
                        j > 0 ? 1u : 0u);
        } else {
          for (int kk = 0; kk < nk; ++kk)
            mma_bf16_ts(tmem + C::o_col(X), tmem + C::s_col(X) + kk * 8,
                        sw128_desc(vt + kk * (16 * 128), C::KV_PLANE, 1024), idO, (j > 0 || kk > 0) ? 1u : 0u);
        }
      };
      bool ok = mbar_wait(&bars[kQReady], 0) && ready(0);
      if (ok) {
        issue_s(0, 0);
        issue_s(1, 0);
        release(0);
      }
      for (int j = 0; ok && j < ntiles; ++j) {
        const bool more = j + 1 < ntiles;
        if (!(ok = ready(2 * j + 1))) break;                       // V_j
        if (!(ok = mbar_wait(&bars[kPFull + 0], j & 1))) break;    // P_A(j) in TMEM
        tc_fence_after();
        issue_o(0, j);
        if (more) {
          if (!(ok = ready(2 * j + 2))) break;                     // K_{j+1}
          issue_s(0, j + 1);                                       // after O_A(j) has read P_A(j)
        }
        if (!(ok = mbar_wait(&bars[kPFull + 1], j & 1))) break;    // P_B(j)
        tc_fence_after();
        issue_o(1, j);
        release(2 * j + 1);                                        // V_j read by both PV products
        if (more) {
          issue_s(1, j + 1);
          release(2 * j + 2);                                      // K_{j+1} read by both QK products
        }
      }
      mma_commit(&bars[kDone]);                    // fires once every MMA issued above has completed
      if (!ok) timeout = true;
    }
  } else if (warp == 9) {
    // ===================================================================== TMA producer (whole warp)
    // One copy per lane: a key tile is UPT units x DH planes for K and as many for V (32 copies at
    // head_dim 128), so lane l copies plane l % DH of unit (l / DH) % UPT of K (first half of the
    // warp) or V (second half).  Each lane loads its unit's block-table entry two tiles ahead.
    // One-byte caches: one 128-byte plane per unit, into the staging ring.
    {
      const int32_t *trow = P.block_tables + (int64_t)c * P.max_blocks_per_seq;
      const int ush = P.block_size == 32 ? 1 : 0;   // log2(16-row units per physical block)
      constexpr int UPT = C::BN / kBlock;             // units per key tile
      constexpr int NPL = KT != 0 ? 1 : C::DH;        // 128-byte planes per unit row
      constexpr int PER = UPT * NPL;                  // copies per K or V tile
      constexpr int NRING = KT != 0 ? C::NU8 : C::NSLOT;
      constexpr int FULL = KT != 0 ? kU8Full : kFull, EMPTY = KT != 0 ? kU8Empty : kEmpty;
      constexpr int PLANE_BYTES = KT != 0 ? C::U8_BYTES : C::KV_PLANE;
      static_assert(2 * PER <= 32, "one copy per lane");
      const int w_lane = lane / PER;                  // 0: K, 1: V, 2+: idle
      const int bb = (lane / NPL) % UPT;              // unit of the tile
      const int hh = lane % NPL;                      // 128-byte plane
      auto ring_of = [&](int i) {
        return KT != 0 ? smem + C::OFF_U8 + (i % NRING) * C::U8_BYTES : slot_of(i);
      };
      auto row_of = [&](int j) {                      // cache row of this lane's unit of key tile tl0 + j
        const int u = (tl0 + j) * UPT + bb;
        int e = 0;
        if (w_lane < 2 && j < ntiles && u * kBlock < kv_len) {
          e = (pre_read && j < 2) ? (j == 0 ? pre_e0 : pre_e1) : __ldg(trow + (u >> ush));
          if (e < 0 || e >= P.num_blocks) {
            flag_error(kErrBlockId);
            e = 0;
          }
        }
        return (((e * P.num_kv_heads + g) << ush) + (u & ((1 << ush) - 1))) * kBlock;
      };
      int y0 = row_of(0), y1 = row_of(1);
      int issued = 0;                                 // ring items whose copies are in flight
      for (int j = 0; j < ntiles && !timeout; ++j) {
        const int y2 = row_of(j + 2);
        const int nu = min(UPT, (kv_len - (tl0 + j) * C::BN + kBlock - 1) / kBlock);
        for (int w = 0; w < 2; ++w) {                 // K, then V of tile j
          const int it = 2 * j + w, slot = it % NRING;
          int ok = 1;
          if (lane == 0) {
            if (it >= NRING) ok = mbar_wait(&bars[EMPTY + slot], ((it / NRING) - 1) & 1);
            if (ok) mbar_arrive_expect_tx(&bars[FULL + slot], nu * NPL * (kBlock * 128));
          }
          if (!__shfl_sync(0xffffffffu, ok, 0)) {
            timeout = true;
            break;
          }
          // x: element 64 * hh of the bf16 row, or byte 0 of the one-byte row (16-byte aligned)
          if (w_lane == w && bb < nu)
            tma_load_2d(ring_of(it) + hh * PLANE_BYTES + bb * (kBlock * 128), w ? &vmap : &kmap, hh * 64, y0,
                        &bars[FULL + slot]);
          issued = it + 1;
        }
        y0 = y1;
        y1 = y2;
      }
      // before leaving, the last tiles this warp issued must have landed (a no-op when the MMA warp
      // consumed them; bounded when a wait elsewhere gave up)
      if (lane == 0)
        for (int k = max(0, issued - NRING); k < issued; ++k)
          (void)mbar_wait(&bars[FULL + (k % NRING)], (k / NRING) & 1);
    }
  } else if (warp >= 10) {
    if constexpr (KT != 0) {
      // ===================================================================== one-byte codes -> f16 tiles
      // Warp 10 converts dims 0-63 (plane 0 of the f16 tile), warp 11 dims 64-127.  Per instruction a warp
      // takes 8 rows (lane % 8) x 4 chunks of 16 codes (lane / 8): the 8 lanes of a quarter-warp share a
      // chunk and cover 8 consecutive rows, so both the 16-byte reads and the two 16-byte writes of each
      // lane fall in 8 distinct bank groups (the swizzle XORs the chunk with row % 8).  Rows past the
      // context, including units the producer did not load, are written as zeros: their K columns are
      // masked, and their V rows meet p = 0, which must not meet a NaN code.
      const int w = warp - 10, r8 = lane & 7, cq = lane >> 3;
      const int c = 4 * w + cq;                         // chunk of 16 codes = dims [16c, 16c + 16)
      for (int it = 0; it < 2 * ntiles; ++it) {
        const int su = it % C::NU8, slot = it % C::NSLOT;
        const bool ok = mbar_wait(&bars[kU8Full + su], (it / C::NU8) & 1) &&
                        (it < C::NSLOT || mbar_wait(&bars[kEmpty + slot], ((it / C::NSLOT) - 1) & 1));
        if (!__all_sync(0xffffffffu, ok)) {
          timeout = true;
          break;
        }
        const uint8_t *src = smem + C::OFF_U8 + su * C::U8_BYTES;
        uint8_t *dst = slot_of(it) + w * C::KV_PLANE;
        const int nvalid = kv_len - (tl0 + (it >> 1)) * C::BN;  // rows of this tile holding keys (may exceed BN)
        // eight 16-byte reads in flight per lane, then their conversions and writes; the row test is
        // compiled only into the last tile's pass (a test per read keeps the reads from batching)
        auto convert = [&](auto partial_c) {
          constexpr bool kPartial = decltype(partial_c)::value;
#pragma unroll 1
          for (int i0 = 0; i0 < C::BN / 8; i0 += 8) {
            uint4 v[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              const int R = 8 * (i0 + k) + r8;
              v[k] = (!kPartial || R < nvalid) ? *reinterpret_cast<const uint4 *>(src + R * 128 + ((c ^ r8) << 4))
                                               : make_uint4(0, 0, 0, 0);   // code 0 is +0 in both types
            }
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              const int R = 8 * (i0 + k) + r8;
              uint4 lo, hi;
              bytes4_to_h2<KT>(v[k].x, lo.x, lo.y);
              bytes4_to_h2<KT>(v[k].y, lo.z, lo.w);
              bytes4_to_h2<KT>(v[k].z, hi.x, hi.y);
              bytes4_to_h2<KT>(v[k].w, hi.z, hi.w);
              *reinterpret_cast<uint4 *>(dst + R * 128 + (((2 * cq) ^ r8) << 4)) = lo;
              *reinterpret_cast<uint4 *>(dst + R * 128 + (((2 * cq + 1) ^ r8) << 4)) = hi;
            }
          }
        };
        if (nvalid >= C::BN)
          convert(std::false_type{});
        else
          convert(std::true_type{});
        fence_async_smem();
        mbar_arrive(&bars[kU8Empty + su]);
        mbar_arrive(&bars[kFull + slot]);
      }
    }
  }
  }
  // ---- teardown: every MMA has completed before TMEM is released (bounded waits throughout; on a
  // timeout the error word is set and the CTA leaves without its output)
  if (warp == 8 && lane == 0) (void)mbar_wait(&bars[kDone], 0);
  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// ----------------------------------------------------------------------------- merge of split key ranges
// For each split work item of a plan and head group: every row (position, head) of the item's query-tile
// pair combines its pieces' partials,  out = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s  (M = max_s m_s;
// a piece in which the row saw no key has m = -inf, l = 0 and is left out), times the V scale of a
// one-byte cache.  One warp per row, eight rows per CTA (grid z = the item's 32 groups of eight rows, so
// the merge has as many CTAs in flight as the partials need); lane s holds piece s's (m, l), and each lane
// sums its D/32 dims over the pieces with up to kMergeBatch independent vector loads in flight.
constexpr int kMergeBatch = 8;

template <int D, bool ONE_BYTE>
__global__ void __launch_bounds__(256) prefill_combine_kernel(const PrefillParams P,
                                                              const __grid_constant__ PrefillCombineList L) {
  griddep_wait();  // the partials come from the prefill kernel just before this one
  griddep_launch();
  const int32_t w0 = L.item[blockIdx.y][0], w1 = L.item[blockIdx.y][1];
  const int c = w0 & 0xffff, pair = (w0 >> 16) & 0xffff, pieces = w1 & 0xff, slot0 = (w1 >> 8) & 0xffffff;
  if (c >= P.num_chunks) return;
  const int q0 = P.cu_q_lens[c];
  const int Cn = P.cu_q_lens[c + 1] - q0;
  const int ppt = 128 / P.hpr;
  const int nx = (Cn + 2 * ppt - 1) / (2 * ppt);
  if (Cn <= 0 || pair >= nx) return;
  const int p0 = (nx - 1 - pair) * 2 * ppt;
  const int lane = threadIdx.x & 31;
  const int rr = blockIdx.z * 8 + (threadIdx.x >> 5);   // row of the item's 256 (tile A: 0-127, B: 128-255)
  const int r = rr & 127;
  const int pos_i = p0 + (rr >> 7) * ppt + r / P.hpr;
  if (pos_i >= Cn) return;                               // a padding row (the same for the whole warp)
  const int hg0 = blockIdx.x * P.hpr;
  auto row_of = [&](int s) { return ((int64_t)(slot0 + s) * gridDim.x + blockIdx.x) * 256 + rr; };
  constexpr int DPL = D / 32;
  float acc[DPL];
#pragma unroll
  for (int e = 0; e < DPL; ++e) acc[e] = 0.f;
  float M = -INFINITY;
  for (int s = lane; s < pieces; s += 32) M = fmaxf(M, P.ws_ml[row_of(s) * 2]);
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
  float den = 0.f;
  for (int s0 = 0; s0 < pieces; s0 += 32) {
    // lane k: weight of piece s0 + k (0 for a piece the row saw no key of)
    float w = 0.f;
    if (s0 + lane < pieces) {
      const float2 ml = *reinterpret_cast<const float2 *>(P.ws_ml + row_of(s0 + lane) * 2);
      if (ml.x != -INFINITY) {
        w = exp2f(ml.x - M);
        den = fmaf(w, ml.y, den);
      }
    }
    const int cnt = min(32, pieces - s0);
    for (int k0 = 0; k0 < cnt; k0 += kMergeBatch) {
      float ov[kMergeBatch][DPL];
#pragma unroll
      for (int k = 0; k < kMergeBatch; ++k) {
        if (k0 + k < cnt) {
          const float *op = P.ws_o + row_of(s0 + k0 + k) * D + lane * DPL;
          if constexpr (DPL == 4) {
            const float4 v = *reinterpret_cast<const float4 *>(op);
            ov[k][0] = v.x; ov[k][1] = v.y; ov[k][2] = v.z; ov[k][3] = v.w;
          } else {
            const float2 v = *reinterpret_cast<const float2 *>(op);
            ov[k][0] = v.x; ov[k][1] = v.y;
          }
        }
      }
#pragma unroll
      for (int k = 0; k < kMergeBatch; ++k) {
        const float wk = __shfl_sync(0xffffffffu, w, (k0 + k) & 31);
        if (k0 + k < cnt && wk > 0.f) {
#pragma unroll
          for (int e = 0; e < DPL; ++e) acc[e] = fmaf(wk, ov[k][e], acc[e]);
        }
      }
    }
  }
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) den += __shfl_xor_sync(0xffffffffu, den, off);
  const float vs = ONE_BYTE ? P.v_scale[hg0 / P.group] : 1.f;
  const float inv = den > 0.f ? vs / den : 0.f;
  __nv_bfloat16 *orow = P.out + ((int64_t)(q0 + pos_i) * P.num_q_heads + hg0 + r % P.hpr) * D + lane * DPL;
#pragma unroll
  for (int e = 0; e < DPL; e += 2)
    *reinterpret_cast<__nv_bfloat162 *>(orow + e) = __floats2bfloat162_rn(acc[e] * inv, acc[e + 1] * inv);
}

// ----------------------------------------------------------------------------- host plan
// The launch order and key-range split of a prefill call, from the host copies of its lengths.  Work is
// counted in key tiles per CTA (a query-tile pair of one head group); a CTA runs on one SM.  Candidate
// piece lengths (fractions of the work per SM, and no split) are scored by the makespan of a
// longest-first greedy schedule on the SMs, each piece of a split CTA costing one more tile of set-up;
// the shortest schedule wins, ties to fewer pieces.
struct PrefillPlanHost {
  PrefillPlan<true> plan;
  PrefillCombineList combine;
  int n_items = 0;
  int n_combine = 0;
  int n_slots = 0;   // workspace slots (pieces of split items)
};

// Greedy schedule cost: pieces (lengths in tiles, `copies` CTAs each) longest first onto `sms` SMs.
inline int64_t lpt_makespan(std::vector<int> len, int copies, int sms) {
  std::sort(len.begin(), len.end(), std::greater<int>());
  std::priority_queue<int64_t, std::vector<int64_t>, std::greater<int64_t>> load;
  for (int i = 0; i < sms; ++i) load.push(0);
  int64_t worst = 0;
  for (const int t : len)
    for (int k = 0; k < copies; ++k) {
      const int64_t v = load.top() + t;
      load.pop();
      load.push(v);
      worst = std::max(worst, v);
    }
  return worst;
}

// Returns false when the lengths are out of range (the kernel would flag them) or the work does not fit
// the plan's lists; the caller then launches unplanned.
inline bool plan_prefill(const int32_t *hcu, const int32_t *hctx, int num_chunks, int hpr, int groups_x, int sm_count,
                         int max_q_len, int ctx_limit, PrefillPlanHost &out) {
  if (num_chunks <= 0 || num_chunks > kPlanChunks || groups_x <= 0 || sm_count <= 0) return false;
  const int ppt = 128 / hpr;
  struct Pair {
    int c, k, T;
  };
  std::vector<Pair> pairs;
  int64_t W = 0;
  for (int c = 0; c < num_chunks; ++c) {
    const int Cn = hcu[c + 1] - hcu[c], ctx = hctx[c], H = ctx - Cn;
    if (Cn < 0 || H < 0 || ctx > ctx_limit || Cn > max_q_len) return false;
    const int nx = (Cn + 2 * ppt - 1) / (2 * ppt);
    if (nx > 65535) return false;
    out.plan.pairs[c] = nx;
    for (int k = 0; k < nx; ++k) {
      const int p0 = (nx - 1 - k) * 2 * ppt, p_end = std::min(Cn, p0 + 2 * ppt);
      const int T = (H + p_end + 127) / 128;
      pairs.push_back({c, k, T});
      W += T;
    }
  }
  if (pairs.empty() || pairs.size() > static_cast<size_t>(kPlanItems)) return false;
  auto n_pieces = [](int T, int per) { return (per <= 0 || T <= per) ? 1 : std::min(255, (T + per - 1) / per); };
  auto pieces_for = [&](int per, std::vector<int> *len) {
    int total = 0;
    for (const Pair &p : pairs) {
      const int n = n_pieces(p.T, per);
      const int q = (p.T + n - 1) / n;
      for (int s = 0; s < n; ++s)
        if (len) len->push_back(std::min(q, p.T - s * q) + (n > 1 ? 1 : 0));
      total += n;
    }
    return total;
  };
  // candidate piece lengths; splitting is only weighed while the schedule stays cheap to score
  int best_per = 0;
  {
    std::vector<int> len;
    pieces_for(0, &len);
    int64_t best = lpt_makespan(len, groups_x, sm_count);
    const double per_sm = static_cast<double>(W) * groups_x / sm_count;
    if (static_cast<int64_t>(pairs.size()) * groups_x <= 16384) {
      for (int f10 = 3; f10 <= 10; ++f10) {
        const int per = std::max(4, static_cast<int>(per_sm * f10 / 10.0 + 0.999));
        if (pieces_for(per, nullptr) > kPlanItems) continue;
        len.clear();
        pieces_for(per, &len);
        const int64_t ms = lpt_makespan(len, groups_x, sm_count);
        if (ms < best) {
          best = ms;
          best_per = per;
        }
      }
    }
  }
  // items, longest piece first (ties in chunk, pair, piece order); slots for the split pairs
  struct Item {
    int c, k, s, n, q, len, slot;
  };
  std::vector<Item> items;
  int slots = 0, n_comb = 0;
  for (const Pair &p : pairs) {
    const int n = n_pieces(p.T, best_per);
    const int q = (p.T + n - 1) / n;
    if (q > 65535) return false;
    if (n > 1) {
      out.combine.item[n_comb][0] = p.c | (p.k << 16);
      out.combine.item[n_comb][1] = n | (slots << 8);
      ++n_comb;
    }
    for (int s = 0; s < n; ++s) items.push_back({p.c, p.k, s, n, q, std::min(q, p.T - s * q), n > 1 ? slots + s : 0});
    if (n > 1) slots += n;
  }
  if (slots >= (1 << 23)) return false;
  std::stable_sort(items.begin(), items.end(), [](const Item &a, const Item &b) { return a.len > b.len; });
  for (size_t i = 0; i < items.size(); ++i) {
    const Item &it = items[i];
    out.plan.item[i][0] = it.c | (it.k << 16);
    out.plan.item[i][1] = it.s | (it.n << 8) | (it.q << 16);
    out.plan.slot[i] = it.slot;
  }
  out.n_items = static_cast<int>(items.size());
  out.n_combine = n_comb;
  out.n_slots = slots;
  return true;
}

// Workspace bytes of a plan: the partial rows of every piece of its split items.
inline size_t prefill_plan_workspace(const PrefillPlanHost &pl, int groups_x, int head_dim) {
  return static_cast<size_t>(pl.n_slots) * groups_x * 256 * (head_dim + 2) * sizeof(float);
}

// ----------------------------------------------------------------------------- host launch
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_tiled_fn() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// Tensor map over a cache [num_blocks][Hkv][16][D] (bf16) seen as rows of D elements; box = 16 rows x 64
// elements with the 128-byte swizzle the UMMA K-major / MN-major operands expect.
inline bool make_cache_map(CUtensorMap *map, const void *base, int64_t rows, int D) {
  EncodeTiledFn fn = encode_tiled_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(D) * 2};
  cuuint32_t box[2] = {64, static_cast<cuuint32_t>(kBlock)};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The same over a one-byte cache (FP8 E4M3 or INT8 codes): box = 16 rows x 128 bytes, 128-byte swizzle.
inline bool make_cache_map_u8(CUtensorMap *map, const void *base, int64_t rows, int D) {
  EncodeTiledFn fn = encode_tiled_fn();
  if (!fn || D != 128) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(D)};
  cuuint32_t box[2] = {128, static_cast<cuuint32_t>(kBlock)};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, int KT>
int launch_prefill_d(const PrefillParams &P, const void *k_cache, const void *v_cache, int num_chunks, int max_q_len,
                     const PrefillPlanHost *plan, cudaStream_t st) {
  using C = PrefillCfg<D, KT>;
  CUtensorMap km, vm;
  const int64_t rows = P.num_blocks * P.num_kv_heads * P.block_size;
  if (KT != 0 ? (!make_cache_map_u8(&km, k_cache, rows, D) || !make_cache_map_u8(&vm, v_cache, rows, D))
              : (!make_cache_map(&km, k_cache, rows, D) || !make_cache_map(&vm, v_cache, rows, D)))
    return -3;
  auto prepare = [&](auto kernel) {
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) != cudaSuccess)
      return false;
#if PA_PREFILL_SPLIT_REGS
    // setmaxnreg.inc waits until the block's launch allocation can cover the new split: never launch a
    // build whose register count per thread would not
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, kernel) != cudaSuccess ||
        fa.numRegs * C::THREADS < 2 * 128 * C::REGS_SOFTMAX + 128 * C::REGS_PRODUCER)
      return false;
#endif
    return true;
  };
  const unsigned gx = static_cast<unsigned>(P.num_q_heads / P.hpr);
  if (plan != nullptr) {
    if (!prepare(paged_prefill_kernel<D, KT, true>)) return -3;
    if (launch_pdl(paged_prefill_kernel<D, KT, true>, dim3(gx, static_cast<unsigned>(plan->n_items)),
                   dim3(C::THREADS), C::SMEM, st, km, vm, P, plan->plan) != cudaSuccess)
      return -3;
    if (plan->n_combine > 0 &&
        launch_pdl(prefill_combine_kernel<D, (KT != 0)>, dim3(gx, static_cast<unsigned>(plan->n_combine), 32),
                   dim3(256), 0, st, P, plan->combine) != cudaSuccess)
      return -3;
    return 0;
  }
  if (!prepare(paged_prefill_kernel<D, KT, false>)) return -3;
  const int ppt = C::BM / P.hpr;
  const int tiles = (max_q_len + 2 * ppt - 1) / (2 * ppt);
  if (tiles > 65535) return -1;
  dim3 grid(gx, tiles, num_chunks);
  return launch_pdl(paged_prefill_kernel<D, KT, false>, grid, dim3(C::THREADS), C::SMEM, st, km, vm, P,
                    PrefillPlan<false>{}) == cudaSuccess
             ? 0
             : -3;
}

// kv_dtype: 0 bf16, 1 FP8 E4M3, 2 INT8 (one-byte types: head_dim 128, k_scale / v_scale per KV head).
// plan (optional): the planned order and split of the launch, its partials in ws (plan's workspace bytes).
inline int launch_prefill(void *out, const void *q, const int32_t *cu_q_lens, int num_chunks, const void *k_cache,
                          const void *v_cache, const int32_t *block_tables, int max_blocks_per_seq,
                          const int32_t *context_lens, int num_q_heads, int num_kv_heads, int head_dim,
                          int64_t num_blocks, int block_size, float scale, int kv_dtype, const float *k_scale,
                          const float *v_scale, int max_q_len, int max_context_len, const PrefillPlanHost *plan,
                          void *ws, cudaStream_t st) {
  if (num_chunks > 65535 || num_q_heads > 65535) return -1;
  if (num_blocks * num_kv_heads * block_size >= (int64_t(1) << 31)) return -2;
  PrefillParams P;
  P.out = static_cast<__nv_bfloat16 *>(out);
  P.q = static_cast<const __nv_bfloat16 *>(q);
  P.cu_q_lens = cu_q_lens;
  P.block_tables = block_tables;
  P.context_lens = context_lens;
  P.num_blocks = num_blocks;
  P.block_size = block_size;
  P.max_blocks_per_seq = max_blocks_per_seq;
  P.num_q_heads = num_q_heads;
  P.num_kv_heads = num_kv_heads;
  P.group = num_q_heads / num_kv_heads;
  P.hpr = (P.group <= 128 && 128 % P.group == 0) ? P.group : 1;
  P.max_context_len = max_context_len;
  P.num_chunks = num_chunks;
  P.qscale = scale * 1.4426950408889634f;
  P.k_scale = k_scale;
  P.v_scale = v_scale;
  P.ws_o = static_cast<float *>(ws);
  P.ws_ml = plan != nullptr && ws != nullptr
                ? P.ws_o + static_cast<int64_t>(plan->n_slots) * (num_q_heads / P.hpr) * 256 * head_dim
                : nullptr;
  if (kv_dtype != 0 && (head_dim != 128 || k_scale == nullptr || v_scale == nullptr)) return -1;
  if (plan != nullptr && plan->n_slots > 0 && ws == nullptr) return -1;
  if (kv_dtype == 1) return launch_prefill_d<128, 1>(P, k_cache, v_cache, num_chunks, max_q_len, plan, st);
  if (kv_dtype == 2) return launch_prefill_d<128, 2>(P, k_cache, v_cache, num_chunks, max_q_len, plan, st);
  return head_dim == 128 ? launch_prefill_d<128, 0>(P, k_cache, v_cache, num_chunks, max_q_len, plan, st)
                         : launch_prefill_d<64, 0>(P, k_cache, v_cache, num_chunks, max_q_len, plan, st);
}

}  // namespace pa
