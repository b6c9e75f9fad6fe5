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
// Keys come in tiles of 64 (4 physical blocks): one TMA box of 16 rows x 64 elements per block and per
// 64-element plane of head_dim, into the UMMA 128-byte-swizzled layout, three tiles in flight (tensor
// map over the cache seen as [num_blocks*Hkv*16][head_dim]; no multicast).  Each query tile has two S
// buffers in TMEM, so S of key tile j+2 is computed while the softmax still works on tile j.
// Per key tile j and query tile X:
//   S_X = Q_X K_j^T  (M=128, N=64, fp32 in TMEM)   ->  softmax warps: base-2 online softmax, P_X (bf16,
//   K-major swizzled) into shared memory          ->  O_X += P_X V_j  (M=128, N=head_dim, fp32 in TMEM).
// p is taken relative to a per-row reference max; only when a tile's max exceeds it by more than 2^8
// does the row move the reference and rescale its O row in TMEM (tcgen05.ld/st) and its sum l.  O and l
// always share the reference, so out = O / l is exact whichever reference was used.
#pragma once
#include "pa_common.cuh"

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

// This thread's TMEM lane, 32 consecutive fp32 columns starting at taddr's column.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// This thread's TMEM lane, 64 consecutive fp32 columns (one load, one wait).
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, float (&v)[64]) {
  uint32_t r[64];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x64.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, "
      "%32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, "
      "%48, %49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63}, [%64];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]),
        "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]),
        "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]),
        "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]),
        "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 64; ++i) v[i] = __uint_as_float(r[i]);
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
  float qscale;         // scale * log2(e)
};

#ifndef PA_PREFILL_STAGES
#define PA_PREFILL_STAGES 4
#endif

template <int D>
struct PrefillCfg {
  static constexpr int BM = 128;                  // rows per query tile (= TMEM lanes)
  static constexpr int BN = 64;                   // keys per key tile (4 blocks)
  static constexpr int STAGES = PA_PREFILL_STAGES;  // K/V tiles in flight: S runs two tiles ahead of PV
  static constexpr int DH = D / 64;               // 64-element (128-byte) planes of a head_dim row
  static constexpr int Q_PLANE = BM * 128;        // 16 KB
  static constexpr int KV_PLANE = BN * 128;       // 8 KB
  static constexpr int Q_BYTES = DH * Q_PLANE;
  static constexpr int KV_BYTES = DH * KV_PLANE;  // one K or V tile
  static constexpr int P_BYTES = BM * 128;        // 128 rows x 64 keys bf16
  static constexpr int OFF_QA = 0;
  static constexpr int OFF_QB = OFF_QA + Q_BYTES;
  static constexpr int OFF_K = OFF_QB + Q_BYTES;
  static constexpr int OFF_V = OFF_K + STAGES * KV_BYTES;
  static constexpr int OFF_PA = OFF_V + STAGES * KV_BYTES;
  static constexpr int OFF_PB = OFF_PA + P_BYTES;
  static constexpr int OFF_BAR = OFF_PB + P_BYTES;
  static constexpr int NBAR = 24;
  static constexpr int SMEM = OFF_BAR + NBAR * 8 + 16 + 1024;  // + slack to align the base to 1024
  static constexpr uint32_t TMEM_COLS = 512;
  // TMEM columns: S of tile X, buffer b at 64*(2X+b); O of tile X at 256 + 128X
  __host__ __device__ static constexpr uint32_t s_col(int X, int b) { return 64u * (2u * X + b); }
  __host__ __device__ static constexpr uint32_t o_col(int X) { return 256u + 128u * X; }
  static constexpr int THREADS = 320;
  static_assert(D == 64 || D == 128, "head_dim");
  static_assert(SMEM <= 227 * 1024, "shared memory");

};

// mbarrier slots
// kKvFull/kKvEmpty: per stage; kSFull: per (tile X, buffer b) at kSFull + 2X + b; kOFull, kPFull: per tile
enum : int {
  kKvFull = 0,
  kKvEmpty = kKvFull + PA_PREFILL_STAGES,
  kSFull = kKvEmpty + PA_PREFILL_STAGES,
  kOFull = kSFull + 4,
  kPFull = kOFull + 2,
  kQReady = kPFull + 2,
  kDone = kQReady + 1,
  kNumBars = kDone + 1
};

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 2^x for a packed pair on the FMA pipe (to take load off the MUFU unit): x = n + f with n = rint(x)
// (add/subtract 1.5*2^23) and f in [-0.5, 0.5]; 2^f by a cubic fitted here to minimise the relative
// error on that interval (max 7.5e-5, below the bf16 resolution P is rounded to); 2^n is added to the
// exponent field.  Arguments below -125 give 0 (as the flush-to-zero ex2 does for results in the
// denormal range); -inf gives 0.
__device__ __forceinline__ uint64_t ex2_poly2(float xa, float xb) {
  const float x0 = fmaxf(xa, -125.f), x1 = fmaxf(xb, -125.f);
  const uint64_t shifter = f2pack(12582912.f, 12582912.f), xx = f2pack(x0, x1);
  uint64_t t, n2, f2;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(t) : "l"(xx), "l"(shifter));
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(n2) : "l"(t), "l"(shifter));
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(f2) : "l"(xx), "l"(n2));
  uint64_t p = f2pack(0.05517394095659256f, 0.05517394095659256f);
  p = ffma2(p, f2, f2pack(0.24261131882667542f, 0.24261131882667542f));
  p = ffma2(p, f2, f2pack(0.6932605504989624f, 0.6932605504989624f));
  p = ffma2(p, f2, f2pack(0.9999280571937561f, 0.9999280571937561f));
  const float2 tv = f2unpack(t), pv = f2unpack(p);
  const float a = x0 > -125.f ? __int_as_float(__float_as_int(pv.x) + (__float_as_int(tv.x) << 23)) : 0.f;
  const float b = x1 > -125.f ? __int_as_float(__float_as_int(pv.y) + (__float_as_int(tv.y) << 23)) : 0.f;
  return f2pack(a, b);
}

// One 8-key chunk in PA_PREFILL_POLY_EVERY takes its exponentials from ex2_poly2 (0 = none).
#ifndef PA_PREFILL_POLY_EVERY
#define PA_PREFILL_POLY_EVERY 0
#endif

template <int D>
__global__ void __launch_bounds__(320, 1)
    paged_prefill_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                         const PrefillParams P) {
  using C = PrefillCfg<D>;
  static_assert(kNumBars <= C::NBAR, "barrier slots");
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int c = blockIdx.z;
  const int hg0 = blockIdx.y * P.hpr;                 // first query head of this CTA's rows
  const int g = hg0 / P.group;                        // their KV head
  const int ppt = C::BM / P.hpr;                      // positions per query tile
  // any input may come from the kernel before this one on the stream (launched with PDL)
  griddep_wait();
  griddep_launch();

  const int q0 = P.cu_q_lens[c];
  const int Cn = P.cu_q_lens[c + 1] - q0;
  const int ctx = P.context_lens[c];
  const int H = ctx - Cn;
  if (Cn < 0 || H < 0 || ctx > min(P.max_blocks_per_seq * P.block_size, P.max_context_len)) {
    if (tid == 0 && blockIdx.x == 0 && blockIdx.y == 0) flag_error(kErrLength);
    return;
  }
  const int p0 = blockIdx.x * 2 * ppt;               // first position of tile A
  if (p0 >= Cn) return;
  const int p_end = min(Cn, p0 + 2 * ppt);
  const int kv_len = H + p_end;                       // keys visible to some row of this CTA
  const int ntiles = (kv_len + C::BN - 1) / C::BN;

  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + C::NBAR);
  if (warp == 8) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  if (tid == 0) {
    for (int i = 0; i < C::STAGES; ++i) {
      mbar_init(&bars[kKvFull + i], 1);
      mbar_init(&bars[kKvEmpty + i], 1);
    }
    for (int i = 0; i < 4; ++i) mbar_init(&bars[kSFull + i], 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars[kOFull + i], 1);
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

  if (warp < 8) {
    // ===================================================================== softmax warpgroups
    const int X = warp >> 2;                          // 0: tile A, 1: tile B
    const int r = tid & 127;                          // row = TMEM lane
    const int pos_i = p0 + X * ppt + r / P.hpr;       // position within the chunk
    const int h = hg0 + r % P.hpr;
    const bool row_ok = pos_i < Cn;
    const int pos = row_ok ? H + pos_i : kv_len - 1;  // padding rows behave like the last row
    uint8_t *sQ = smem + (X ? C::OFF_QB : C::OFF_QA);
    uint8_t *sP = smem + (X ? C::OFF_PB : C::OFF_PA);
    // Q row into the K-major 128-byte-swizzled tile (chunk ch of row r at ch ^ (r % 8))
    {
      uint8_t *rowp = sQ + r * 128;
      if (row_ok) {
        const uint4 *src = reinterpret_cast<const uint4 *>(P.q + ((int64_t)(q0 + pos_i) * P.num_q_heads + h) * D);
#pragma unroll
        for (int ch = 0; ch < D / 8; ++ch)
          *reinterpret_cast<uint4 *>(rowp + (ch >> 3) * C::Q_PLANE + (((ch & 7) ^ (r & 7)) << 4)) = src[ch];
      } else {
#pragma unroll
        for (int ch = 0; ch < D / 8; ++ch)
          *reinterpret_cast<uint4 *>(rowp + (ch >> 3) * C::Q_PLANE + (ch & 7) * 16) = make_uint4(0, 0, 0, 0);
      }
      fence_async_smem();
      mbar_arrive(&bars[kQReady]);
    }
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t o_addr = tmem + lane_base + C::o_col(X);
    constexpr float kRescale = 8.f;
    const float qs = P.qscale;
    float m_ref = -INFINITY, l_run = 0.f;
    for (int j = 0; j < ntiles; ++j) {
      // every wait's outcome is made warp-uniform: the tcgen05.ld/st below are warp-collective
      if (!__all_sync(0xffffffffu, mbar_wait(&bars[kSFull + 2 * X + (j & 1)], (j >> 1) & 1))) { timeout = true; break; }
      tc_fence_after();
      float s[C::BN];
      tmem_ld64(tmem + lane_base + C::s_col(X, j & 1), s);
      const int kbase = j * C::BN;
      // scaled row max of this tile; masked keys (past the row's position) become -inf
      float mt_ = -INFINITY;
      if (kbase + C::BN - 1 <= pos) {
        // max of s * qscale: the max of s for a positive scale, the min for a negative one; eight
        // independent partial results so the reduction is not one long dependent chain
        float e[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) e[k] = s[k];
        if (qs >= 0.f) {
#pragma unroll
          for (int k = 8; k < C::BN; ++k) e[k & 7] = fmaxf(e[k & 7], s[k]);
#pragma unroll
          for (int w = 4; w >= 1; w >>= 1)
#pragma unroll
            for (int k = 0; k < w; ++k) e[k] = fmaxf(e[k], e[k + w]);
        } else {
#pragma unroll
          for (int k = 8; k < C::BN; ++k) e[k & 7] = fminf(e[k & 7], s[k]);
#pragma unroll
          for (int w = 4; w >= 1; w >>= 1)
#pragma unroll
            for (int k = 0; k < w; ++k) e[k] = fminf(e[k], e[k + w]);
        }
        mt_ = e[0] * qs;
      } else {
        float e[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) e[k] = -INFINITY;
#pragma unroll
        for (int k = 0; k < C::BN; ++k)
          if (kbase + k <= pos) e[k & 7] = fmaxf(e[k & 7], s[k] * qs);
#pragma unroll
        for (int w = 4; w >= 1; w >>= 1)
#pragma unroll
          for (int k = 0; k < w; ++k) e[k] = fmaxf(e[k], e[k + w]);
        mt_ = e[0];
      }
      const bool diag = kbase + C::BN - 1 > pos;       // some key of this tile is past the row
      // the previous tile's PV must be complete before O is rescaled or P is overwritten
      if (j > 0 && !__all_sync(0xffffffffu, mbar_wait(&bars[kOFull + X], (j - 1) & 1))) { timeout = true; break; }
      tc_fence_after();
      const bool bump = mt_ > m_ref + kRescale;
      if (__any_sync(0xffffffffu, bump)) {
        const float m_new = bump ? mt_ : m_ref;
        const float alpha = exp2f(m_ref - m_new);
        if (j > 0) {
#pragma unroll 1
          for (int cc = 0; cc < D / 32; ++cc) {
            float ov[32];
            tmem_ld32(o_addr + cc * 32, ov);
#pragma unroll
            for (int k = 0; k < 32; ++k) ov[k] *= alpha;
            tmem_st32(o_addr + cc * 32, ov);
          }
        }
        l_run *= alpha;
        m_ref = m_new;
      }
      // last key tile: V rows of keys no row may see are zeroed (tile A's threads, one row each), so
      // that 0 * (whatever the cache holds past the context) never reaches the MMA
      if (X == 0 && r < C::BN && (j + 1) * C::BN > kv_len && kbase + r >= kv_len) {
        uint8_t *vt = smem + C::OFF_V + (j % C::STAGES) * C::KV_BYTES;
#pragma unroll
        for (int hh = 0; hh < C::DH; ++hh)
#pragma unroll
          for (int ch = 0; ch < 8; ++ch)
            *reinterpret_cast<uint4 *>(vt + hh * C::KV_PLANE + r * 128 + ch * 16) = make_uint4(0, 0, 0, 0);
      }
      uint64_t ls2[4] = {0ull, 0ull, 0ull, 0ull};   // independent partial row sums
      const uint64_t qs2 = f2pack(qs, qs), nm2 = f2pack(-m_ref, -m_ref);
      uint8_t *prow = sP + r * 128;
#pragma unroll
      for (int q8 = 0; q8 < C::BN / 8; ++q8) {
        uint32_t pk[4];
#pragma unroll
        for (int k2 = 0; k2 < 4; ++k2) {
          // x = s * qscale - m_ref for two keys at once; keys past the row's position get p = 0
          float2 x = f2unpack(ffma2(f2pack(s[q8 * 8 + 2 * k2], s[q8 * 8 + 2 * k2 + 1]), qs2, nm2));
          if (diag) {
            const int t = kbase + q8 * 8 + 2 * k2;
            if (t > pos) x.x = -INFINITY;
            if (t + 1 > pos) x.y = -INFINITY;
          }
#if PA_PREFILL_POLY_EVERY > 0
          float a, b;
          if (q8 % PA_PREFILL_POLY_EVERY == PA_PREFILL_POLY_EVERY - 1) {
            const float2 e = f2unpack(ex2_poly2(x.x, x.y));
            a = e.x;
            b = e.y;
          } else {
            a = ex2(x.x);
            b = ex2(x.y);
          }
#else
          const float a = ex2(x.x);
          const float b = ex2(x.y);
#endif
          ls2[k2] = f2add(ls2[k2], f2pack(a, b));
          pk[k2] = pack_bf16x2(a, b);
        }
        *reinterpret_cast<uint4 *>(prow + ((q8 ^ (r & 7)) << 4)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      }
      const float2 lsv = f2unpack(f2add(f2add(ls2[0], ls2[1]), f2add(ls2[2], ls2[3])));
      const float ls = lsv.x + lsv.y;
      l_run += ls;
      fence_async_smem();
      tc_fence_before();
      mbar_arrive(&bars[kPFull + X]);
    }
    // ---- epilogue: out = O / l once the last PV is done
    if (!timeout && __all_sync(0xffffffffu, mbar_wait(&bars[kOFull + X], (ntiles - 1) & 1))) {
      tc_fence_after();
      const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
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
  } else if (warp == 8) {
    // ===================================================================== MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16(128, C::BN, false);
      constexpr uint32_t idO = idesc_bf16(128, D, true);
      const uint32_t qa = smem_u32(smem + C::OFF_QA), qb = smem_u32(smem + C::OFF_QB);
      const uint32_t pa = smem_u32(smem + C::OFF_PA), pb = smem_u32(smem + C::OFF_PB);
      const uint32_t kb0 = smem_u32(smem + C::OFF_K), vb0 = smem_u32(smem + C::OFF_V);
      auto issue_s = [&](int X, int j) {
        const uint32_t qx = X ? qb : qa;
        const uint32_t kt = kb0 + (j % C::STAGES) * C::KV_BYTES;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t ko = (kk & 3) * 32;
          mma_bf16(tmem + C::s_col(X, j & 1), sw128_desc(qx + (kk >> 2) * C::Q_PLANE + ko, 16, 1024),
                   sw128_desc(kt + (kk >> 2) * C::KV_PLANE + ko, 16, 1024), idS, kk > 0);
        }
        mma_commit(&bars[kSFull + 2 * X + (j & 1)]);
      };
      auto issue_o = [&](int X, int j) {
        const uint32_t px = X ? pb : pa;
        const uint32_t vt = vb0 + (j % C::STAGES) * C::KV_BYTES;
#pragma unroll
        for (int kk = 0; kk < C::BN / 16; ++kk)
          mma_bf16(tmem + C::o_col(X), sw128_desc(px + kk * 32, 16, 1024),
                   sw128_desc(vt + kk * (16 * 128), C::KV_PLANE, 1024), idO, (j > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&bars[kOFull + X]);
      };
      auto kv_ready = [&](int j) {
        const bool r = mbar_wait(&bars[kKvFull + (j % C::STAGES)], (j / C::STAGES) & 1);
        tc_fence_after();
        return r;
      };
      // S runs up to two key tiles ahead of PV (two S buffers per query tile)
      bool ok = mbar_wait(&bars[kQReady], 0) && kv_ready(0);
      if (ok) {
        issue_s(0, 0);
        issue_s(1, 0);
      }
      if (ok && ntiles > 1 && (ok = kv_ready(1))) {
        issue_s(0, 1);
        issue_s(1, 1);
      }
      for (int j = 0; ok && j < ntiles; ++j) {
        if (!(ok = mbar_wait(&bars[kPFull + 0], j & 1))) break;
        tc_fence_after();
        issue_o(0, j);
        const bool more = j + 2 < ntiles;
        if (more) {
          if (!(ok = kv_ready(j + 2))) break;
          issue_s(0, j + 2);   // into the buffer softmax A has just finished reading
        }
        if (!(ok = mbar_wait(&bars[kPFull + 1], j & 1))) break;
        tc_fence_after();
        issue_o(1, j);
        mma_commit(&bars[kKvEmpty + (j % C::STAGES)]);   // every product reading tile j issued
        if (more) issue_s(1, j + 2);
      }
      mma_commit(&bars[kDone]);                    // fires once every MMA issued above has completed
      if (!ok) timeout = true;
    }
  } else {
    // ===================================================================== TMA producer
    if (lane == 0) {
      const int32_t *trow = P.block_tables + (int64_t)c * P.max_blocks_per_seq;
      int j = 0;
      for (; j < ntiles; ++j) {
        const int st = j % C::STAGES;
        if (j >= C::STAGES && !mbar_wait(&bars[kKvEmpty + st], ((j - C::STAGES) / C::STAGES) & 1)) {
          timeout = true;
          break;
        }
        const int nb = min(C::BN / kBlock, (kv_len - j * C::BN + kBlock - 1) / kBlock);
        mbar_arrive_expect_tx(&bars[kKvFull + st], nb * 2 * C::DH * (kBlock * 128));
        const int upb = P.block_size / kBlock;   // 16-row units per physical block
        for (int bb = 0; bb < nb; ++bb) {
          const int u = j * (C::BN / kBlock) + bb;   // 16-token unit of the sequence
          int e = __ldg(trow + u / upb);
          if (e < 0 || e >= P.num_blocks) {
            flag_error(kErrBlockId);
            e = 0;
          }
          const int y = ((e * P.num_kv_heads + g) * upb + u % upb) * kBlock;
#pragma unroll
          for (int hh = 0; hh < C::DH; ++hh) {
            const int off = st * C::KV_BYTES + hh * C::KV_PLANE + bb * (kBlock * 128);
            tma_load_2d(smem + C::OFF_K + off, &kmap, hh * 64, y, &bars[kKvFull + st]);
            tma_load_2d(smem + C::OFF_V + off, &vmap, hh * 64, y, &bars[kKvFull + st]);
          }
        }
      }
      // before leaving, the last (at most two) tiles this thread issued must have landed (a no-op when
      // the MMA warp consumed them; bounded when a wait elsewhere gave up)
      for (int k = max(0, j - C::STAGES); k < j; ++k)
        (void)mbar_wait(&bars[kKvFull + (k % C::STAGES)], (k / C::STAGES) & 1);
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

template <int D>
int launch_prefill_d(const PrefillParams &P, const void *k_cache, const void *v_cache, int num_chunks, int max_q_len,
                     cudaStream_t st) {
  using C = PrefillCfg<D>;
  CUtensorMap km, vm;
  const int64_t rows = P.num_blocks * P.num_kv_heads * P.block_size;
  if (!make_cache_map(&km, k_cache, rows, D) || !make_cache_map(&vm, v_cache, rows, D)) return -3;
  if (cudaFuncSetAttribute(paged_prefill_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) !=
      cudaSuccess)
    return -3;
  const int ppt = C::BM / P.hpr;
  dim3 grid((max_q_len + 2 * ppt - 1) / (2 * ppt), P.num_q_heads / P.hpr, num_chunks);
  return launch_pdl(paged_prefill_kernel<D>, grid, dim3(C::THREADS), C::SMEM, st, km, vm, P) == cudaSuccess ? 0 : -3;
}

inline int launch_prefill(void *out, const void *q, const int32_t *cu_q_lens, int num_chunks, const void *k_cache,
                          const void *v_cache, const int32_t *block_tables, int max_blocks_per_seq,
                          const int32_t *context_lens, int num_q_heads, int num_kv_heads, int head_dim,
                          int64_t num_blocks, int block_size, float scale, int max_q_len, int max_context_len,
                          cudaStream_t st) {
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
  P.qscale = scale * 1.4426950408889634f;
  return head_dim == 128 ? launch_prefill_d<128>(P, k_cache, v_cache, num_chunks, max_q_len, st)
                         : launch_prefill_d<64>(P, k_cache, v_cache, num_chunks, max_q_len, st);
}

}  // namespace pa
