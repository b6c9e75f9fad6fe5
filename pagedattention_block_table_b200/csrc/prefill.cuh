// prefill.cuh -- paged causal prefill on the tcgen05 tensor cores (sm_100a).
//
// What it computes (vLLM overview page, "Continuous Batching": prefill chunks share the batch with
// decoding requests; Core Concepts page §3.2: the chunk's K/V sit in the paged cache, read through
// the block table): for chunk c with history H_c and C_c new tokens, query row i (position H_c + i)
// of head h attends to positions t <= H_c + i of KV head h / G:
//     out[i][h] = softmax_t(scale * q[i][h] . K[t]) V[t].
//
// Design: one CTA (4 warps, one query row per thread) per (128-row query tile, query head, chunk).
// Q is staged once into shared memory in the UMMA K-major 128-byte-swizzled layout.  Keys come in
// tiles of 128 (8 physical blocks): for each block one TMA box of 16 rows x 64 elements per half of
// head_dim is fetched into the same swizzled layout (tensor map over the cache viewed as
// [num_blocks*Hkv*16][head_dim]; no multicast), double-buffered.  One thread issues
//   S = Q K^T   (tcgen05.mma kind::f16, M=128, N=128, K=16 steps, fp32 accumulator in TMEM)
// each thread reads its row of S from TMEM (tcgen05.ld 32x32b), applies the causal mask and a base-2
// online softmax, writes P (bf16) into shared memory in the K-major swizzled layout, and one thread
// issues
//   O += P V  (V used as an MN-major B operand straight from its TMA layout, fp32 accumulator in TMEM).
// p is taken relative to a per-row reference max m_ref; only when a tile's max exceeds m_ref by more
// than 2^8 does the row move m_ref up and rescale its O row in TMEM (tcgen05.ld/st) and its sum l.
// O and l always share m_ref, so out = O / l is exact whichever m_ref was used; p stays <= 256.
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
  int max_blocks_per_seq;
  int num_q_heads;
  int num_kv_heads;
  int group;
  int max_context_len;
  float qscale;  // scale * log2(e)
};

template <int D>
struct PrefillCfg {
  static constexpr int BM = 128;                  // query rows per CTA (= TMEM lanes = threads)
  static constexpr int BN = 128;                  // keys per tile (8 blocks of 16)
  static constexpr int DH = D / 64;               // 64-element (128-byte) planes of a head_dim row
  static constexpr int PLANE = 128 * 128;         // bytes of one 128-row x 64-element plane
  static constexpr int Q_BYTES = DH * PLANE;
  static constexpr int KV_BYTES = DH * PLANE;     // one K or V tile (128 keys)
  static constexpr int P_BYTES = 2 * PLANE;       // 128 rows x 128 keys
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_BYTES;
  static constexpr int OFF_V = OFF_K + 2 * KV_BYTES;
  static constexpr int OFF_P = OFF_V + 2 * KV_BYTES;
  static constexpr int OFF_BAR = OFF_P + P_BYTES;
  static constexpr int SMEM = OFF_BAR + 64 + 1024;  // + slack to align the base to 1024
  static constexpr uint32_t TMEM_COLS = 256;
  static constexpr uint32_t S_COL = 0;
  static constexpr uint32_t O_COL = 128;
  static_assert(D == 64 || D == 128, "head_dim");
};

template <int D>
__global__ void __launch_bounds__(128, 1)
    paged_prefill_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                         const PrefillParams P) {
  using C = PrefillCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5;
  const int mt = blockIdx.x, h = blockIdx.y, c = blockIdx.z;
  const int g = h / P.group;

  const int q0 = P.cu_q_lens[c];
  const int Cn = P.cu_q_lens[c + 1] - q0;
  const int ctx = P.context_lens[c];
  const int H = ctx - Cn;
  if (Cn < 0 || H < 0 || ctx > min(P.max_blocks_per_seq * kBlock, P.max_context_len)) {
    if (tid == 0 && mt == 0 && h == 0) flag_error(kErrLength);
    griddep_wait();
    return;
  }
  const int i0 = mt * C::BM;
  if (i0 >= Cn) {
    griddep_wait();
    return;
  }
  const int rows = min(C::BM, Cn - i0);
  const int kv_len = H + i0 + rows;                   // keys visible to some row of this tile
  const int ntiles = (kv_len + C::BN - 1) / C::BN;

  uint8_t *sQ = smem + C::OFF_Q;
  uint8_t *sK = smem + C::OFF_K;
  uint8_t *sV = smem + C::OFF_V;
  uint8_t *sP = smem + C::OFF_P;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);  // 0,1: K/V tile stages; 2: S; 3: O
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 4);

  if (warp == 0) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  if (tid == 0) {
    for (int b = 0; b < 4; ++b) mbar_init(&bars[b], 1);
    fence_mbar_init();
  }

  // ---- Q rows into shared memory (K-major, 128-byte swizzle: chunk c of row r at c ^ (r % 8))
  {
    uint8_t *rowp = sQ + tid * 128;
    if (tid < rows) {
      const uint4 *src = reinterpret_cast<const uint4 *>(P.q + ((int64_t)(q0 + i0 + tid) * P.num_q_heads + h) * D);
#pragma unroll
      for (int ch = 0; ch < D / 8; ++ch) {
        const uint4 v = src[ch];
        *reinterpret_cast<uint4 *>(rowp + (ch >> 3) * C::PLANE + (((ch & 7) ^ (tid & 7)) << 4)) = v;
      }
    } else {
#pragma unroll
      for (int ch = 0; ch < D / 8; ++ch)
        *reinterpret_cast<uint4 *>(rowp + (ch >> 3) * C::PLANE + (ch & 7) * 16) = make_uint4(0, 0, 0, 0);
    }
  }
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int32_t *trow = P.block_tables + (int64_t)c * P.max_blocks_per_seq;

  // K and V of key tile j (blocks 8j .. 8j+7 that hold keys < kv_len) into stage j % 2
  auto issue_tile = [&](int j) {
    const int stage = j & 1;
    const int nb = min(8, (kv_len - j * C::BN + kBlock - 1) / kBlock);
    mbar_arrive_expect_tx(&bars[stage], nb * 2 * C::DH * (kBlock * 128));
    for (int bb = 0; bb < nb; ++bb) {
      int e = __ldg(trow + j * 8 + bb);
      if (e < 0 || e >= P.num_blocks) {
        flag_error(kErrBlockId);
        e = 0;
      }
      const int y = (e * P.num_kv_heads + g) * kBlock;
#pragma unroll
      for (int hh = 0; hh < C::DH; ++hh) {
        const int off = stage * C::KV_BYTES + hh * C::PLANE + bb * (kBlock * 128);
        tma_load_2d(sK + off, &kmap, hh * 64, y, &bars[stage]);
        tma_load_2d(sV + off, &vmap, hh * 64, y, &bars[stage]);
      }
    }
  };
  // the cache may still be written by the kernel before this one on the stream (the append)
  griddep_wait();
  griddep_launch();
  int issued = 0;
  if (tid == 0) {
    issue_tile(0);
    if (ntiles > 1) issue_tile(1);
  }
  issued = ntiles > 1 ? 2 : 1;

  float m_ref = -INFINITY, l_run = 0.f;
  const bool row_ok = tid < rows;
  const int pos = row_ok ? H + i0 + tid : kv_len - 1;   // padding rows behave like the last row
  const uint32_t lane = static_cast<uint32_t>(warp * 32) << 16;
  constexpr uint32_t idS = idesc_bf16(128, C::BN, false);
  constexpr uint32_t idO = idesc_bf16(128, D, true);
  constexpr float kRescale = 8.f;                       // log2 of the largest p allowed (256)
  bool timeout = false;
  bool s_inflight = false, o_inflight = false;  // thread 0: committed MMAs not yet seen complete
  int j = 0;

  for (; j < ntiles; ++j) {
    const int stage = j & 1;
    timeout |= !mbar_wait(&bars[stage], (j >> 1) & 1);
    uint8_t *kt = sK + stage * C::KV_BYTES;
    uint8_t *vt = sV + stage * C::KV_BYTES;
    if ((j + 1) * C::BN > kv_len) {
      // last tile: V rows of keys no row may see are zeroed so that 0 * V stays 0 in the MMA
      if (j * C::BN + tid >= kv_len) {
#pragma unroll
        for (int hh = 0; hh < C::DH; ++hh)
#pragma unroll
          for (int ch = 0; ch < 8; ++ch)
            *reinterpret_cast<uint4 *>(vt + hh * C::PLANE + tid * 128 + ch * 16) = make_uint4(0, 0, 0, 0);
      }
      fence_async_smem();
    }
    tc_fence_before();
    if (__syncthreads_or(timeout)) break;
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t koff = (kk >> 2) * C::PLANE + (kk & 3) * 32;
        mma_bf16(tmem + C::S_COL, sw128_desc(smem_u32(sQ) + koff, 16, 1024), sw128_desc(smem_u32(kt) + koff, 16, 1024),
                 idS, kk > 0);
      }
      mma_commit(&bars[2]);
      s_inflight = true;
    }
    {
      const bool ok = mbar_wait(&bars[2], j & 1);
      timeout |= !ok;
      if (ok) s_inflight = false;
    }
    tc_fence_after();

    // -- row max of this tile (masked)
    const int kbase = j * C::BN;
    float mt_ = -INFINITY;
#pragma unroll 1
    for (int cc = 0; cc < C::BN / 32; ++cc) {
      float s[32];
      tmem_ld32(tmem + lane + C::S_COL + cc * 32, s);
#pragma unroll
      for (int k = 0; k < 32; ++k) {
        const float x = (kbase + cc * 32 + k <= pos) ? s[k] * P.qscale : -INFINITY;
        mt_ = fmaxf(mt_, x);
      }
    }
    // -- move the reference max (and rescale this row of O and l) only when p would exceed 2^8
    const bool bump = mt_ > m_ref + kRescale;
    if (__any_sync(0xffffffffu, bump)) {
      const float m_new = bump ? mt_ : m_ref;
      const float alpha = exp2f(m_ref - m_new);          // 0 when m_ref is still -inf
      if (j > 0) {
#pragma unroll 1
        for (int cc = 0; cc < D / 32; ++cc) {
          float ov[32];
          tmem_ld32(tmem + lane + C::O_COL + cc * 32, ov);
#pragma unroll
          for (int k = 0; k < 32; ++k) ov[k] *= alpha;
          tmem_st32(tmem + lane + C::O_COL + cc * 32, ov);
        }
      }
      l_run *= alpha;
      m_ref = m_new;
    }
    // -- p = 2^(s - m_ref) into the P tile (bf16, K-major swizzled), row sum
    float ls = 0.f;
    uint8_t *prow = sP + tid * 128;
#pragma unroll 1
    for (int cc = 0; cc < C::BN / 32; ++cc) {
      float s[32];
      tmem_ld32(tmem + lane + C::S_COL + cc * 32, s);
      uint32_t pk[16];
#pragma unroll
      for (int k = 0; k < 32; k += 2) {
        const int t = kbase + cc * 32 + k;
        const float p0 = (t <= pos) ? exp2f(s[k] * P.qscale - m_ref) : 0.f;
        const float p1 = (t + 1 <= pos) ? exp2f(s[k + 1] * P.qscale - m_ref) : 0.f;
        ls += p0 + p1;
        pk[k / 2] = pack_bf16x2(p0, p1);
      }
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        const int kb = cc * 32 + q4 * 8;              // first key of this 16-byte chunk
        const int ch = (kb & 63) >> 3;
        *reinterpret_cast<uint4 *>(prow + (kb >> 6) * C::PLANE + ((ch ^ (tid & 7)) << 4)) =
            make_uint4(pk[4 * q4], pk[4 * q4 + 1], pk[4 * q4 + 2], pk[4 * q4 + 3]);
      }
    }
    l_run += ls;
    fence_async_smem();
    tc_fence_before();
    if (__syncthreads_or(timeout)) break;
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < C::BN / 16; ++kk) {
        const uint32_t aoff = (kk >> 2) * C::PLANE + (kk & 3) * 32;
        mma_bf16(tmem + C::O_COL, sw128_desc(smem_u32(sP) + aoff, 16, 1024),
                 sw128_desc(smem_u32(vt) + kk * (16 * 128), C::PLANE, 1024), idO, (j > 0 || kk > 0) ? 1u : 0u);
      }
      mma_commit(&bars[3]);
      o_inflight = true;
    }
    {
      const bool ok = mbar_wait(&bars[3], j & 1);
      timeout |= !ok;
      if (ok) o_inflight = false;
    }
    tc_fence_after();
    if (j + 2 < ntiles) {
      if (tid == 0) issue_tile(j + 2);  // both MMAs reading this stage are complete
      issued = j + 3;
    }
  }

  if (j < ntiles) {
    // a wait gave up (error word already set): let this CTA's outstanding copies and MMAs land
    // (bounded), then release TMEM and leave without writing
    if (tid == 0) {
      for (int k = j; k < issued; ++k) (void)mbar_wait(&bars[k & 1], (k >> 1) & 1);
      if (s_inflight) (void)mbar_wait(&bars[2], j & 1);
      if (o_inflight) (void)mbar_wait(&bars[3], j & 1);
    }
  } else {
    // out = O / l, read back from TMEM in 32-column pieces (every thread takes part in the loads)
    const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
    uint4 *dst = reinterpret_cast<uint4 *>(P.out + ((int64_t)(q0 + i0 + (row_ok ? tid : 0)) * P.num_q_heads + h) * D);
#pragma unroll 1
    for (int cc = 0; cc < D / 32; ++cc) {
      float ov[32];
      tmem_ld32(tmem + lane + C::O_COL + cc * 32, ov);
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
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
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
  const int64_t rows = P.num_blocks * P.num_kv_heads * kBlock;
  if (!make_cache_map(&km, k_cache, rows, D) || !make_cache_map(&vm, v_cache, rows, D)) return -3;
  if (cudaFuncSetAttribute(paged_prefill_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) !=
      cudaSuccess)
    return -3;
  dim3 grid((max_q_len + C::BM - 1) / C::BM, P.num_q_heads, num_chunks);
  return launch_pdl(paged_prefill_kernel<D>, grid, dim3(128), C::SMEM, st, km, vm, P) == cudaSuccess ? 0 : -3;
}

inline int launch_prefill(void *out, const void *q, const int32_t *cu_q_lens, int num_chunks, const void *k_cache,
                          const void *v_cache, const int32_t *block_tables, int max_blocks_per_seq,
                          const int32_t *context_lens, int num_q_heads, int num_kv_heads, int head_dim,
                          int64_t num_blocks, float scale, int max_q_len, int max_context_len, cudaStream_t st) {
  if (num_chunks > 65535 || num_q_heads > 65535) return -1;
  if (num_blocks * num_kv_heads * kBlock >= (int64_t(1) << 31)) return -2;
  PrefillParams P;
  P.out = static_cast<__nv_bfloat16 *>(out);
  P.q = static_cast<const __nv_bfloat16 *>(q);
  P.cu_q_lens = cu_q_lens;
  P.block_tables = block_tables;
  P.context_lens = context_lens;
  P.num_blocks = num_blocks;
  P.max_blocks_per_seq = max_blocks_per_seq;
  P.num_q_heads = num_q_heads;
  P.num_kv_heads = num_kv_heads;
  P.group = num_q_heads / num_kv_heads;
  P.max_context_len = max_context_len;
  P.qscale = scale * 1.4426950408889634f;
  return head_dim == 128 ? launch_prefill_d<128>(P, k_cache, v_cache, num_chunks, max_q_len, st)
                         : launch_prefill_d<64>(P, k_cache, v_cache, num_chunks, max_q_len, st);
}

}  // namespace pa
