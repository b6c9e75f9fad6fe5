// decode_mma.cuh -- paged decode attention for GQA groups on the tensor cores (sm_100a).
//
// Same operation and split-K scheme as paged_decode_kernel (decode.cuh): for sequence b and query head
// h, out = softmax(scale * q . K^T) V over the context, token t read through the block table.  With a
// group of G query heads per KV head, every K/V element meets G queries, so the CUDA-core kernel's
// work per byte of KV grows with G; at G = 8 it is compute-bound at about half the HBM bandwidth.  Here
// the products go to the tensor cores instead (warp-level mma.sync m16n8k16, fp32 accumulate): the
// CTA's query heads are the 16 rows of the A operand (padded with zeros when G < 16), and a 16-token
// block is one N=16 QK^T product and one K=16 PV product per warp.
//
// Per warp and 16-token block:
//   S[16 heads][16 tokens] = Q K^T     2 n-tiles of 8 tokens x D/16 k-steps; Q's fragments sit in
//                                      registers for the whole launch, K's are read from shared memory
//   online softmax in base 2 on S's fragments (a row's 16 scores are spread over the 4 lanes of a quad)
//   O[16][D] += P V                    P (bf16) is built from S's fragments in registers; V's fragments
//                                      come from shared memory with ldmatrix.trans (V is token-major)
// bf16 caches: bf16 products.  K and V tiles reach shared memory by 2-D TMA (the cache seen as rows of D
// elements, one 16-row x 128-byte box per 128-byte plane, 128-byte swizzle, into this CTA's own shared
// memory), so ldmatrix and the 16-byte K loads are free of bank conflicts.  The dims of a k-step are
// permuted (the same way for Q and K, which leaves the dot product unchanged) so that each lane's K
// fragments come from two 16-byte loads.
//
// One-byte caches (FP8 E4M3, INT8; head_dim 128): the products run in f16 (m16n8k16, f32 accumulate).
// Every E4M3 and INT8 code is exact in f16.  Q is scaled per row by a power of two into [1, 2) before it
// is rounded to f16 (exact for every bf16 entry within 2^-14 of the row's largest), and that power, the
// softmax scale and the K scale multiply the scores; the V scale multiplies the output.  A lane converts
// the 32 bytes [32p, 32p+32) of a K row into 16 f16 pairs (k-step s takes pairs 2s and 2s+1, and Q uses
// the same dims).  V needs pairs along tokens: a lane reads 16 dims [16g, 16g + 16) of two token rows
// and a byte permute pairs the two rows' codes of each dim before the conversion, which gives the B
// fragment of n-tile e (column g = dim 16g + e); n-tile e of the output then holds dims 32p + e and
// 32p + 16 + e.  With up to 8 query heads (the rows 8-15 of the products above would stay empty) the
// one-byte products are transposed instead: S^T = K Q^T puts the block's 16 tokens on M and the heads on
// N, O^T += V^T P^T the dims on M, so each block takes 8 + 8 products instead of 16 + 16; the scores'
// C fragments are turned into P^T's B fragments by movmatrix, and a head's softmax column spans the 8
// lanes of one pair index.
#pragma once
#include "decode.cuh"
#include "prefill.cuh"   // tensor-map encoding, 2-D TMA load

namespace pa {

template <int KT, int D, int NW, int STAGES>
struct DecodeMmaCfg {
  static constexpr int E = KT == 0 ? 2 : 1;             // bytes per cache element
  static constexpr int ROWB = D * E;                    // bytes of one token row of one head
  static constexpr int PLANES = ROWB / 128;             // 128-byte planes of a row
  static constexpr int PLANE = kBlock * 128;            // one 16-row plane: 2 KB
  static constexpr int TILE = PLANES * PLANE;           // one (unit, head) K or V tile
  static constexpr int KS = D / 16;                     // k-steps of the QK product
  static constexpr int NT = D / 8;                      // 8-dim n-tiles of the PV product
  static constexpr int BAR_BYTES = STAGES * 8;
  static constexpr int ML = 16 * D;                     // offset of the (m, l) pairs in a warp's merge area
  // a warp's tiles, reused at the end as its merge area (16 rows of O and their (m, l)), then its barriers
  static constexpr int DATA = 2 * STAGES * TILE > (ML + 32) * 4 ? 2 * STAGES * TILE : (ML + 32) * 4;
  // swizzled tiles need 1024-byte alignment: each warp's area is a multiple of 1024
  static constexpr int WARP_BYTES = ((DATA + BAR_BYTES) + 1023) / 1024 * 1024;
  static constexpr int SMEM = NW * WARP_BYTES + 1024;   // + slack to align the base
  static_assert(D == 64 || D == 128, "head_dim");
  static_assert(KT == 0 || D == 128, "one-byte caches: head_dim 128");
};

// 2-D TMA load with an L2 cache hint (the decode reads every KV byte once: evict first).
__device__ __forceinline__ void tma_load_2d_hint(void *dst, const CUtensorMap *map, int x, int y, uint64_t *bar,
                                                 uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_u32(dst)),
      "l"(map), "r"(x), "r"(y), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// D(16x8, fp32) += A(16x16, bf16, row-major) * B(16x8, bf16, column-major); fragments as in the PTX ISA's
// m16n8k16 layout (group = lane / 4, pair = lane % 4).
__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// The same with f16 operands.
__device__ __forceinline__ void mma_16816_f16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                              uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// An 8x8 matrix of 16-bit values held as m16n8k16 C-fragment pairs (lane (g, t): row g, columns 2t, 2t + 1),
// transposed across the warp: lane (g, t) gets row g, columns 2t, 2t + 1 of the transpose.
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t a) {
  uint32_t d;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(d) : "r"(a));
  return d;
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

// Byte offset of 16-byte chunk c (0..D/8-1) of row r in a tile of 128-byte-swizzled 64-element planes.
__device__ __forceinline__ uint32_t sw_chunk(int r, int c) {
  return static_cast<uint32_t>((c >> 3) * (kBlock * 128) + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}

// KT: cache element (0 bf16, 1 FP8 E4M3, 2 INT8).  HI: the CTA serves more than 8 query heads (rows 8-15
// of the products are real).
template <int KT, int D, int NW, int STAGES, bool HI, bool ORDERED>
__global__ void __launch_bounds__(NW * 32)
    paged_decode_mma_kernel(const DecodeParams P, const __grid_constant__ CUtensorMap kmap,
                            const __grid_constant__ CUtensorMap vmap, const __grid_constant__ WorkOrder<ORDERED> W) {
  using C = DecodeMmaCfg<KT, D, NW, STAGES>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int grp = lane >> 2, pr = lane & 3;           // fragment row group and pair index
  const int split = ORDERED ? (W.item[blockIdx.y] >> 16) : static_cast<int>(blockIdx.z);
  const int b = ORDERED ? (W.item[blockIdx.y] & 0xffff) : static_cast<int>(blockIdx.y);
  const int hpc = P.group < 16 ? P.group : 16;        // query heads of this CTA (rows of the products)
  const int sub_groups = P.group / hpc;
  const int g = blockIdx.x / sub_groups;
  const int h0 = g * P.group + (blockIdx.x % sub_groups) * hpc;
  // any input may come from the kernel before this one on the stream (launched with PDL)
  griddep_wait();
  griddep_launch();

  // ---- this warp's first block-table entries, read beside the context length instead of after it (the
  // window's units do not depend on the length; entries past the context are not used or checked)
  const int32_t *trow = P.block_tables + (int64_t)b * P.max_blocks_per_seq;
  const int upb = P.block_size / kBlock;   // 16-token units per block: 1 or 2
  const int blk0 = split * P.split_tokens / kBlock;
  int e0 = 0;
  {
    const int u = blk0 + warp + NW * lane;
    if (u / upb < P.max_blocks_per_seq) e0 = __ldg(trow + u / upb);
  }

  // ---- context length, validated: never read past the table row or the launch bound
  int L = P.context_lens[b];
  {
    const int lim = min(P.max_blocks_per_seq * P.block_size, P.max_context_len);
    if (L < 0 || L > lim) {
      if (threadIdx.x == 0 && split == 0) flag_error(kErrLength);
      L = L < 0 ? 0 : lim;
    }
  }
  const int n_splits = (L + P.split_tokens - 1) / P.split_tokens;
  if (split >= (n_splits > 1 ? n_splits : 1)) return;
  const bool final_out = n_splits <= 1;
  const int t0 = split * P.split_tokens;
  const int t1 = min(L, t0 + P.split_tokens);
  const int nblk = t1 > t0 ? (t1 - t0 + kBlock - 1) / kBlock : 0;

  uint8_t *wbase = smem + warp * C::WARP_BYTES;
  uint64_t *bars = reinterpret_cast<uint64_t *>(wbase + C::DATA);
  const int nwb = nblk > warp ? (nblk - warp + NW - 1) / NW : 0;  // blocks of this warp
  if (lane == 0) {
    for (int s = 0; s < STAGES; ++s) mbar_init(&bars[s], 1);
    fence_mbar_init();
  }
  __syncwarp();

  // ---- block-table window: lane k holds the 16-row tile index of this warp's unit win*32 + k (window 0
  // from the entries read above)
  auto load_window = [&](int win) -> int {
    const int i = win * 32 + lane;
    int tile = 0;
    if (i < nwb) {
      const int u = blk0 + warp + NW * i;
      int e = win == 0 ? e0 : __ldg(trow + u / upb);
      if (e < 0 || e >= P.num_blocks) {
        flag_error(kErrBlockId);
        e = 0;
      }
      tile = (e * P.num_kv_heads + g) * upb + u % upb;
    }
    return tile;
  };
  int tw = load_window(0);
  const uint64_t pol = l2_evict_first_policy();
  auto issue = [&](int i) {  // warp-uniform call
    if (i >= nwb) return;
    if ((i & 31) == 0 && i > 0) tw = load_window(i >> 5);
    const int tile = __shfl_sync(0xffffffffu, tw, i & 31);
    const int s = i % STAGES;
    if (lane == 0) mbar_arrive_expect_tx(&bars[s], 2 * C::TILE);
    __syncwarp();
    if (lane < 2 * C::PLANES) {   // one 16-row x 128-byte box per lane: K planes, then V planes
      const int pl = lane % C::PLANES;
      const bool v = lane >= C::PLANES;
      tma_load_2d_hint(wbase + ((v ? STAGES : 0) + s) * C::TILE + pl * C::PLANE, v ? &vmap : &kmap,
                       pl * (128 / C::E), tile * kBlock, &bars[s], pol);
    }
  };

  int issued = 0;
  for (; issued < STAGES && issued < nwb; ++issued) issue(issued);

  // ---- Q fragments (rows h0 + grp and h0 + grp + 8).  bf16 cache: unscaled bf16; k-step 4t+u of plane t
  // holds dims 64t + 16*pr + 4u + {0,1} (A[0], A[1]) and + {2,3} (A[2], A[3]).  One-byte caches: f16 scaled
  // per row; k-step s holds dims 32*pr + 4s + {0,1} and + {2,3}; qsc_* multiplies the row's scores.
  uint32_t qlo[C::KS][2], qhi[C::KS][2];
  float qsc_lo = P.qscale, qsc_hi = P.qscale;
  if constexpr (KT != 0) {
    const float ks = P.k_scale[g];
    auto load_row = [&](int row, uint32_t (&qf)[C::KS][2], float &qsc) {
      float v[32];
      if (row < hpc) {
        const uint4 *src =
            reinterpret_cast<const uint4 *>(P.q + ((int64_t)b * P.num_q_heads + h0 + row) * D + 32 * pr);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const uint4 w = src[c];
          const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            v[8 * c + 2 * t] = bf16lo(ww[t]);
            v[8 * c + 2 * t + 1] = bf16hi(ww[t]);
          }
        }
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] = 0.f;
      }
      float amax = 0.f;
#pragma unroll
      for (int e = 0; e < 32; ++e) amax = fmaxf(amax, fabsf(v[e]));
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
      // the row's largest |q| has binary exponent ex; q * 2^-ex lies within (-2, 2)
      int ex = amax > 0.f ? static_cast<int>((__float_as_uint(amax) >> 23) & 0xff) - 127 : 0;
      ex = ex < -126 ? -126 : (ex > 126 ? 126 : ex);
      const float down = __uint_as_float(static_cast<uint32_t>(127 - ex) << 23);
      qsc = __uint_as_float(static_cast<uint32_t>(127 + ex) << 23) * (P.qscale * ks);
#pragma unroll
      for (int s2 = 0; s2 < C::KS; ++s2) {
        qf[s2][0] = pack_f16x2(v[4 * s2] * down, v[4 * s2 + 1] * down);
        qf[s2][1] = pack_f16x2(v[4 * s2 + 2] * down, v[4 * s2 + 3] * down);
      }
    };
    load_row(grp, qlo, qsc_lo);
    if constexpr (HI) {
      load_row(grp + 8, qhi, qsc_hi);
    } else {
      // transposed products: this lane's score columns are queries 2pr and 2pr + 1
      const float s0 = __shfl_sync(0xffffffffu, qsc_lo, 8 * pr), s1 = __shfl_sync(0xffffffffu, qsc_lo, 8 * pr + 4);
      qsc_lo = s0;
      qsc_hi = s1;
    }
  } else {
#pragma unroll
  for (int t = 0; t < C::PLANES; ++t) {
    uint4 w[2] = {make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0)};
    if (grp < hpc) {
      const uint4 *src = reinterpret_cast<const uint4 *>(P.q + ((int64_t)b * P.num_q_heads + h0 + grp) * D +
                                                          64 * t + 16 * pr);
      w[0] = src[0];
      w[1] = src[1];
    }
    const uint32_t ww[8] = {w[0].x, w[0].y, w[0].z, w[0].w, w[1].x, w[1].y, w[1].z, w[1].w};
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      qlo[4 * t + u][0] = ww[2 * u];
      qlo[4 * t + u][1] = ww[2 * u + 1];
    }
    if constexpr (HI) {
      uint4 x[2] = {make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0)};
      if (grp + 8 < hpc) {
        const uint4 *src = reinterpret_cast<const uint4 *>(P.q + ((int64_t)b * P.num_q_heads + h0 + grp + 8) * D +
                                                            64 * t + 16 * pr);
        x[0] = src[0];
        x[1] = src[1];
      }
      const uint32_t xx[8] = {x[0].x, x[0].y, x[0].z, x[0].w, x[1].x, x[1].y, x[1].z, x[1].w};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        qhi[4 * t + u][0] = xx[2 * u];
        qhi[4 * t + u][1] = xx[2 * u + 1];
      }
    }
  }
  }

  // ---- running state per row: reference max (log2 units), this lane's share of the sum, O fragments
  constexpr float kRescale = 8.f;
  float m_lo = -INFINITY, m_hi = -INFINITY, l_lo = 0.f, l_hi = 0.f;
  float o[C::NT][4];
#pragma unroll
  for (int j = 0; j < C::NT; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;

  const uint32_t wbase_s = smem_u32(wbase);
  bool ok = true;
  int i = 0;
  for (; i < nwb; ++i) {
    const int s = i % STAGES;
    const bool got = mbar_wait(&bars[s], (i / STAGES) & 1);
    if (__any_sync(0xffffffffu, !got)) {
      ok = false;
      break;
    }
    const int jb = warp + NW * i;                       // block index within the split
    const int nvalid = min(kBlock, t1 - (t0 + jb * kBlock));
    const uint32_t Kt = wbase_s + s * C::TILE;
    const uint32_t Vt = wbase_s + (STAGES + s) * C::TILE;
    if (nvalid < kBlock) {
      // V rows past the context are zeroed: P is 0 there, but 0 * (whatever the cache holds) may not be
      uint8_t *vt = wbase + (STAGES + s) * C::TILE;
      constexpr int CPR = C::ROWB / 16;   // 16-byte chunks per row
      for (int idx = lane; idx < (kBlock - nvalid) * CPR; idx += 32) {
        const int r = nvalid + idx / CPR, c = idx % CPR;
        *reinterpret_cast<uint4 *>(vt + sw_chunk(r, c)) = make_uint4(0, 0, 0, 0);
      }
      fence_async_smem();   // before the TMA writes this slot again
      __syncwarp();
    }

    if constexpr (KT != 0 && !HI) {
      // ---- one-byte caches, up to 8 query heads: the products are transposed so that the block's 16
      // tokens fill the M side of m16n8k16 and the (at most 8) query heads its N side, which halves the
      // products per block.  S^T = K Q^T: the A fragments are K's converted codes (lane (grp, pr): tokens
      // grp and grp + 8, bytes [32pr, 32pr + 32) of their rows; k-step s takes dims 32pr + 4s + {0,1} and
      // {2,3}, the dims Q's fragments use), the B fragments Q's rows.  Lane (grp, pr) then holds the scores
      // of tokens grp, grp + 8 for queries 2pr, 2pr + 1.
      float sc[4];
      {
        float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        const uint4 k0 = lds128(Kt + sw_chunk(grp, 2 * pr));
        const uint4 k1 = lds128(Kt + sw_chunk(grp, 2 * pr + 1));
        const uint4 k2 = lds128(Kt + sw_chunk(grp + 8, 2 * pr));
        const uint4 k3 = lds128(Kt + sw_chunk(grp + 8, 2 * pr + 1));
        const uint32_t klo[8] = {k0.x, k0.y, k0.z, k0.w, k1.x, k1.y, k1.z, k1.w};
        const uint32_t khi[8] = {k2.x, k2.y, k2.z, k2.w, k3.x, k3.y, k3.z, k3.w};
#pragma unroll
        for (int s2 = 0; s2 < C::KS; ++s2) {
          uint32_t a0, a1, a2, a3;
          bytes4_to_h2<KT>(klo[s2], a0, a2);
          bytes4_to_h2<KT>(khi[s2], a1, a3);
          mma_16816_f16(acc[s2 & 1], a0, a1, a2, a3, qlo[s2][0], qlo[s2][1]);
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) sc[e] = acc[0][e] + acc[1][e];
      }
      // -- online softmax per query column: a column's 16 scores sit with the 8 lanes of one pr
      float x[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int tok = grp + ((e & 2) ? 8 : 0);
        x[e] = tok < nvalid ? sc[e] * ((e & 1) ? qsc_hi : qsc_lo) : -INFINITY;
      }
      float bm0 = fmaxf(x[0], x[2]), bm1 = fmaxf(x[1], x[3]);
#pragma unroll
      for (int off = 4; off <= 16; off <<= 1) {
        bm0 = fmaxf(bm0, __shfl_xor_sync(0xffffffffu, bm0, off));
        bm1 = fmaxf(bm1, __shfl_xor_sync(0xffffffffu, bm1, off));
      }
      // the reference of a column moves only when the block's max exceeds it by more than 2^8 (or on the
      // first block); O and l are rescaled with it, so O / l is exact whichever reference is used
      if (bm0 > m_lo + kRescale) {
        const float alpha = m_lo == -INFINITY ? 0.f : exp2f(m_lo - bm0);
        m_lo = bm0;
        l_lo *= alpha;
#pragma unroll
        for (int j = 0; j < C::NT / 2; ++j) {
          o[j][0] *= alpha;
          o[j][2] *= alpha;
        }
      }
      if (bm1 > m_hi + kRescale) {
        const float alpha = m_hi == -INFINITY ? 0.f : exp2f(m_hi - bm1);
        m_hi = bm1;
        l_hi *= alpha;
#pragma unroll
        for (int j = 0; j < C::NT / 2; ++j) {
          o[j][1] *= alpha;
          o[j][3] *= alpha;
        }
      }
      const float p0 = exp2f(x[0] - m_lo), p1 = exp2f(x[1] - m_hi), p2 = exp2f(x[2] - m_lo),
                  p3 = exp2f(x[3] - m_hi);
      l_lo += p0 + p2;
      l_hi += p1 + p3;
      // P^T as the B operand of O^T += V^T P^T: the C layout of tokens 0-7 (and 8-15) x queries, transposed
      // across the warp by movmatrix, is the B fragment (tokens 2pr, 2pr + 1 (+ 8) of query grp)
      const uint32_t pb0 = movmatrix_trans(pack_f16x2(p0, p1));
      const uint32_t pb1 = movmatrix_trans(pack_f16x2(p2, p3));
      __syncwarp();
      // -- O^T += V^T P^T: m-tile j holds dims 16grp + 2j (rows grp) and 16grp + 2j + 1 (rows grp + 8).  Lane
      // (grp, pr) reads dims [16grp, 16grp + 16) of token rows 2pr, 2pr + 1 and 2pr + 8, 2pr + 9; a byte
      // permute pairs two rows' codes of one dim, which is an A fragment register
      {
        const uint4 r0 = lds128(Vt + sw_chunk(2 * pr, grp));
        const uint4 r1 = lds128(Vt + sw_chunk(2 * pr + 1, grp));
        const uint4 r2 = lds128(Vt + sw_chunk(2 * pr + 8, grp));
        const uint4 r3 = lds128(Vt + sw_chunk(2 * pr + 9, grp));
        const uint32_t va[4] = {r0.x, r0.y, r0.z, r0.w}, vc[4] = {r1.x, r1.y, r1.z, r1.w};
        const uint32_t vd[4] = {r2.x, r2.y, r2.z, r2.w}, vf[4] = {r3.x, r3.y, r3.z, r3.w};
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          uint32_t a0, a1, a2, a3;
          bytes4_to_h2<KT>(__byte_perm(va[q4], vc[q4], 0x5140), a0, a1);   // dims 4q4, 4q4 + 1
          bytes4_to_h2<KT>(__byte_perm(vd[q4], vf[q4], 0x5140), a2, a3);
          mma_16816_f16(o[2 * q4], a0, a1, a2, a3, pb0, pb1);
          bytes4_to_h2<KT>(__byte_perm(va[q4], vc[q4], 0x7362), a0, a1);   // dims 4q4 + 2, 4q4 + 3
          bytes4_to_h2<KT>(__byte_perm(vd[q4], vf[q4], 0x7362), a2, a3);
          mma_16816_f16(o[2 * q4 + 1], a0, a1, a2, a3, pb0, pb1);
        }
      }
    } else {
      // -- S = Q K^T: n-tile nt holds tokens 8nt..8nt+7; lane (grp, pr) reads token 8nt+grp's dims
      // 64t + 16pr .. +16 (two 16-byte chunks of plane t)
      // (two accumulators per n-tile, even and odd k-steps, so that the dependent chain of products on one
      // accumulator is half as long)
      float sc[2][4];
  #pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        const int R = 8 * nt + grp;
        if constexpr (KT == 0) {
  #pragma unroll
          for (int t = 0; t < C::PLANES; ++t) {
            const uint4 k0 = lds128(Kt + sw_chunk(R, 8 * t + 2 * pr));
            const uint4 k1 = lds128(Kt + sw_chunk(R, 8 * t + 2 * pr + 1));
            const uint32_t kw[8] = {k0.x, k0.y, k0.z, k0.w, k1.x, k1.y, k1.z, k1.w};
  #pragma unroll
            for (int u = 0; u < 4; ++u) {
              const int ks = 4 * t + u;
              mma_16816(acc[ks & 1], qlo[ks][0], HI ? qhi[ks][0] : 0u, qlo[ks][1], HI ? qhi[ks][1] : 0u, kw[2 * u],
                        kw[2 * u + 1]);
            }
          }
        } else {
          // the row's bytes [32pr, 32pr + 32): 16 f16 pairs, k-step s takes pairs 2s and 2s + 1
          const uint4 k0 = lds128(Kt + sw_chunk(R, 2 * pr));
          const uint4 k1 = lds128(Kt + sw_chunk(R, 2 * pr + 1));
          const uint32_t kw[8] = {k0.x, k0.y, k0.z, k0.w, k1.x, k1.y, k1.z, k1.w};
  #pragma unroll
          for (int s2 = 0; s2 < C::KS; ++s2) {
            uint32_t b0, b1;
            bytes4_to_h2<KT>(kw[s2], b0, b1);
            mma_16816_f16(acc[s2 & 1], qlo[s2][0], HI ? qhi[s2][0] : 0u, qlo[s2][1], HI ? qhi[s2][1] : 0u, b0, b1);
          }
        }
  #pragma unroll
        for (int e = 0; e < 4; ++e) sc[nt][e] = acc[0][e] + acc[1][e];
      }

      // -- online softmax: lane (grp, pr) holds row grp's tokens 8nt + 2pr + {0,1} (sc[nt][0..1]) and row
      // grp+8's (sc[nt][2..3]); a row's max comes from the 4 lanes of its quad
      float x[2][4];
  #pragma unroll
      for (int nt = 0; nt < 2; ++nt)
  #pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int tok = 8 * nt + 2 * pr + (e & 1);
          x[nt][e] = tok < nvalid ? sc[nt][e] * (e < 2 ? qsc_lo : qsc_hi) : -INFINITY;
        }
      float bm_lo = fmaxf(fmaxf(x[0][0], x[0][1]), fmaxf(x[1][0], x[1][1]));
      bm_lo = fmaxf(bm_lo, __shfl_xor_sync(0xffffffffu, bm_lo, 1));
      bm_lo = fmaxf(bm_lo, __shfl_xor_sync(0xffffffffu, bm_lo, 2));
      // the reference moves only when the block's max exceeds it by more than 2^8 (or on the first block);
      // O and l are rescaled with it, so O / l is exact whichever reference is used
      if (bm_lo > m_lo + kRescale) {
        const float alpha = m_lo == -INFINITY ? 0.f : exp2f(m_lo - bm_lo);
        m_lo = bm_lo;
        l_lo *= alpha;
  #pragma unroll
        for (int j = 0; j < C::NT; ++j) {
          o[j][0] *= alpha;
          o[j][1] *= alpha;
        }
      }
      float p[2][4];
  #pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        p[nt][0] = exp2f(x[nt][0] - m_lo);
        p[nt][1] = exp2f(x[nt][1] - m_lo);
        l_lo += p[nt][0] + p[nt][1];
      }
      if constexpr (HI) {
        float bm_hi = fmaxf(fmaxf(x[0][2], x[0][3]), fmaxf(x[1][2], x[1][3]));
        bm_hi = fmaxf(bm_hi, __shfl_xor_sync(0xffffffffu, bm_hi, 1));
        bm_hi = fmaxf(bm_hi, __shfl_xor_sync(0xffffffffu, bm_hi, 2));
        if (bm_hi > m_hi + kRescale) {
          const float alpha = m_hi == -INFINITY ? 0.f : exp2f(m_hi - bm_hi);
          m_hi = bm_hi;
          l_hi *= alpha;
  #pragma unroll
          for (int j = 0; j < C::NT; ++j) {
            o[j][2] *= alpha;
            o[j][3] *= alpha;
          }
        }
  #pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          p[nt][2] = exp2f(x[nt][2] - m_hi);
          p[nt][3] = exp2f(x[nt][3] - m_hi);
          l_hi += p[nt][2] + p[nt][3];
        }
      }
      // P as the A operand of the PV product (K = the block's 16 tokens): its fragments are S's
      if constexpr (KT == 0) {
        const uint32_t pa0 = pack_bf16x2(p[0][0], p[0][1]);
        const uint32_t pa2 = pack_bf16x2(p[1][0], p[1][1]);
        const uint32_t pa1 = HI ? pack_bf16x2(p[0][2], p[0][3]) : 0u;
        const uint32_t pa3 = HI ? pack_bf16x2(p[1][2], p[1][3]) : 0u;
        __syncwarp();

        // -- O += P V: ldmatrix.trans gives the B fragments of two 8-dim n-tiles per call; lane l addresses
        // row (l/8 % 2)*8 + l%8 (token) of 8-dim chunk 2jj + l/16
        const int vr = ((lane >> 3) & 1) * 8 + (lane & 7);
  #pragma unroll
        for (int jj = 0; jj < C::NT / 2; ++jj) {
          uint32_t v0, v1, v2, v3;
          ldsm_x4_trans(Vt + sw_chunk(vr, 2 * jj + (lane >> 4)), v0, v1, v2, v3);
          mma_16816(o[2 * jj], pa0, pa1, pa2, pa3, v0, v1);
          mma_16816(o[2 * jj + 1], pa0, pa1, pa2, pa3, v2, v3);
        }
      } else {
        // P in f16 (p <= 2^8)
        const uint32_t pa0 = pack_f16x2(p[0][0], p[0][1]);
        const uint32_t pa2 = pack_f16x2(p[1][0], p[1][1]);
        const uint32_t pa1 = HI ? pack_f16x2(p[0][2], p[0][3]) : 0u;
        const uint32_t pa3 = HI ? pack_f16x2(p[1][2], p[1][3]) : 0u;
        __syncwarp();
        // -- O += P V: lane (grp, pr) converts V row (8h + grp)'s bytes [32pr, 32pr + 32) into 16 pairs of
        // adjacent dims; pair j, transposed across the warp, is the B fragment of n-tile j (dims
        // {32p' + 2j, +1}) for the 8 tokens of half h
        // lane (grp, pr) reads dims [16grp, 16grp + 16) of token rows 2pr, 2pr + 1 (half h = 0) and 8 + 2pr,
        // 9 + 2pr (h = 1); a byte permute pairs the two rows' codes of one dim, which is the B fragment of
        // n-tile e (column grp = dim 16grp + e) for tokens (2pr, 2pr + 1) + 8h
        uint32_t vb[2][16];
  #pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint4 r0 = lds128(Vt + sw_chunk(8 * h + 2 * pr, grp));
          const uint4 r1 = lds128(Vt + sw_chunk(8 * h + 2 * pr + 1, grp));
          const uint32_t a[4] = {r0.x, r0.y, r0.z, r0.w}, c[4] = {r1.x, r1.y, r1.z, r1.w};
  #pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            bytes4_to_h2<KT>(__byte_perm(a[q4], c[q4], 0x5140), vb[h][4 * q4], vb[h][4 * q4 + 1]);
            bytes4_to_h2<KT>(__byte_perm(a[q4], c[q4], 0x7362), vb[h][4 * q4 + 2], vb[h][4 * q4 + 3]);
          }
        }
  #pragma unroll
        for (int e = 0; e < C::NT; ++e) mma_16816_f16(o[e], pa0, pa1, pa2, pa3, vb[0][e], vb[1][e]);
      }
    }
    __syncwarp();
    if (issued < nwb) issue(issued++);
  }
  if (!ok) {
    // a wait gave up: give the copies this warp still has in flight a bounded chance to land, then drop
    // this warp's state (the error word already says why)
    for (int k = i; k < issued; ++k) (void)mbar_wait(&bars[k % STAGES], (k / STAGES) & 1);
    m_lo = m_hi = -INFINITY;
    l_lo = l_hi = 0.f;
#pragma unroll
    for (int j = 0; j < C::NT; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
  }
  constexpr bool kTr = KT != 0 && !HI;               // transposed products (one-byte, up to 8 heads)
  if constexpr (kTr) {
    // a column's sum is spread over the 8 lanes of one pr
#pragma unroll
    for (int off = 4; off <= 16; off <<= 1) {
      l_lo += __shfl_xor_sync(0xffffffffu, l_lo, off);
      l_hi += __shfl_xor_sync(0xffffffffu, l_hi, off);
    }
  } else {
    l_lo += __shfl_xor_sync(0xffffffffu, l_lo, 1);
    l_lo += __shfl_xor_sync(0xffffffffu, l_lo, 2);
    if constexpr (HI) {
      l_hi += __shfl_xor_sync(0xffffffffu, l_hi, 1);
      l_hi += __shfl_xor_sync(0xffffffffu, l_hi, 2);
    }
  }

  // ---- merge the warps: each writes its rows' (O, m, l) over its consumed tiles, then the CTA combines
  __syncwarp();
  float *mrg = reinterpret_cast<float *>(wbase);
  if constexpr (kTr) {
    // m-tile j of this lane: queries 2pr, 2pr + 1 at dims 16grp + 2j (o[j][0..1]) and + 1 (o[j][2..3])
#pragma unroll
    for (int j = 0; j < C::NT / 2; ++j) {
      const int d0 = 16 * grp + 2 * j;
      *reinterpret_cast<float2 *>(mrg + (2 * pr) * D + d0) = make_float2(o[j][0], o[j][2]);
      *reinterpret_cast<float2 *>(mrg + (2 * pr + 1) * D + d0) = make_float2(o[j][1], o[j][3]);
    }
    if (grp == 0) {
      mrg[C::ML + 2 * (2 * pr)] = m_lo;
      mrg[C::ML + 2 * (2 * pr) + 1] = l_lo;
      mrg[C::ML + 2 * (2 * pr + 1)] = m_hi;
      mrg[C::ML + 2 * (2 * pr + 1) + 1] = l_hi;
    }
  } else {
#pragma unroll
  for (int j = 0; j < C::NT; ++j) {
    if constexpr (KT == 0) {
      // n-tile j of this lane holds dims 8j + 2pr, +1
      *reinterpret_cast<float2 *>(mrg + grp * D + 8 * j + 2 * pr) = make_float2(o[j][0], o[j][1]);
      if constexpr (HI)
        *reinterpret_cast<float2 *>(mrg + (grp + 8) * D + 8 * j + 2 * pr) = make_float2(o[j][2], o[j][3]);
    } else {
      // one-byte caches: n-tile j of this lane holds dims 32pr + j and 32pr + 16 + j
      mrg[grp * D + 32 * pr + j] = o[j][0];
      mrg[grp * D + 32 * pr + 16 + j] = o[j][1];
      if constexpr (HI) {
        mrg[(grp + 8) * D + 32 * pr + j] = o[j][2];
        mrg[(grp + 8) * D + 32 * pr + 16 + j] = o[j][3];
      }
    }
  }
  if (pr == 0) {
    mrg[C::ML + 2 * grp] = m_lo;
    mrg[C::ML + 2 * grp + 1] = l_lo;
    if constexpr (HI) {
      mrg[C::ML + 2 * (grp + 8)] = m_hi;
      mrg[C::ML + 2 * (grp + 8) + 1] = l_hi;
    }
  }
  }
  __syncthreads();

  const float vs = KT != 0 ? P.v_scale[g] : 1.f;
  for (int idx = threadIdx.x; idx < hpc * D; idx += NW * 32) {
    const int qi = idx / D, d = idx % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w) M = fmaxf(M, reinterpret_cast<const float *>(smem + w * C::WARP_BYTES)[C::ML + 2 * qi]);
    float Lsum = 0.f, O = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < NW; ++w) {
        const float *mw = reinterpret_cast<const float *>(smem + w * C::WARP_BYTES);
        const float sc_w = exp2f(mw[C::ML + 2 * qi] - M);
        Lsum += sc_w * mw[C::ML + 2 * qi + 1];
        O += sc_w * mw[qi * D + d];
      }
    }
    const int h = h0 + qi;
    if (final_out) {
      const float val = Lsum > 0.f ? O / Lsum * vs : 0.f;
      P.out[((int64_t)b * P.num_q_heads + h) * D + d] = __float2bfloat16_rn(val);
    } else {
      const int64_t row = ((int64_t)b * P.num_q_heads + h) * P.max_splits + split;
      P.ws_o[row * D + d] = O * vs;
      if (d == 0) {
        P.ws_ml[row * 2] = M;
        P.ws_ml[row * 2 + 1] = Lsum;
      }
    }
  }
}

}  // namespace pa
