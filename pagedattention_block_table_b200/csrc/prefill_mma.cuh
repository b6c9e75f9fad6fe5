// prefill_mma.cuh -- paged causal prefill over a one-byte cache (FP8 E4M3 or INT8, head_dim 128), on the
// warp-level tensor cores (sm_100a).
//
// What it computes is the prefill of prefill.cuh (vLLM overview page, "Continuous Batching"; Core Concepts
// page §3.2): for chunk c with history H_c and C_c new tokens, query row i (position H_c + i) of head h
// attends to positions t <= H_c + i of KV head h / G, reading K[t] = code * k_scale and V[t] = code *
// v_scale through the block table (KV Cache to vLLM page §2.2: one-byte KV with a scale per KV head).
//
// Design.  The products run in f16 (mma.sync m16n8k16, f32 accumulate) as in the one-byte path of the
// tensor-core decode (decode_mma.cuh): codes are exact in f16, Q is scaled per row by a power of two into
// [1, 2) before it is rounded to f16, that power with the softmax and K scales multiplies the scores and
// the V scale the output.  A CTA serves 64 query rows of one KV head -- rows stack the heads of the group
// that share the KV head (row r = position r / hpr, head r % hpr) -- as four warps of 16 rows, and walks
// the keys its rows can see in 16-token units.  One lane issues the 2-D TMA loads of each unit's K and V
// tiles (16 rows x 128 bytes, 128-byte swizzle, into this CTA's own shared memory) STAGES units ahead;
// all four warps consume every unit and release it on an mbarrier.  Per warp and unit: S = Q K^T (2
// n-tiles of 8 keys x 8 k-steps), the causal mask per row, a base-2 online softmax on S's fragments
// (reference max moved only past 2^8), O += P V (16 n-tiles).  V codes of keys past the context are
// replaced by zero in registers before the product, since 0 * a stale code that decodes to NaN is NaN.
#pragma once
#include "decode_mma.cuh"

namespace pa {

struct PrefillMmaParams {
  __nv_bfloat16 *out;
  const __nv_bfloat16 *q;
  const int32_t *cu_q_lens;
  const int32_t *block_tables;
  const int32_t *context_lens;
  const float *k_scale;
  const float *v_scale;
  int64_t num_blocks;
  int block_size;       // 16 or 32 tokens per physical block
  int max_blocks_per_seq;
  int num_q_heads;
  int num_kv_heads;
  int group;            // Hq / Hkv
  int hpr;              // query heads stacked per position in a row tile (G if 64 % G == 0, else 1)
  int max_context_len;
  float qscale;         // scale * log2(e)
};

template <int NW, int STAGES>
struct PrefillMmaCfg {
  static constexpr int D = 128;
  static constexpr int ROWS = 16 * NW;                 // query rows of a CTA
  static constexpr int TILE = kBlock * 128;            // one 16-token K or V tile: 2 KB
  static constexpr int OFF_BAR = 2 * STAGES * TILE;
  static constexpr int SMEM = OFF_BAR + 2 * STAGES * 8 + 1024;   // + slack to align the base
};

template <int KT, int NW, int STAGES>
__global__ void __launch_bounds__(NW * 32)
    paged_prefill_mma_kernel(const PrefillMmaParams P, const __grid_constant__ CUtensorMap kmap,
                             const __grid_constant__ CUtensorMap vmap) {
  using C = PrefillMmaCfg<NW, STAGES>;
  constexpr int D = C::D;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int grp = lane >> 2, pr = lane & 3;
  const int hg0 = blockIdx.x * P.hpr;                  // first query head of this CTA's rows
  const int g = hg0 / P.group;                         // their KV head
  const int ppt = C::ROWS / P.hpr;                     // positions per row tile
  const int c = blockIdx.z;
  griddep_wait();
  griddep_launch();

  const int q0 = P.cu_q_lens[c];
  const int Cn = P.cu_q_lens[c + 1] - q0;
  const int ctx = P.context_lens[c];
  const int H = ctx - Cn;
  if (Cn < 0 || H < 0 || ctx > min(P.max_blocks_per_seq * P.block_size, P.max_context_len)) {
    if (threadIdx.x == 0 && blockIdx.x == 0 && blockIdx.y == 0) flag_error(kErrLength);
    return;
  }
  const int ntile = (Cn + ppt - 1) / ppt;              // row tiles of this chunk
  if (ntile > static_cast<int>(gridDim.y)) {           // chunk longer than the max_q_len launched for
    if (threadIdx.x == 0 && blockIdx.x == 0 && blockIdx.y == 0) flag_error(kErrLength);
    return;
  }
  if (static_cast<int>(blockIdx.y) >= ntile) return;
  const int p0 = (ntile - 1 - static_cast<int>(blockIdx.y)) * ppt;   // longest rows first
  const int kv_len = H + min(Cn, p0 + ppt);            // keys some row of this CTA sees
  const int nunits = (kv_len + kBlock - 1) / kBlock;

  uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);
  uint64_t *empty = full + STAGES;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], NW);
    }
    fence_mbar_init();
  }
  __syncthreads();

  // ---- producer (warp 0, lane 0): the K and V tiles of unit u into stage u % STAGES
  const int32_t *trow = P.block_tables + (int64_t)c * P.max_blocks_per_seq;
  const int upb = P.block_size / kBlock;
  const uint64_t pol = l2_evict_first_policy();
  auto issue = [&](int u) {
    const int s = u % STAGES;
    int e = __ldg(trow + u / upb);
    if (e < 0 || e >= P.num_blocks) {
      flag_error(kErrBlockId);
      e = 0;
    }
    const int tile = (e * P.num_kv_heads + g) * upb + u % upb;
    mbar_arrive_expect_tx(&full[s], 2 * C::TILE);
    tma_load_2d_hint(smem + s * C::TILE, &kmap, 0, tile * kBlock, &full[s], pol);
    tma_load_2d_hint(smem + (STAGES + s) * C::TILE, &vmap, 0, tile * kBlock, &full[s], pol);
  };
  const bool producer = warp == 0 && lane == 0;
  int issued = 0;
  if (producer)
    for (; issued < STAGES && issued < nunits; ++issued) issue(issued);

  // ---- this warp's two fragment rows: lo = warp*16 + grp, hi = lo + 8
  const int r_lo = warp * 16 + grp, r_hi = r_lo + 8;
  const int pi_lo = p0 + r_lo / P.hpr, pi_hi = p0 + r_hi / P.hpr;
  const int h_lo = hg0 + r_lo % P.hpr, h_hi = hg0 + r_hi % P.hpr;
  const bool ok_lo = pi_lo < Cn, ok_hi = pi_hi < Cn;
  const int pos_lo = ok_lo ? H + pi_lo : kv_len - 1;   // padding rows behave like the last row
  const int pos_hi = ok_hi ? H + pi_hi : kv_len - 1;

  // Q rows in f16, scaled per row by a power of two; k-step s holds dims 32pr + 4s + {0,1} and + {2,3}
  const float ks = P.k_scale[g];
  uint32_t qlo[8][2], qhi[8][2];
  float qsc_lo, qsc_hi;
  auto load_row = [&](bool ok, int pi, int h, uint32_t (&qf)[8][2], float &qsc) {
    float v[32];
    if (ok) {
      const uint4 *src = reinterpret_cast<const uint4 *>(P.q + ((int64_t)(q0 + pi) * P.num_q_heads + h) * D + 32 * pr);
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        const uint4 w = src[cc];
        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          v[8 * cc + 2 * t] = bf16lo(ww[t]);
          v[8 * cc + 2 * t + 1] = bf16hi(ww[t]);
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
    int ex = amax > 0.f ? static_cast<int>((__float_as_uint(amax) >> 23) & 0xff) - 127 : 0;
    ex = ex < -126 ? -126 : (ex > 126 ? 126 : ex);
    const float down = __uint_as_float(static_cast<uint32_t>(127 - ex) << 23);
    qsc = __uint_as_float(static_cast<uint32_t>(127 + ex) << 23) * (P.qscale * ks);
#pragma unroll
    for (int s2 = 0; s2 < 8; ++s2) {
      qf[s2][0] = pack_f16x2(v[4 * s2] * down, v[4 * s2 + 1] * down);
      qf[s2][1] = pack_f16x2(v[4 * s2 + 2] * down, v[4 * s2 + 3] * down);
    }
  };
  load_row(ok_lo, pi_lo, h_lo, qlo, qsc_lo);
  load_row(ok_hi, pi_hi, h_hi, qhi, qsc_hi);

  constexpr float kRescale = 8.f;
  float m_lo = -INFINITY, m_hi = -INFINITY, l_lo = 0.f, l_hi = 0.f;
  float o[16][4];
#pragma unroll
  for (int j = 0; j < 16; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;

  const uint32_t sbase = smem_u32(smem);
  bool ok = true;
  int u = 0;
  for (; u < nunits; ++u) {
    const int s = u % STAGES;
    const bool got = mbar_wait(&full[s], (u / STAGES) & 1);
    if (__any_sync(0xffffffffu, !got)) {
      ok = false;
      break;
    }
    const uint32_t Kt = sbase + s * C::TILE, Vt = sbase + (STAGES + s) * C::TILE;
    const int kb = u * kBlock;

    // -- S = Q K^T on two accumulators per n-tile (even and odd k-steps)
    float sc[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
      const int R = 8 * nt + grp;
      const uint4 k0 = lds128(Kt + sw_chunk(R, 2 * pr));
      const uint4 k1 = lds128(Kt + sw_chunk(R, 2 * pr + 1));
      const uint32_t kw[8] = {k0.x, k0.y, k0.z, k0.w, k1.x, k1.y, k1.z, k1.w};
#pragma unroll
      for (int s2 = 0; s2 < 8; ++s2) {
        uint32_t b0, b1;
        bytes4_to_h2<KT>(kw[s2], b0, b1);
        mma_16816_f16(acc[s2 & 1], qlo[s2][0], qhi[s2][0], qlo[s2][1], qhi[s2][1], b0, b1);
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) sc[nt][e] = acc[0][e] + acc[1][e];
    }

    // -- causal online softmax: lane holds rows lo (e = 0, 1) and hi (e = 2, 3), keys kb + 8nt + 2pr + (e & 1)
    float x[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int t = kb + 8 * nt + 2 * pr + (e & 1);
        const int pos = e < 2 ? pos_lo : pos_hi;
        x[nt][e] = t <= pos ? sc[nt][e] * (e < 2 ? qsc_lo : qsc_hi) : -INFINITY;
      }
    float bm_lo = fmaxf(fmaxf(x[0][0], x[0][1]), fmaxf(x[1][0], x[1][1]));
    float bm_hi = fmaxf(fmaxf(x[0][2], x[0][3]), fmaxf(x[1][2], x[1][3]));
    bm_lo = fmaxf(bm_lo, __shfl_xor_sync(0xffffffffu, bm_lo, 1));
    bm_hi = fmaxf(bm_hi, __shfl_xor_sync(0xffffffffu, bm_hi, 1));
    bm_lo = fmaxf(bm_lo, __shfl_xor_sync(0xffffffffu, bm_lo, 2));
    bm_hi = fmaxf(bm_hi, __shfl_xor_sync(0xffffffffu, bm_hi, 2));
    // a row may see no key of this unit (bm = -inf): it keeps its reference
    if (bm_lo > m_lo + kRescale) {
      const float alpha = m_lo == -INFINITY ? 0.f : exp2f(m_lo - bm_lo);
      m_lo = bm_lo;
      l_lo *= alpha;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        o[j][0] *= alpha;
        o[j][1] *= alpha;
      }
    }
    if (bm_hi > m_hi + kRescale) {
      const float alpha = m_hi == -INFINITY ? 0.f : exp2f(m_hi - bm_hi);
      m_hi = bm_hi;
      l_hi *= alpha;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        o[j][2] *= alpha;
        o[j][3] *= alpha;
      }
    }
    float p[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      p[nt][0] = exp2f(x[nt][0] - m_lo);
      p[nt][1] = exp2f(x[nt][1] - m_lo);
      p[nt][2] = exp2f(x[nt][2] - m_hi);
      p[nt][3] = exp2f(x[nt][3] - m_hi);
      l_lo += p[nt][0] + p[nt][1];
      l_hi += p[nt][2] + p[nt][3];
    }
    const uint32_t pa0 = pack_f16x2(p[0][0], p[0][1]), pa1 = pack_f16x2(p[0][2], p[0][3]);
    const uint32_t pa2 = pack_f16x2(p[1][0], p[1][1]), pa3 = pack_f16x2(p[1][2], p[1][3]);
    __syncwarp();

    // -- O += P V: lane (grp, pr) pairs the codes of dims [16grp, 16grp + 16) of key rows 2pr, 2pr + 1
    // (h = 0) and 8 + 2pr, 9 + 2pr (h = 1); codes of keys past the context become 0 first
    uint32_t vb[2][16];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int ra = 8 * h + 2 * pr;
      uint4 r0 = lds128(Vt + sw_chunk(ra, grp));
      uint4 r1 = lds128(Vt + sw_chunk(ra + 1, grp));
      if (kb + kBlock > kv_len) {
        if (kb + ra >= kv_len) r0 = make_uint4(0, 0, 0, 0);
        if (kb + ra + 1 >= kv_len) r1 = make_uint4(0, 0, 0, 0);
      }
      const uint32_t a[4] = {r0.x, r0.y, r0.z, r0.w}, b[4] = {r1.x, r1.y, r1.z, r1.w};
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        bytes4_to_h2<KT>(__byte_perm(a[q4], b[q4], 0x5140), vb[h][4 * q4], vb[h][4 * q4 + 1]);
        bytes4_to_h2<KT>(__byte_perm(a[q4], b[q4], 0x7362), vb[h][4 * q4 + 2], vb[h][4 * q4 + 3]);
      }
    }
#pragma unroll
    for (int e = 0; e < 16; ++e) mma_16816_f16(o[e], pa0, pa1, pa2, pa3, vb[0][e], vb[1][e]);
    __syncwarp();
    // release the unit; the producer refills its stage once every warp has
    if (lane == 0) mbar_arrive(&empty[s]);
    if (producer && issued < nunits) {
      const int sn = issued % STAGES;
      if (!mbar_wait(&empty[sn], ((issued / STAGES) - 1) & 1)) {
        ok = false;
      } else {
        issue(issued);
        ++issued;
      }
    }
    if (!__all_sync(0xffffffffu, ok)) {
      ok = false;
      break;
    }
  }
  if (!ok) {
    // a wait gave up: let the copies this CTA has in flight land (bounded), write nothing
    if (producer)
      for (int k = u; k < issued; ++k) (void)mbar_wait(&full[k % STAGES], (k / STAGES) & 1);
    return;
  }

  // ---- out = O / l * v_scale: lane holds dims 32pr + e (o[e][0|2]) and 32pr + 16 + e (o[e][1|3])
  l_lo += __shfl_xor_sync(0xffffffffu, l_lo, 1);
  l_lo += __shfl_xor_sync(0xffffffffu, l_lo, 2);
  l_hi += __shfl_xor_sync(0xffffffffu, l_hi, 1);
  l_hi += __shfl_xor_sync(0xffffffffu, l_hi, 2);
  const float vs = P.v_scale[g];
  auto store_row = [&](bool okr, int pi, int h, float l, int i0, int i1) {
    if (!okr) return;
    const float inv = l > 0.f ? vs / l : 0.f;
    uint4 *dst = reinterpret_cast<uint4 *>(P.out + ((int64_t)(q0 + pi) * P.num_q_heads + h) * D + 32 * pr);
#pragma unroll
    for (int half = 0; half < 2; ++half) {          // dims 32pr + 16*half + [0, 16)
      const int col = half ? i1 : i0;
      uint32_t w[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) w[k] = pack_bf16x2(o[2 * k][col] * inv, o[2 * k + 1][col] * inv);
      dst[2 * half] = make_uint4(w[0], w[1], w[2], w[3]);
      dst[2 * half + 1] = make_uint4(w[4], w[5], w[6], w[7]);
    }
  };
  store_row(ok_lo, pi_lo, h_lo, l_lo, 0, 1);
  store_row(ok_hi, pi_hi, h_hi, l_hi, 2, 3);
}

// Launch for one-byte caches (kv_dtype 1 or 2) at head_dim 128.  Returns 0, -1 (sizes) or -3 (CUDA).
inline int launch_prefill_mma(int kv_dtype, void *out, const void *q, const int32_t *cu_q_lens, int num_chunks,
                              const void *k_cache, const void *v_cache, const int32_t *block_tables,
                              int max_blocks_per_seq, const int32_t *context_lens, int num_q_heads,
                              int num_kv_heads, int64_t num_blocks, int block_size, float scale,
                              const float *k_scale, const float *v_scale, int max_q_len, int max_context_len,
                              cudaStream_t st) {
  constexpr int NW = 4, STAGES = 4;
  using C = PrefillMmaCfg<NW, STAGES>;
  if (num_chunks > 65535 || num_q_heads > 65535) return -1;
  PrefillMmaParams P;
  P.out = static_cast<__nv_bfloat16 *>(out);
  P.q = static_cast<const __nv_bfloat16 *>(q);
  P.cu_q_lens = cu_q_lens;
  P.block_tables = block_tables;
  P.context_lens = context_lens;
  P.k_scale = k_scale;
  P.v_scale = v_scale;
  P.num_blocks = num_blocks;
  P.block_size = block_size;
  P.max_blocks_per_seq = max_blocks_per_seq;
  P.num_q_heads = num_q_heads;
  P.num_kv_heads = num_kv_heads;
  P.group = num_q_heads / num_kv_heads;
  P.hpr = (P.group <= C::ROWS && C::ROWS % P.group == 0) ? P.group : 1;
  P.max_context_len = max_context_len;
  P.qscale = scale * 1.4426950408889634f;
  const int64_t rows = num_blocks * num_kv_heads * block_size;
  CUtensorMap km, vm;
  if (!make_cache_map_u8(&km, k_cache, rows, 128) || !make_cache_map_u8(&vm, v_cache, rows, 128)) return -3;
  const int ppt = C::ROWS / P.hpr;
  const int tiles = (max_q_len + ppt - 1) / ppt;
  if (tiles > 65535) return -1;
  dim3 grid(num_q_heads / P.hpr, tiles, num_chunks);
  auto kern = kv_dtype == 1 ? paged_prefill_mma_kernel<1, NW, STAGES> : paged_prefill_mma_kernel<2, NW, STAGES>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) != cudaSuccess) return -3;
  return launch_pdl(kern, grid, dim3(NW * 32), C::SMEM, st, P, km, vm) == cudaSuccess ? 0 : -3;
}

}  // namespace pa
