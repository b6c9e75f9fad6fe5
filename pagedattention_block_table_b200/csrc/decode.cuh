// decode.cuh -- paged decode attention (split-K) and its log-sum-exp reduce, sm_100a.
//
// What it computes (Core Concepts page §3.2; KV Cache to vLLM page §1.2, §2.2): for each
// sequence b and query head h, out = softmax(scale * q . K^T) V over the sequence's context,
// where token t's K/V row is read through the block table: physical block table[b][t/16],
// slot t%16, KV head h / G (GQA: G query heads share one KV head).
//
// Design (B200): the work unit is (sequence, KV head, split of `split_tokens` tokens).  One
// CTA per unit; its warps take the split's 16-token blocks round-robin and each warp runs its
// own pipeline: lane 0 pulls the (block, head) K tile and V tile -- each one contiguous
// 16*head_dim run in the [block][head][16][D] layout -- into shared memory with 1-D bulk async
// copies (mbarrier completion, this CTA's own shared memory only), STAGES blocks ahead.  All query
// heads of the group are processed against each tile, so every KV byte crosses HBM once.
// Scores use an fp32 online softmax in base 2 (q is pre-scaled by scale*log2(e)); partial
// sums are combined with warp shuffles.  Warps of a CTA merge their (max, sum, output) in
// shared memory; a sequence covering several splits writes fp32 partials that
// `lse_reduce_kernel` combines:  out = sum_p 2^(m_p-M) o_p / sum_p 2^(m_p-M) l_p.
// This CUDA-core kernel serves bf16 groups of fewer than 4 query heads, one query head per KV head over a
// one-byte cache, and one-byte caches at head_dim 64; larger groups use the tensor-core kernel of
// decode_mma.cuh (same work units, same partials).
#pragma once
#include "pa_common.cuh"

namespace pa {

struct DecodeParams {
  __nv_bfloat16 *out;
  const __nv_bfloat16 *q;
  const uint8_t *k_cache;
  const uint8_t *v_cache;
  const int32_t *block_tables;
  const int32_t *context_lens;
  const float *k_scale;
  const float *v_scale;
  float *ws_o;   // [B][Hq][max_splits][D] partial outputs (unnormalised)
  float *ws_ml;  // [B][Hq][max_splits][2]  partial (max in log2 units, sum)
  int64_t num_blocks;
  int block_size;       // 16 or 32 tokens per physical block
  int max_blocks_per_seq;
  int num_q_heads;
  int num_kv_heads;
  int group;        // Hq / Hkv
  int split_tokens; // multiple of 16
  int max_splits;   // ceil(max_context_len / split_tokens)
  int max_context_len;
  float qscale;     // scale * log2(e)
};

template <int KT, int D, int QPB, int NW, int STAGES>
struct DecodeCfg {
  static constexpr int E = KT == 0 ? 2 : 1;          // bytes per cache element
  static constexpr int RB = D * E;                   // bytes per token row of one head
  static constexpr int TILE = kBlock * RB;           // bytes of one (block, head) K or V tile
  static constexpr int LPT = (RB / 16) >= 8 ? 8 : RB / 16;  // lanes per token in QK
  static constexpr int TPP = 32 / LPT;               // tokens per QK pass
  static constexpr int NP = kBlock / TPP;            // QK passes per block
  static constexpr int CPL = RB / 16 / LPT;          // 16-byte chunks per lane per token
  static constexpr int CE = 16 / E;                  // elements per 16-byte chunk
  static constexpr int DPL = CPL * CE;               // dims per lane in QK
  static constexpr int LPV = D / 8;                  // lanes per V row in PV (8 elements each)
  static constexpr int RPL = 32 / LPV;               // V rows per PV step
  static constexpr int NU = kBlock / RPL;            // PV steps per block
  static constexpr int P_BYTES = kBlock * QPB * 8;    // p as duplicated pairs (p, p)
  static constexpr int A_BYTES = 16;                 // alpha[QPB], padded
  static constexpr int BAR_BYTES = STAGES * 8;
  static constexpr int WARP_BYTES = ((2 * STAGES * TILE + P_BYTES + A_BYTES + BAR_BYTES) + 127) / 128 * 128;
  static constexpr int SMEM = NW * WARP_BYTES;
  static constexpr int MERGE_FLOATS = QPB * (D + 2);
  static_assert(QPB == 1 || QPB == 2 || QPB == 4, "queries per CTA");
  static_assert(QPB <= LPT, "one query per lane after the reduce-scatter");
  static_assert(MERGE_FLOATS * 4 <= 2 * STAGES * TILE, "merge area fits in the warp's tiles");
};

// Sum `acc[0..N)` over the LPT lanes of a token group, leaving lane-dependent query `qsel`'s
// full sum in acc[0] (reduce-scatter: each butterfly step halves the values a lane keeps).
template <int N, int LPT>
__device__ __forceinline__ float group_reduce_scatter(float (&acc)[N], int lane) {
  int nv = N;
#pragma unroll
  for (int off = LPT / 2; off >= 1; off >>= 1) {
    if (nv > 1) {
      const int half = nv / 2;
      const bool up = (lane & off) != 0;
#pragma unroll
      for (int i = 0; i < N / 2; ++i) {
        if (i < half) {
          const float send = up ? acc[i] : acc[i + half];
          const float keep = up ? acc[i + half] : acc[i];
          acc[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
        }
      }
      nv = half;
    } else {
      acc[0] += __shfl_xor_sync(0xffffffffu, acc[0], off);
    }
  }
  return acc[0];
}

// Query index (within the CTA's QPB) whose sum group_reduce_scatter leaves in this lane.
template <int N, int LPT>
__device__ __forceinline__ int group_reduce_qsel(int lane) {
  int nv = N, qb = 0;
#pragma unroll
  for (int off = LPT / 2; off >= 1; off >>= 1) {
    if (nv > 1) {
      const int half = nv / 2;
      if (lane & off) qb += half;
      nv = half;
    }
  }
  return qb;
}

// Work order of an ordered launch: row y of the grid (units, count) serves the (sequence, split) pair
// item[y] = split << 16 | sequence.  The host lists every pair, longest first, so the launch ends on
// the short ones; CTAs are dispatched in index order.  Passed as a kernel parameter (read from the
// constant bank, no extra memory round trip before a CTA can start).
constexpr int kOrderedItems = 4000;
template <bool ORDERED>
struct WorkOrder {
  int32_t item[ORDERED ? kOrderedItems : 1];   // a natural-order launch carries no list
};

template <int KT, int D, int QPB, int NW, int STAGES, bool ORDERED>
__global__ void __launch_bounds__(NW * 32)
    paged_decode_kernel(const DecodeParams P, const __grid_constant__ WorkOrder<ORDERED> W) {
  using C = DecodeCfg<KT, D, QPB, NW, STAGES>;
  extern __shared__ __align__(128) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // natural order, grid (units, sequences, splits): every sequence's first split is scheduled before
  // any second one, so the CTAs that find their split past a short sequence's end cluster in the last
  // waves.  Ordered launch, grid (units, count): see WorkOrder.
  const int split = ORDERED ? (W.item[blockIdx.y] >> 16) : static_cast<int>(blockIdx.z);
  const int unit = blockIdx.x;
  const int b = ORDERED ? (W.item[blockIdx.y] & 0xffff) : static_cast<int>(blockIdx.y);
  const int sub_groups = P.group / QPB;
  const int g = unit / sub_groups;
  const int h0 = g * P.group + (unit % sub_groups) * QPB;  // first query head of this CTA
  // any input may come from the kernel before this one on the stream (launched with PDL)
  griddep_wait();
  griddep_launch();

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
  const int blk0 = t0 / kBlock;

  uint8_t *wbase = smem + warp * C::WARP_BYTES;
  uint64_t *p_s = reinterpret_cast<uint64_t *>(wbase + 2 * STAGES * C::TILE);
  float *alpha_s = reinterpret_cast<float *>(p_s + kBlock * QPB);
  uint64_t *bars = reinterpret_cast<uint64_t *>(reinterpret_cast<uint8_t *>(alpha_s) + C::A_BYTES);

  const int nwb = nblk > warp ? (nblk - warp + NW - 1) / NW : 0;  // blocks of this warp
  if (lane == 0) {
    for (int s = 0; s < STAGES; ++s) mbar_init(&bars[s], 1);
    fence_mbar_init();
  }
  __syncwarp();

  const int qsel = group_reduce_qsel<QPB, C::LPT>(lane);

  // ---- block-table window: lane k holds the 16-token tile index (in the flat array of 16-row tiles
  // [num_blocks][Hkv][block_size/16]) of this warp's unit win*32 + k; a unit is 16 tokens, so a
  // 32-token block is read as two units
  const int32_t *trow = P.block_tables + (int64_t)b * P.max_blocks_per_seq;
  const int upb = P.block_size / kBlock;   // units per block: 1 or 2
  auto load_window = [&](int win) -> int {
    const int i = win * 32 + lane;
    int tile = 0;
    if (i < nwb) {
      const int u = blk0 + warp + NW * i;   // unit index within the sequence
      int e = __ldg(trow + u / upb);
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
    if (lane == 0) {
      const int s = i % STAGES;
      const int64_t off = (int64_t)tile * C::TILE;
      mbar_arrive_expect_tx(&bars[s], 2 * C::TILE);
      bulk_g2s(wbase + s * C::TILE, P.k_cache + off, C::TILE, &bars[s], pol);
      bulk_g2s(wbase + (STAGES + s) * C::TILE, P.v_cache + off, C::TILE, &bars[s], pol);
    }
  };

  // ---- running state: this lane's query qsel (m, l); o[q][8 dims] for all queries
  float m_run = -INFINITY, l_run = 0.f;
  uint64_t o2[QPB][4];  // packed pairs of this lane's 8 output dims, per query
#pragma unroll
  for (int qi = 0; qi < QPB; ++qi)
#pragma unroll
    for (int e = 0; e < 4; ++e) o2[qi][e] = 0ull;

  const int c = lane % C::LPV, hv = lane / C::LPV;
  int issued = 0;
  for (; issued < STAGES && issued < nwb; ++issued) issue(issued);
  bool ok = true;

  // ---- query registers (loaded while the first tiles are in flight): the dims this lane
  // multiplies in QK, pre-scaled
  const int r = lane / C::LPT, j = lane % C::LPT;
  uint64_t qf2[QPB][C::DPL / 2];  // packed (even, odd) dim pairs, pre-scaled
  {
    float qs = P.qscale;
    if (KT != 0) qs *= P.k_scale[g];
#pragma unroll
    for (int qi = 0; qi < QPB; ++qi) {
      const __nv_bfloat16 *qrow = P.q + ((int64_t)b * P.num_q_heads + h0 + qi) * D;
#pragma unroll
      for (int k = 0; k < C::CPL; ++k) {
        const int d0 = (k * C::LPT + j) * C::CE;
#pragma unroll
        for (int e8 = 0; e8 < C::CE; e8 += 8) {
          const uint4 w = *reinterpret_cast<const uint4 *>(qrow + d0 + e8);
          const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int t = 0; t < 4; ++t)
            qf2[qi][(k * C::CE + e8) / 2 + t] = f2pack(bf16lo(ww[t]) * qs, bf16hi(ww[t]) * qs);
        }
      }
    }
  }

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
    const uint8_t *Kt = wbase + s * C::TILE;
    const uint8_t *Vt = wbase + (STAGES + s) * C::TILE;

    // -- scores: token t = pp*TPP + r, LPT lanes per token
    float sc[C::NP];
#pragma unroll
    for (int pp = 0; pp < C::NP; ++pp) {
      const int t = pp * C::TPP + r;
      uint64_t acc2[QPB];
#pragma unroll
      for (int qi = 0; qi < QPB; ++qi) acc2[qi] = 0ull;
#pragma unroll
      for (int k = 0; k < C::CPL; ++k) {
        const uint4 raw = *reinterpret_cast<const uint4 *>(Kt + t * C::RB + (k * C::LPT + j) * 16);
        const uint32_t ww[4] = {raw.x, raw.y, raw.z, raw.w};
        if constexpr (KT == 0) {
#pragma unroll
          for (int t2 = 0; t2 < 4; ++t2) {
            const uint64_t kv2 = bf16x2_to_f2(ww[t2]);
#pragma unroll
            for (int qi = 0; qi < QPB; ++qi) acc2[qi] = ffma2(qf2[qi][k * C::CE / 2 + t2], kv2, acc2[qi]);
          }
        } else {
#pragma unroll
          for (int t2 = 0; t2 < 4; ++t2) {
            uint64_t a2, b2;
            bytes4_to_f2<KT>(ww[t2], a2, b2);
#pragma unroll
            for (int qi = 0; qi < QPB; ++qi) {
              acc2[qi] = ffma2(qf2[qi][k * C::CE / 2 + 2 * t2], a2, acc2[qi]);
              acc2[qi] = ffma2(qf2[qi][k * C::CE / 2 + 2 * t2 + 1], b2, acc2[qi]);
            }
          }
        }
      }
      float acc[QPB];
#pragma unroll
      for (int qi = 0; qi < QPB; ++qi) {
        const float2 a = f2unpack(acc2[qi]);
        acc[qi] = a.x + a.y;
      }
      const float sv = group_reduce_scatter<QPB, C::LPT>(acc, lane);
      sc[pp] = t < nvalid ? sv : -INFINITY;
    }

    // -- online softmax for query qsel over this block's 16 tokens
    float mb = sc[0];
#pragma unroll
    for (int pp = 1; pp < C::NP; ++pp) mb = fmaxf(mb, sc[pp]);
#pragma unroll
    for (int off = C::LPT; off < 32; off <<= 1) mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, off));
    const float m_new = fmaxf(m_run, mb);
    const float alpha = exp2f(m_run - m_new);
    float ps = 0.f;
#pragma unroll
    for (int pp = 0; pp < C::NP; ++pp) {
      const float pv = exp2f(sc[pp] - m_new);
      ps += pv;
      p_s[(pp * C::TPP + r) * QPB + qsel] = f2pack(pv, pv);
    }
#pragma unroll
    for (int off = C::LPT; off < 32; off <<= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
    l_run = l_run * alpha + ps;
    m_run = m_new;
    if (r == 0) alpha_s[qsel] = alpha;
    __syncwarp();

    // -- o = alpha*o + P V: lane owns dims [8c, 8c+8) and tokens u*RPL + hv
#pragma unroll
    for (int qi = 0; qi < QPB; ++qi) {
      const float a = alpha_s[qi];
      const uint64_t a2 = f2pack(a, a);
#pragma unroll
      for (int e = 0; e < 4; ++e) o2[qi][e] = fmul2(o2[qi][e], a2);
    }
#pragma unroll
    for (int u = 0; u < C::NU; ++u) {
      const int t = u * C::RPL + hv;
      if (t < nvalid) {
        uint64_t v2[4];
        if constexpr (KT == 0) {
          const uint4 raw = *reinterpret_cast<const uint4 *>(Vt + t * C::RB + c * 16);
          v2[0] = bf16x2_to_f2(raw.x);
          v2[1] = bf16x2_to_f2(raw.y);
          v2[2] = bf16x2_to_f2(raw.z);
          v2[3] = bf16x2_to_f2(raw.w);
        } else {
          const uint2 raw = *reinterpret_cast<const uint2 *>(Vt + t * C::RB + c * 8);
          bytes4_to_f2<KT>(raw.x, v2[0], v2[1]);
          bytes4_to_f2<KT>(raw.y, v2[2], v2[3]);
        }
        uint64_t pq[QPB];
        if constexpr (QPB % 2 == 0) {
#pragma unroll
          for (int qi = 0; qi < QPB; qi += 2) {
            const ulonglong2 pp2 = *reinterpret_cast<const ulonglong2 *>(p_s + t * QPB + qi);
            pq[qi] = pp2.x;
            pq[qi + 1] = pp2.y;
          }
        } else {
#pragma unroll
          for (int qi = 0; qi < QPB; ++qi) pq[qi] = p_s[t * QPB + qi];
        }
#pragma unroll
        for (int qi = 0; qi < QPB; ++qi)
#pragma unroll
          for (int e = 0; e < 4; ++e) o2[qi][e] = ffma2(pq[qi], v2[e], o2[qi][e]);
      }
    }
    __syncwarp();
    if (issued < nwb) issue(issued++);
  }
  if (!ok) {
    // a wait gave up: give the copies this warp still has in flight a bounded chance to land,
    // then drop this warp's state (the error word already says why)
    for (int k = i; k < issued; ++k) (void)mbar_wait(&bars[k % STAGES], (k / STAGES) & 1);
    m_run = -INFINITY;
    l_run = 0.f;
#pragma unroll
    for (int qi = 0; qi < QPB; ++qi)
#pragma unroll
      for (int e = 0; e < 4; ++e) o2[qi][e] = 0ull;
  }
  float o[QPB][8];
#pragma unroll
  for (int qi = 0; qi < QPB; ++qi)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 v = f2unpack(o2[qi][e]);
      o[qi][2 * e] = v.x;
      o[qi][2 * e + 1] = v.y;
    }

  // ---- merge the RPL token-parity lane groups, then the warps
#pragma unroll
  for (int off = C::LPV; off < 32; off <<= 1)
#pragma unroll
    for (int qi = 0; qi < QPB; ++qi)
#pragma unroll
      for (int e = 0; e < 8; ++e) o[qi][e] += __shfl_xor_sync(0xffffffffu, o[qi][e], off);
  __syncwarp();
  float *mrg = reinterpret_cast<float *>(wbase);  // this warp's tiles are all consumed
  if (hv == 0) {
#pragma unroll
    for (int qi = 0; qi < QPB; ++qi)
#pragma unroll
      for (int e = 0; e < 8; ++e) mrg[qi * D + c * 8 + e] = o[qi][e];
  }
  if (r == 0) {
    mrg[QPB * D + 2 * qsel] = m_run;
    mrg[QPB * D + 2 * qsel + 1] = l_run;
  }
  __syncthreads();

  const float vs = KT != 0 ? P.v_scale[g] : 1.f;
  for (int idx = threadIdx.x; idx < QPB * D; idx += NW * 32) {
    const int qi = idx / D, d = idx % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w)
      M = fmaxf(M, reinterpret_cast<const float *>(smem + w * C::WARP_BYTES)[QPB * D + 2 * qi]);
    float Lsum = 0.f, O = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < NW; ++w) {
        const float *mw = reinterpret_cast<const float *>(smem + w * C::WARP_BYTES);
        const float sc_w = exp2f(mw[QPB * D + 2 * qi] - M);
        Lsum += sc_w * mw[QPB * D + 2 * qi + 1];
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

// Combine the split partials of every (sequence, query head) whose context spans more than one
// split: out = sum_p 2^(m_p - M) o_p / sum_p 2^(m_p - M) l_p,  M = max_p m_p.
// One warp per (sequence, query head): lane p holds split p's (m, l) so the max and the weights come
// from one round of independent loads and shuffles; then every lane sums its D/32 output dims over
// the splits with independent vector loads.
constexpr int kReduceFast = 8;   // splits up to which the reduce issues all its loads at once

template <int D>
__global__ void __launch_bounds__(128) lse_reduce_kernel(const DecodeParams P) {
  const int h = blockIdx.x * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  const int b = blockIdx.y;
  griddep_wait();  // partials come from the decode kernel just before this one
  griddep_launch();
  if (h >= P.num_q_heads) return;
  int L = P.context_lens[b];
  const int lim = min(P.max_blocks_per_seq * P.block_size, P.max_context_len);
  L = L < 0 ? 0 : (L > lim ? lim : L);
  const int n = (L + P.split_tokens - 1) / P.split_tokens;
  if (n <= 1) return;  // written directly by the decode kernel
  const int64_t row0 = ((int64_t)b * P.num_q_heads + h) * P.max_splits;
  constexpr int DPL = D / 32;
  float acc[DPL];
#pragma unroll
  for (int e = 0; e < DPL; ++e) acc[e] = 0.f;
  float den = 0.f;
  if (n <= kReduceFast) {
    // up to kReduceFast splits: every load is issued before any result is used (one memory round trip)
    const float m_l = lane < n ? P.ws_ml[(row0 + lane) * 2] : -INFINITY;
    const float l_l = lane < n ? P.ws_ml[(row0 + lane) * 2 + 1] : 0.f;
    float ov[kReduceFast][DPL];
#pragma unroll
    for (int k = 0; k < kReduceFast; ++k) {
      if (k < n) {
        const float *op = P.ws_o + (row0 + k) * D + lane * DPL;
        if constexpr (DPL == 4) {
          const float4 v = *reinterpret_cast<const float4 *>(op);
          ov[k][0] = v.x; ov[k][1] = v.y; ov[k][2] = v.z; ov[k][3] = v.w;
        } else {
          const float2 v = *reinterpret_cast<const float2 *>(op);
          ov[k][0] = v.x; ov[k][1] = v.y;
        }
      }
    }
    float M = m_l;
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    const float w = (lane < n && M != -INFINITY) ? exp2f(m_l - M) : 0.f;
    float lw = w * l_l;
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) lw += __shfl_xor_sync(0xffffffffu, lw, off);
    den = lw;
#pragma unroll
    for (int k = 0; k < kReduceFast; ++k) {
      const float wk = __shfl_sync(0xffffffffu, w, k);
      if (k < n) {
#pragma unroll
        for (int e = 0; e < DPL; ++e) acc[e] = fmaf(wk, ov[k][e], acc[e]);
      }
    }
  } else {
    // global max over all splits first (n may exceed 32)
    float M = -INFINITY;
    for (int p = lane; p < n; p += 32) M = fmaxf(M, P.ws_ml[(row0 + p) * 2]);
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    for (int p0 = 0; p0 < n; p0 += 32) {
      const int p = p0 + lane;
      float w = 0.f, lw = 0.f;
      if (p < n && M != -INFINITY) {
        w = exp2f(P.ws_ml[(row0 + p) * 2] - M);
        lw = w * P.ws_ml[(row0 + p) * 2 + 1];
      }
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) lw += __shfl_xor_sync(0xffffffffu, lw, off);
      den += lw;
      const int cnt = min(32, n - p0);
#pragma unroll 4
      for (int k = 0; k < cnt; ++k) {
        const float wk = __shfl_sync(0xffffffffu, w, k);
        const float *op = P.ws_o + (row0 + p0 + k) * D + lane * DPL;
        if constexpr (DPL == 4) {
          const float4 v = *reinterpret_cast<const float4 *>(op);
          acc[0] = fmaf(wk, v.x, acc[0]);
          acc[1] = fmaf(wk, v.y, acc[1]);
          acc[2] = fmaf(wk, v.z, acc[2]);
          acc[3] = fmaf(wk, v.w, acc[3]);
        } else {
          const float2 v = *reinterpret_cast<const float2 *>(op);
          acc[0] = fmaf(wk, v.x, acc[0]);
          acc[1] = fmaf(wk, v.y, acc[1]);
        }
      }
    }
  }
  const float inv = den > 0.f ? 1.f / den : 0.f;
  __nv_bfloat16 *orow = P.out + ((int64_t)b * P.num_q_heads + h) * D + lane * DPL;
#pragma unroll
  for (int e = 0; e < DPL; e += 2)
    *reinterpret_cast<__nv_bfloat162 *>(orow + e) = __floats2bfloat162_rn(acc[e] * inv, acc[e + 1] * inv);
}

}  // namespace pa
