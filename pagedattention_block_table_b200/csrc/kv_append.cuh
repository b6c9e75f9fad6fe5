// kv_append.cuh -- scatter new tokens' K/V into their physical slots, and the copy-on-write
// block copy.  Both are pure HBM traffic: 16-byte vector loads and stores, consecutive threads
// on consecutive 16-byte chunks of one row so every warp access is coalesced.
//
// Core Concepts page §3.2 ("PagedAttention 如何工作"): each decode step writes the new token's
// K/V at the end of the sequence's current block; prefill writes all prompt tokens.
// vLLM overview page, section 二 "Prefix Sharing": a diverging request writes into a copy of
// the shared page (copy-on-write), the shared page itself stays unchanged.
#pragma once
#include "pa_common.cuh"

namespace pa {

// One thread = one 16-byte chunk (8 bf16) of one token's row for one KV head, K and V.
// Row n*Hkv + h of k/v goes to cache[slot/bs][h][slot%bs][:] (bs = block size, 16 or 32).
__global__ void kv_append_bf16_kernel(uint4 *__restrict__ k_cache, uint4 *__restrict__ v_cache,
                                      const uint4 *__restrict__ k, const uint4 *__restrict__ v,
                                      const int64_t *__restrict__ slot_mapping, int64_t num_tokens,
                                      int num_kv_heads, int chunks_per_row, int64_t num_slots, int bs) {
  griddep_wait();  // inputs or the cache may belong to the kernel before this one (PDL launch)
  griddep_launch();
  const int64_t total = num_tokens * num_kv_heads * chunks_per_row;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int c = static_cast<int>(i % chunks_per_row);
    const int64_t row = i / chunks_per_row;  // n * Hkv + h
    const int h = static_cast<int>(row % num_kv_heads);
    const int64_t n = row / num_kv_heads;
    const int64_t slot = slot_mapping[n];
    if (slot < 0) continue;
    if (slot >= num_slots) {
      flag_error(kErrSlot);
      continue;
    }
    const int64_t blk = slot / bs, off = slot % bs;
    const int64_t dst = ((blk * num_kv_heads + h) * bs + off) * chunks_per_row + c;
    const uint4 kv = __ldcs(k + i);  // streamed: read once
    const uint4 vv = __ldcs(v + i);
    k_cache[dst] = kv;
    v_cache[dst] = vv;
  }
}

// One-byte variants (FP8 E4M3: KT 1, INT8: KT 2): one thread = 8 elements.  code = E4M3_rn_satfinite(x / scale[h]), the
// quotient an IEEE round-to-nearest binary32 division.
__device__ __forceinline__ uint2 quant8(uint4 x, float s) {
  uint32_t w[4] = {x.x, x.y, x.z, x.w};
  uint32_t out[2];
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    uint32_t packed = 0;
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const uint32_t ww = w[2 * j + k];
      float2 f = make_float2(__fdiv_rn(bf16lo(ww), s), __fdiv_rn(bf16hi(ww), s));
      const __nv_fp8x2_storage_t q = __nv_cvt_float2_to_fp8x2(f, __NV_SATFINITE, __NV_E4M3);
      packed |= static_cast<uint32_t>(q) << (16 * k);
    }
    out[j] = packed;
  }
  return make_uint2(out[0], out[1]);
}

// INT8 variant: code = clamp(round-half-even(x / scale[h]), -127, 127), the quotient an IEEE
// round-to-nearest binary32 division; a NaN quotient stores 0.
__device__ __forceinline__ uint2 quant8_int8(uint4 x, float s) {
  const uint32_t w[4] = {x.x, x.y, x.z, x.w};
  uint32_t out[2] = {0u, 0u};
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const uint32_t ww = w[e >> 1];
    const float q = __fdiv_rn((e & 1) ? bf16hi(ww) : bf16lo(ww), s);
    int c = q == q ? __float2int_rn(q) : 0;
    c = c > 127 ? 127 : (c < -127 ? -127 : c);
    out[e >> 2] |= (static_cast<uint32_t>(c) & 0xffu) << (8 * (e & 3));
  }
  return make_uint2(out[0], out[1]);
}

template <int KT>
__global__ void kv_append_fp8_kernel(uint2 *__restrict__ k_cache, uint2 *__restrict__ v_cache,
                                     const uint4 *__restrict__ k, const uint4 *__restrict__ v,
                                     const int64_t *__restrict__ slot_mapping, int64_t num_tokens,
                                     int num_kv_heads, int chunks_per_row, int64_t num_slots, int bs,
                                     const float *__restrict__ k_scale, const float *__restrict__ v_scale) {
  griddep_wait();
  griddep_launch();
  const int64_t total = num_tokens * num_kv_heads * chunks_per_row;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int c = static_cast<int>(i % chunks_per_row);
    const int64_t row = i / chunks_per_row;
    const int h = static_cast<int>(row % num_kv_heads);
    const int64_t n = row / num_kv_heads;
    const int64_t slot = slot_mapping[n];
    if (slot < 0) continue;
    if (slot >= num_slots) {
      flag_error(kErrSlot);
      continue;
    }
    const int64_t blk = slot / bs, off = slot % bs;
    const int64_t dst = ((blk * num_kv_heads + h) * bs + off) * chunks_per_row + c;
    if constexpr (KT == 1) {
      k_cache[dst] = quant8(__ldcs(k + i), k_scale[h]);
      v_cache[dst] = quant8(__ldcs(v + i), v_scale[h]);
    } else {
      k_cache[dst] = quant8_int8(__ldcs(k + i), k_scale[h]);
      v_cache[dst] = quant8_int8(__ldcs(v + i), v_scale[h]);
    }
  }
}

// Copy-on-write: grid.y = pair; each thread moves 16-byte vectors of the K and V blocks.
__global__ void copy_blocks_kernel(uint4 *__restrict__ k_cache, uint4 *__restrict__ v_cache,
                                   const int32_t *__restrict__ pairs, int64_t vecs_per_block,
                                   int64_t num_blocks) {
  griddep_wait();
  griddep_launch();
  const int p = blockIdx.y;
  const int32_t src = pairs[2 * p], dst = pairs[2 * p + 1];
  if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
    if (threadIdx.x == 0 && blockIdx.x == 0) flag_error(kErrBlockId);
    return;
  }
  const uint4 *ks = k_cache + src * vecs_per_block;
  const uint4 *vs = v_cache + src * vecs_per_block;
  uint4 *kd = k_cache + dst * vecs_per_block;
  uint4 *vd = v_cache + dst * vecs_per_block;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < vecs_per_block;
       i += (int64_t)gridDim.x * blockDim.x) {
    const uint4 a = ks[i];
    const uint4 b = vs[i];
    kd[i] = a;
    vd[i] = b;
  }
}

// Swap (vLLM overview, section 三: pages move out to CPU memory when GPU memory runs short and come
// back when needed): copy whole blocks between two pools, typically the device cache and a pinned
// host pool mapped into the device's address space.  grid.y = pair; every thread keeps several
// 16-byte loads in flight before storing, since host memory is microseconds away.
__global__ void swap_blocks_kernel(uint4 *__restrict__ dst_k, uint4 *__restrict__ dst_v, int64_t dst_num_blocks,
                                   const uint4 *__restrict__ src_k, const uint4 *__restrict__ src_v,
                                   int64_t src_num_blocks, const int32_t *__restrict__ pairs, int64_t vecs_per_block) {
  griddep_wait();
  griddep_launch();
  const int p = blockIdx.y;
  const int32_t s = pairs[2 * p], d = pairs[2 * p + 1];
  if (s < 0 || s >= src_num_blocks || d < 0 || d >= dst_num_blocks) {
    if (threadIdx.x == 0 && blockIdx.x == 0) flag_error(kErrBlockId);
    return;
  }
  const uint4 *ks = src_k + s * vecs_per_block;
  const uint4 *vs = src_v + s * vecs_per_block;
  uint4 *kd = dst_k + d * vecs_per_block;
  uint4 *vd = dst_v + d * vecs_per_block;
  constexpr int U = 4;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i0 = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i0 < vecs_per_block; i0 += U * stride) {
    uint4 a[U], b[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t i = i0 + u * stride;
      if (i < vecs_per_block) {
        a[u] = ks[i];
        b[u] = vs[i];
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t i = i0 + u * stride;
      if (i < vecs_per_block) {
        kd[i] = a[u];
        vd[i] = b[u];
      }
    }
  }
}

}  // namespace pa
