// api.cu -- the extern "C" boundary of libpagedattn.so: host-side argument checks, launch
// configuration, and the per-device error word.  Declarations and argument contracts are in
// include/pagedattn.h.  Everything runs asynchronously on the caller's stream; nothing here
// allocates device memory.
#include <math.h>
#include <stdio.h>

#include <atomic>
#include <vector>

#include "../../include/pagedattn.h"
#include "decode.cuh"
#include "kv_append.cuh"
#include "prefill.cuh"
#include "decode_mma.cuh"

// Launch shapes of the decode kernel (warps per CTA, pipeline stages per warp); overridable
// at build time for tuning sweeps.  Two stages for the small tiles (one-byte caches, head_dim 64):
// their shared memory then allows 6 CTAs per SM instead of 3, and the extra resident warps hide the
// dequantisation's dependent latencies.  Measured on the MHA batch over an FP8 cache (32 x 64 heads,
// contexts 2049..8193): 4 stages 5.06-5.22 TB/s, 3 stages 5.88, 2 stages 6.31 (same bytes in flight
// per SM in each case).
#ifndef PA_DEC_NW
#define PA_DEC_NW 4
#endif
#ifndef PA_DEC_STAGES_BF16_128
#define PA_DEC_STAGES_BF16_128 2
#endif
#ifndef PA_DEC_MMA_MIN_GROUP
#define PA_DEC_MMA_MIN_GROUP 4
#endif
#ifndef PA_DEC_MMA_MIN_GROUP_Q8
// one-byte caches: every group at head_dim 128 (transposed products): G = 2 ran at 5.76 TB/s on the tensor
// cores against 3.88 on the CUDA cores, the MHA FP8 batch (G = 1) at 7.29 against 6.42-6.51
#define PA_DEC_MMA_MIN_GROUP_Q8 1
#endif
#ifndef PA_DEC_MMA_STAGES
#define PA_DEC_MMA_STAGES 2
#endif
// one-byte tiles are half the size of bf16 ones: more stages for the same bytes in flight.  FP8: 3 (4 CTAs per
// SM; 5.68 TB/s against 5.51 with 4 stages on the Llama-3-8B FP8 batch); INT8: 4 (5.45 against 5.17 with 3)
#ifndef PA_DEC_MMA_STAGES_FP8
#define PA_DEC_MMA_STAGES_FP8 3
#endif
#ifndef PA_DEC_MMA_STAGES_INT8
#define PA_DEC_MMA_STAGES_INT8 4
#endif
#ifndef PA_DEC_STAGES_SMALL
#define PA_DEC_STAGES_SMALL 2
#endif

namespace {

constexpr int kMaxDevices = 64;

int device_sm_count() {
  static std::atomic<int> cache[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return 148;
  if (dev >= kMaxDevices) {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n > 0 ? n : 148;
  }
  int v = cache[dev].load(std::memory_order_relaxed);
  if (v == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cache[dev].store(n, std::memory_order_relaxed);
    v = n;
  }
  return v;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

pa_status launch_status() {
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    fprintf(stderr, "pagedattn: launch failed: %s\n", cudaGetErrorString(e));
    return PA_ECUDA;
  }
  return PA_OK;
}

int queries_per_cta(int group) {
  if (group % 4 == 0) return 4;
  if (group % 2 == 0) return 2;
  return 1;
}

// Groups of at least PA_DEC_MMA_MIN_GROUP query heads per KV head over a bf16 cache, and groups of at
// least PA_DEC_MMA_MIN_GROUP_Q8 over a one-byte cache at head_dim 128, decode on the tensor cores
// (decode_mma.cuh): one CTA takes up to 16 heads of a group.  The rest use the CUDA-core kernel.
// Measured on B200 (pa_paged_attention GB/s, CUDA graphs of calls): the Llama-3-8B batch (G = 4)
// 6,030-6,090 on the CUDA cores, 6,370 on the tensor cores; the 32-sequence batch with G = 8 (64 / 8
// heads) 3,210 and 5,280.
bool decode_uses_mma(int kv_dtype, int group, int head_dim) {
  if (!(group <= 16 || group % 16 == 0)) return false;
  if (kv_dtype == PA_KV_BF16) return group >= PA_DEC_MMA_MIN_GROUP;
  // one-byte caches: f16 products on dequantised tiles, head_dim 128
  return head_dim == 128 && group >= PA_DEC_MMA_MIN_GROUP_Q8;
}
int decode_heads_per_cta(int kv_dtype, int group, int head_dim) {
  if (decode_uses_mma(kv_dtype, group, head_dim)) return group < 16 ? group : 16;
  return queries_per_cta(group);
}
int decode_mma_smem(int kv_dtype, int head_dim) {
  if (kv_dtype == PA_KV_FP8_E4M3) return pa::DecodeMmaCfg<1, 128, PA_DEC_NW, PA_DEC_MMA_STAGES_FP8>::SMEM;
  if (kv_dtype == PA_KV_INT8) return pa::DecodeMmaCfg<2, 128, PA_DEC_NW, PA_DEC_MMA_STAGES_INT8>::SMEM;
  return head_dim == 128 ? pa::DecodeMmaCfg<0, 128, PA_DEC_NW, PA_DEC_MMA_STAGES>::SMEM
                         : pa::DecodeMmaCfg<0, 64, PA_DEC_NW, PA_DEC_MMA_STAGES>::SMEM;
}

template <typename K>
pa_status set_smem(K kernel, int bytes) {
  // cudaFuncSetAttribute applies to the current device; cheap to repeat.
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
    return launch_status();
  return PA_OK;
}

template <int KT, int D, int QPB>
constexpr int stages_for() {
  return (KT == 0 && D == 128) ? PA_DEC_STAGES_BF16_128 : PA_DEC_STAGES_SMALL;
}

template <int KT, int D, int QPB>
int decode_smem() {
  return pa::DecodeCfg<KT, D, QPB, PA_DEC_NW, stages_for<KT, D, QPB>()>::SMEM;
}

int decode_smem_rt(int kt, int d, int qpb) {
#define PA_SM(KT, D, Q) \
  if (kt == KT && d == D && qpb == Q) return decode_smem<KT, D, Q>();
  PA_SM(0, 64, 1) PA_SM(0, 64, 2) PA_SM(0, 64, 4) PA_SM(0, 128, 1) PA_SM(0, 128, 2) PA_SM(0, 128, 4)
  PA_SM(1, 64, 1) PA_SM(1, 64, 2) PA_SM(1, 64, 4) PA_SM(1, 128, 1) PA_SM(1, 128, 2) PA_SM(1, 128, 4)
  PA_SM(2, 64, 1) PA_SM(2, 64, 2) PA_SM(2, 64, 4) PA_SM(2, 128, 1) PA_SM(2, 128, 2) PA_SM(2, 128, 4)
#undef PA_SM
  return 0;
}

template <int KT, int D, int QPB, bool ORDERED>
pa_status launch_decode_as(const pa::DecodeParams &P, const pa::WorkOrder<ORDERED> &W, dim3 grid, cudaStream_t st) {
  constexpr int S = stages_for<KT, D, QPB>();
  using C = pa::DecodeCfg<KT, D, QPB, PA_DEC_NW, S>;
  auto kern = pa::paged_decode_kernel<KT, D, QPB, PA_DEC_NW, S, ORDERED>;
  pa_status s = set_smem(kern, C::SMEM);
  if (s != PA_OK) return s;
  if (pa::launch_pdl(kern, grid, dim3(PA_DEC_NW * 32), C::SMEM, st, P, W) != cudaSuccess) return launch_status();
  return launch_status();
}

// order: null for the natural order over grid (units, sequences, splits); else the longest-first list
// of (sequence, split) pairs with grid (units, its length)
template <int KT, int D, int QPB>
pa_status launch_decode(const pa::DecodeParams &P, const pa::WorkOrder<true> *order, int n_order, dim3 grid,
                        cudaStream_t st) {
  if (order) return launch_decode_as<KT, D, QPB, true>(P, *order, dim3(grid.x, n_order, 1), st);
  return launch_decode_as<KT, D, QPB, false>(P, pa::WorkOrder<false>{}, grid, st);
}

// Longest-first list of every (sequence, split) pair of a launch, from the host's copy of the context
// lengths: a counting sort on the tokens each pair holds (min(S, L - z*S), clamped to [0, S]), stable
// in (split, sequence).  Every pair z < max_splits is listed whatever the host lengths say, so the
// result never depends on them, only the order does.  Returns the number of pairs, or 0 (natural
// order) when they do not fit the kernel-parameter list or all lengths are equal.
int build_work_order(const int32_t *host_lens, int num_seqs, int S, int max_context_len, int max_splits,
                     int32_t *item) {
  const int64_t n = (int64_t)num_seqs * max_splits;
  if (n <= 1 || n > pa::kOrderedItems || S <= 0) return 0;
  bool uniform = true;   // equal lengths: the sorted list is the natural order, so launch without one
  for (int b = 1; b < num_seqs && uniform; ++b) uniform = host_lens[b] == host_lens[0];
  if (uniform) return 0;
  std::vector<int> count(S + 2, 0);
  auto tokens = [&](int b, int z) {
    int L = host_lens[b];
    L = L < 0 ? 0 : (L > max_context_len ? max_context_len : L);
    const int64_t t = (int64_t)L - (int64_t)z * S;
    return static_cast<int>(t < 0 ? 0 : (t > S ? S : t));
  };
  for (int z = 0; z < max_splits; ++z)
    for (int b = 0; b < num_seqs; ++b) ++count[S - tokens(b, z)];   // bucket 0 holds the longest
  int run = 0;
  for (int k = 0; k <= S; ++k) {
    const int c = count[k];
    count[k] = run;
    run += c;
  }
  for (int z = 0; z < max_splits; ++z)
    for (int b = 0; b < num_seqs; ++b) item[count[S - tokens(b, z)]++] = (z << 16) | b;
  return static_cast<int>(n);
}

pa_status dispatch_decode(int kt, int d, int qpb, const pa::DecodeParams &P, const pa::WorkOrder<true> *order,
                          int n_order, dim3 grid, cudaStream_t st) {
#define PA_DD(KT, D, Q) \
  if (kt == KT && d == D && qpb == Q) return launch_decode<KT, D, Q>(P, order, n_order, grid, st);
  PA_DD(0, 64, 1) PA_DD(0, 64, 2) PA_DD(0, 64, 4) PA_DD(0, 128, 1) PA_DD(0, 128, 2) PA_DD(0, 128, 4)
  PA_DD(1, 64, 1) PA_DD(1, 64, 2) PA_DD(1, 64, 4) PA_DD(1, 128, 1) PA_DD(1, 128, 2) PA_DD(1, 128, 4)
  PA_DD(2, 64, 1) PA_DD(2, 64, 2) PA_DD(2, 64, 4) PA_DD(2, 128, 1) PA_DD(2, 128, 2) PA_DD(2, 128, 4)
#undef PA_DD
  return PA_EUNSUPPORTED;
}

template <int KT, int D, bool HI, bool ORDERED>
pa_status launch_decode_mma_as(const pa::DecodeParams &P, const CUtensorMap &km, const CUtensorMap &vm,
                               const pa::WorkOrder<ORDERED> &W, dim3 grid, cudaStream_t st) {
  constexpr int S = KT == 0 ? PA_DEC_MMA_STAGES : (KT == 1 ? PA_DEC_MMA_STAGES_FP8 : PA_DEC_MMA_STAGES_INT8);
  using C = pa::DecodeMmaCfg<KT, D, PA_DEC_NW, S>;
  auto kern = pa::paged_decode_mma_kernel<KT, D, PA_DEC_NW, S, HI, ORDERED>;
  pa_status s = set_smem(kern, C::SMEM);
  if (s != PA_OK) return s;
  if (pa::launch_pdl(kern, grid, dim3(PA_DEC_NW * 32), C::SMEM, st, P, km, vm, W) != cudaSuccess)
    return launch_status();
  return launch_status();
}

template <int KT, int D, bool HI>
pa_status launch_decode_mma(const pa::DecodeParams &P, const CUtensorMap &km, const CUtensorMap &vm,
                            const pa::WorkOrder<true> *order, int n_order, dim3 grid, cudaStream_t st) {
  if (order) return launch_decode_mma_as<KT, D, HI, true>(P, km, vm, *order, dim3(grid.x, n_order, 1), st);
  return launch_decode_mma_as<KT, D, HI, false>(P, km, vm, pa::WorkOrder<false>{}, grid, st);
}

// Tensor-core decode: tensor maps over the two caches (rows of head_dim elements), then the launch for the
// cache element, head_dim and whether the CTA's heads reach past 8 rows.
pa_status dispatch_decode_mma(int kt, int d, int hpc, const pa::DecodeParams &P, const pa::WorkOrder<true> *order,
                              int n_order, dim3 grid, cudaStream_t st) {
  CUtensorMap km, vm;
  const int64_t rows = P.num_blocks * P.num_kv_heads * P.block_size;
  const bool maps = kt == PA_KV_BF16
                        ? pa::make_cache_map(&km, P.k_cache, rows, d) && pa::make_cache_map(&vm, P.v_cache, rows, d)
                        : pa::make_cache_map_u8(&km, P.k_cache, rows, d) && pa::make_cache_map_u8(&vm, P.v_cache, rows, d);
  if (!maps) {
    fprintf(stderr, "pagedattn: tensor map encoding for the decode failed\n");
    return PA_ECUDA;
  }
  const bool hi = hpc > 8;
#define PA_DM(KT, D)                                                                                 \
  if (kt == KT && d == D)                                                                            \
    return hi ? launch_decode_mma<KT, D, true>(P, km, vm, order, n_order, grid, st)                  \
              : launch_decode_mma<KT, D, false>(P, km, vm, order, n_order, grid, st);
  PA_DM(0, 128) PA_DM(0, 64) PA_DM(1, 128) PA_DM(2, 128)
#undef PA_DM
  return PA_EUNSUPPORTED;
}

int64_t ceil_div64(int64_t a, int64_t b) { return (a + b - 1) / b; }

}  // namespace

extern "C" {

const char *pa_version(void) { return "pagedattn-b200 0.1.0 (sm_100a)"; }

const char *pa_status_string(pa_status s) {
  switch (s) {
    case PA_OK: return "ok";
    case PA_EINVAL: return "invalid argument";
    case PA_EUNSUPPORTED: return "unsupported configuration";
    case PA_ECUDA: return "CUDA error";
    case PA_EDEVICE_OOB: return "device-side out-of-range block id, slot or length";
    case PA_EWORKSPACE: return "workspace missing or too small";
    case PA_ENOMEM: return "not enough free blocks";
    default: return "unknown status";
  }
}

int64_t pa_kv_cache_bytes(int64_t layers, int64_t kv_heads, int64_t head_dim, int64_t seq_len,
                          int64_t batch, int64_t elem_bytes) {
  if (layers < 0 || kv_heads < 0 || head_dim < 0 || seq_len < 0 || batch < 0 || elem_bytes < 0) return -1;
  return 2 * layers * kv_heads * head_dim * seq_len * batch * elem_bytes;
}

pa_status pa_selftest_bounded_wait(pa_stream_t stream) {
  pa::bounded_wait_selftest_kernel<<<1, 1, 0, reinterpret_cast<cudaStream_t>(stream)>>>();
  return launch_status();
}

pa_status pa_get_device_error(pa_stream_t stream) {
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return launch_status();
  unsigned v = 0;
  if (cudaMemcpyFromSymbol(&v, pa::g_error_word, sizeof v) != cudaSuccess) return launch_status();
  if (v == 0) return PA_OK;
  const unsigned zero = 0;
  if (cudaMemcpyToSymbol(pa::g_error_word, &zero, sizeof zero) != cudaSuccess) return launch_status();
  return PA_EDEVICE_OOB;
}

static bool block_size_ok(int bs) { return bs == 16 || bs == 32; }

pa_status pa_kv_append(void *k_cache, void *v_cache, const void *k, const void *v,
                       const int64_t *slot_mapping, int64_t num_tokens, int num_kv_heads, int head_dim,
                       int64_t num_blocks, int block_size, int kv_dtype, const float *k_scale,
                       const float *v_scale, pa_stream_t stream) {
  if (num_tokens < 0 || num_kv_heads <= 0 || num_blocks <= 0) return PA_EINVAL;
  if (!block_size_ok(block_size)) return PA_EUNSUPPORTED;
  if (head_dim != 64 && head_dim != 128) return PA_EUNSUPPORTED;
  if (kv_dtype != PA_KV_BF16 && kv_dtype != PA_KV_FP8_E4M3 && kv_dtype != PA_KV_INT8) return PA_EUNSUPPORTED;
  if (num_tokens == 0) return PA_OK;
  if (!k_cache || !v_cache || !k || !v || !slot_mapping) return PA_EINVAL;
  if (!aligned16(k_cache) || !aligned16(v_cache) || !aligned16(k) || !aligned16(v) || !aligned16(slot_mapping))
    return PA_EINVAL;
  if (kv_dtype != PA_KV_BF16 && (!k_scale || !v_scale)) return PA_EINVAL;
  if (num_blocks > (int64_t(1) << 40)) return PA_EINVAL;
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int chunks = head_dim / 8;  // 8 elements per thread
  const int64_t total = num_tokens * num_kv_heads * chunks;
  const int threads = 256;
  const int64_t want = ceil_div64(total, threads);
  const int grid = static_cast<int>(want < 65536 ? want : 65536);
  if (kv_dtype == PA_KV_BF16) {
    pa::launch_pdl(pa::kv_append_bf16_kernel, dim3(grid), dim3(threads), 0, st, static_cast<uint4 *>(k_cache),
                   static_cast<uint4 *>(v_cache), static_cast<const uint4 *>(k), static_cast<const uint4 *>(v),
                   slot_mapping, num_tokens, num_kv_heads, chunks, num_blocks * block_size, block_size);
  } else {
    auto kern = kv_dtype == PA_KV_FP8_E4M3 ? pa::kv_append_fp8_kernel<1> : pa::kv_append_fp8_kernel<2>;
    pa::launch_pdl(kern, dim3(grid), dim3(threads), 0, st, static_cast<uint2 *>(k_cache),
                   static_cast<uint2 *>(v_cache), static_cast<const uint4 *>(k), static_cast<const uint4 *>(v),
                   slot_mapping, num_tokens, num_kv_heads, chunks, num_blocks * block_size, block_size, k_scale,
                   v_scale);
  }
  return launch_status();
}

pa_status pa_copy_blocks(void *k_cache, void *v_cache, const int32_t *src_dst_pairs, int num_pairs,
                         int num_kv_heads, int head_dim, int64_t num_blocks, int block_size, int kv_dtype,
                         pa_stream_t stream) {
  if (num_pairs < 0 || num_kv_heads <= 0 || num_blocks <= 0) return PA_EINVAL;
  if (!block_size_ok(block_size)) return PA_EUNSUPPORTED;
  if (head_dim != 64 && head_dim != 128) return PA_EUNSUPPORTED;
  if (kv_dtype != PA_KV_BF16 && kv_dtype != PA_KV_FP8_E4M3 && kv_dtype != PA_KV_INT8) return PA_EUNSUPPORTED;
  if (num_pairs == 0) return PA_OK;
  if (num_pairs > 65535) return PA_EINVAL;
  if (!k_cache || !v_cache || !src_dst_pairs) return PA_EINVAL;
  if (!aligned16(k_cache) || !aligned16(v_cache)) return PA_EINVAL;
  const int elem = kv_dtype == PA_KV_BF16 ? 2 : 1;
  const int64_t vecs = (int64_t)num_kv_heads * block_size * head_dim * elem / 16;
  const int threads = 256;
  const int64_t gx = ceil_div64(vecs, threads);
  dim3 grid(static_cast<unsigned>(gx < 64 ? gx : 64), static_cast<unsigned>(num_pairs));
  pa::launch_pdl(pa::copy_blocks_kernel, grid, dim3(threads), 0, reinterpret_cast<cudaStream_t>(stream),
                 static_cast<uint4 *>(k_cache), static_cast<uint4 *>(v_cache), src_dst_pairs, vecs, num_blocks);
  return launch_status();
}

// A pointer the device can dereference: device memory, managed memory, or host memory that is
// pinned and mapped (its device-side address is returned).  Pageable host memory is rejected.
static bool device_accessible(const void *p, void **dev) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  if (a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged) {
    *dev = const_cast<void *>(p);
    return true;
  }
  if (a.type == cudaMemoryTypeHost && a.devicePointer != nullptr) {
    *dev = a.devicePointer;
    return true;
  }
  return false;
}

pa_status pa_swap_blocks(void *dst_k, void *dst_v, int64_t dst_num_blocks, const void *src_k, const void *src_v,
                         int64_t src_num_blocks, const int32_t *src_dst_pairs, int num_pairs, int num_kv_heads,
                         int head_dim, int block_size, int kv_dtype, pa_stream_t stream) {
  if (num_pairs < 0 || num_kv_heads <= 0 || dst_num_blocks <= 0 || src_num_blocks <= 0) return PA_EINVAL;
  if (!block_size_ok(block_size)) return PA_EUNSUPPORTED;
  if (head_dim != 64 && head_dim != 128) return PA_EUNSUPPORTED;
  if (kv_dtype != PA_KV_BF16 && kv_dtype != PA_KV_FP8_E4M3 && kv_dtype != PA_KV_INT8) return PA_EUNSUPPORTED;
  if (num_pairs == 0) return PA_OK;
  if (num_pairs > 65535) return PA_EINVAL;
  if (!dst_k || !dst_v || !src_k || !src_v || !src_dst_pairs) return PA_EINVAL;
  void *dk, *dv, *sk, *sv, *pr;
  if (!device_accessible(dst_k, &dk) || !device_accessible(dst_v, &dv) || !device_accessible(src_k, &sk) ||
      !device_accessible(src_v, &sv) || !device_accessible(src_dst_pairs, &pr))
    return PA_EINVAL;
  if (!aligned16(dk) || !aligned16(dv) || !aligned16(sk) || !aligned16(sv)) return PA_EINVAL;
  const int elem = kv_dtype == PA_KV_BF16 ? 2 : 1;
  const int64_t vecs = (int64_t)num_kv_heads * block_size * head_dim * elem / 16;
  const int threads = 256;
  const int64_t gx = ceil_div64(vecs, threads * 4);
  dim3 grid(static_cast<unsigned>(gx < 16 ? gx : 16), static_cast<unsigned>(num_pairs));
  pa::launch_pdl(pa::swap_blocks_kernel, grid, dim3(threads), 0, reinterpret_cast<cudaStream_t>(stream),
                 static_cast<uint4 *>(dk), static_cast<uint4 *>(dv), dst_num_blocks, static_cast<const uint4 *>(sk),
                 static_cast<const uint4 *>(sv), src_num_blocks, static_cast<const int32_t *>(pr), vecs);
  return launch_status();
}

int pa_paged_attention_auto_split(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                                  int max_context_len, int kv_dtype) {
  if (num_seqs <= 0 || num_kv_heads <= 0 || num_q_heads <= 0 || max_context_len <= 0) return 16;
  const int group = num_q_heads / num_kv_heads;
  const int hpc = decode_heads_per_cta(kv_dtype, group > 0 ? group : 1, head_dim);
  const int64_t units = (int64_t)num_seqs * num_kv_heads * (group / hpc > 0 ? group / hpc : 1);
  const int smem = decode_uses_mma(kv_dtype, group, head_dim) ? decode_mma_smem(kv_dtype, head_dim)
                                                              : decode_smem_rt(kv_dtype, head_dim, hpc);
  int per_sm = smem > 0 ? (227 * 1024) / (smem + 1024) : 1;
  if (per_sm < 1) per_sm = 1;
  if (per_sm > 8) per_sm = 8;
  const int64_t slots = (int64_t)device_sm_count() * per_sm;
  // Splits of at most 2048 tokens, shortened (powers of two, down to 256) until the launch has enough
  // waves of work units.  Measured on B200 (pa_paged_attention GB/s by split length, longest-first
  // launch order):
  //   CUDA-core kernel: Llama-3-8B batch 512: 5182, 1024: 5461, 2048: 5018; FP8 MHA 512: 4544,
  //     1024: 4736, 2048: 4839  -> about 4 waves;
  //   tensor-core kernel: Llama-3-8B batch 512: 6173, 1024: 6383, 2048: 6433 (3.5 waves at 2048); GQA-8
  //     batch 512: 5315, 1024: 5433, 2048: 5725 (1.2 waves); 8 x 32768 tokens 512: 6277, 1024: 6530,
  //     2048: 6386  -> one wave, and 4 waves once a sequence has 8 or more splits.
  int64_t S = 256;
  while (S < max_context_len && S < 2048) S *= 2;
  const bool mma = decode_uses_mma(kv_dtype, group, head_dim);
  auto enough = [&](int64_t s) {
    const int64_t splits = ceil_div64(max_context_len, s);
    const int64_t work = units * splits;
    if (!mma) return work >= 4 * slots;
    return work >= slots && (splits < 8 || work >= 4 * slots);
  };
  while (S > 256 && !enough(S)) S /= 2;
  return static_cast<int>(S);
}

int pa_paged_attention_uses_tensor_cores(int num_q_heads, int num_kv_heads, int head_dim, int kv_dtype) {
  if (num_q_heads <= 0 || num_kv_heads <= 0 || num_q_heads % num_kv_heads != 0) return -1;
  if (head_dim != 64 && head_dim != 128) return -1;
  if (kv_dtype != PA_KV_BF16 && kv_dtype != PA_KV_FP8_E4M3 && kv_dtype != PA_KV_INT8) return -1;
  return decode_uses_mma(kv_dtype, num_q_heads / num_kv_heads, head_dim) ? 1 : 0;
}

size_t pa_paged_attention_workspace_size(int num_seqs, int num_q_heads, int head_dim, int max_context_len,
                                         int split_tokens) {
  if (num_seqs <= 0 || num_q_heads <= 0 || head_dim <= 0 || max_context_len <= 0 || split_tokens <= 0) return 0;
  const int64_t ms = ceil_div64(max_context_len, split_tokens);
  if (ms <= 1) return 0;
  return static_cast<size_t>((int64_t)num_seqs * num_q_heads * ms * (head_dim + 2) * 4);
}

pa_status pa_paged_attention(void *out, const void *q, const void *k_cache, const void *v_cache,
                             const int32_t *block_tables, int max_blocks_per_seq, const int32_t *context_lens,
                             int num_seqs, int num_q_heads, int num_kv_heads, int head_dim, int64_t num_blocks,
                             int block_size, float scale, int kv_dtype, const float *k_scale, const float *v_scale,
                             int max_context_len, int split_tokens, const int32_t *host_context_lens,
                             void *workspace, size_t workspace_bytes, pa_stream_t stream) {
  if (num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || num_blocks <= 0 || max_blocks_per_seq <= 0)
    return PA_EINVAL;
  if (!block_size_ok(block_size)) return PA_EUNSUPPORTED;
  if (num_blocks * num_kv_heads * (block_size / pa::kBlock) >= (int64_t(1) << 31)) return PA_EINVAL;
  if (num_q_heads % num_kv_heads != 0) return PA_EINVAL;
  if (head_dim != 64 && head_dim != 128) return PA_EUNSUPPORTED;
  if (kv_dtype != PA_KV_BF16 && kv_dtype != PA_KV_FP8_E4M3 && kv_dtype != PA_KV_INT8) return PA_EUNSUPPORTED;
  if (max_context_len < 0 || split_tokens < 0 || split_tokens % pa::kBlock != 0) return PA_EINVAL;
  if (!(scale == scale) || isinf(scale)) return PA_EINVAL;
  if (num_seqs == 0) return PA_OK;
  if (num_seqs > 65535) return PA_EINVAL;
  if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens) return PA_EINVAL;
  if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache)) return PA_EINVAL;
  if (kv_dtype != PA_KV_BF16 && (!k_scale || !v_scale)) return PA_EINVAL;
  const int group = num_q_heads / num_kv_heads;
  const bool mma = decode_uses_mma(kv_dtype, group, head_dim);
  const int qpb = decode_heads_per_cta(kv_dtype, group, head_dim);
  if ((int64_t)num_kv_heads * (group / qpb) > (int64_t(1) << 31) - 1) return PA_EINVAL;
  int S = split_tokens;
  if (S == 0) S = pa_paged_attention_auto_split(num_seqs, num_q_heads, num_kv_heads, head_dim, max_context_len, kv_dtype);
  const int64_t max_splits = max_context_len > 0 ? ceil_div64(max_context_len, S) : 1;
  if (max_splits > 65535) return PA_EINVAL;
  const size_t need = pa_paged_attention_workspace_size(num_seqs, num_q_heads, head_dim, max_context_len, S);
  if (need > 0 && (!workspace || workspace_bytes < need || !aligned16(workspace))) return PA_EWORKSPACE;

  pa::DecodeParams P;
  P.out = static_cast<__nv_bfloat16 *>(out);
  P.q = static_cast<const __nv_bfloat16 *>(q);
  P.k_cache = static_cast<const uint8_t *>(k_cache);
  P.v_cache = static_cast<const uint8_t *>(v_cache);
  P.block_tables = block_tables;
  P.context_lens = context_lens;
  P.k_scale = k_scale;
  P.v_scale = v_scale;
  P.num_blocks = num_blocks;
  P.block_size = block_size;
  P.max_blocks_per_seq = max_blocks_per_seq;
  P.num_q_heads = num_q_heads;
  P.num_kv_heads = num_kv_heads;
  P.group = group;
  P.split_tokens = S;
  P.max_splits = static_cast<int>(max_splits);
  P.max_context_len = max_context_len;
  P.qscale = scale * 1.4426950408889634f;
  if (need > 0) {
    P.ws_o = static_cast<float *>(workspace);
    P.ws_ml = P.ws_o + (int64_t)num_seqs * num_q_heads * max_splits * head_dim;
  } else {
    P.ws_o = nullptr;
    P.ws_ml = nullptr;
  }
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  dim3 grid(static_cast<unsigned>(num_kv_heads * (group / qpb)), static_cast<unsigned>(num_seqs),
            static_cast<unsigned>(max_splits));
  // longest-first order of the (sequence, split) pairs when the caller also has the lengths on the host
  static thread_local pa::WorkOrder<true> order;
  const int n_order = host_context_lens ? build_work_order(host_context_lens, num_seqs, S, max_context_len,
                                                           static_cast<int>(max_splits), order.item)
                                        : 0;
  pa_status s = mma ? dispatch_decode_mma(kv_dtype, head_dim, qpb, P, n_order ? &order : nullptr, n_order, grid, st)
                    : dispatch_decode(kv_dtype, head_dim, qpb, P, n_order ? &order : nullptr, n_order, grid, st);
  if (s != PA_OK || max_splits <= 1) return s;
  dim3 rgrid(static_cast<unsigned>((num_q_heads + 3) / 4), static_cast<unsigned>(num_seqs));
  if (head_dim == 128)
    pa::launch_pdl(pa::lse_reduce_kernel<128>, rgrid, dim3(128), 0, st, P);
  else
    pa::launch_pdl(pa::lse_reduce_kernel<64>, rgrid, dim3(128), 0, st, P);
  return launch_status();
}

namespace {
// The plan of a prefill call whose lengths the caller also has on the host (see plan_prefill); false
// when none applies.  Both the workspace query and the call build it the same way.
bool prefill_plan_for(int num_chunks, const int32_t *host_cu_q_lens, const int32_t *host_context_lens,
                      int num_q_heads, int num_kv_heads, int max_blocks_per_seq, int block_size, int max_q_len,
                      int max_context_len, pa::PrefillPlanHost &plan) {
  if (!host_cu_q_lens || !host_context_lens || num_chunks <= 0 || num_kv_heads <= 0 ||
      num_q_heads % num_kv_heads != 0)
    return false;
  const int group = num_q_heads / num_kv_heads;
  const int hpr = (group <= 128 && 128 % group == 0) ? group : 1;
  const int64_t lim = std::min<int64_t>((int64_t)max_blocks_per_seq * block_size, max_context_len);
  return pa::plan_prefill(host_cu_q_lens, host_context_lens, num_chunks, hpr, num_q_heads / hpr, device_sm_count(),
                          max_q_len, static_cast<int>(lim), plan);
}
thread_local pa::PrefillPlanHost g_prefill_plan;   // 20 KB: kept off the stack
}  // namespace

size_t pa_paged_prefill_workspace_size(int num_chunks, const int32_t *host_cu_q_lens, const int32_t *host_context_lens,
                                       int num_q_heads, int num_kv_heads, int head_dim, int max_blocks_per_seq,
                                       int block_size, int max_q_len, int max_context_len) {
  if (head_dim != 64 && head_dim != 128) return 0;
  pa::PrefillPlanHost &plan = g_prefill_plan;
  if (!prefill_plan_for(num_chunks, host_cu_q_lens, host_context_lens, num_q_heads, num_kv_heads, max_blocks_per_seq,
                        block_size, max_q_len, max_context_len, plan))
    return 0;
  const int group = num_q_heads / num_kv_heads;
  const int hpr = (group <= 128 && 128 % group == 0) ? group : 1;
  return pa::prefill_plan_workspace(plan, num_q_heads / hpr, head_dim);
}

pa_status pa_paged_prefill(void *out, const void *q, const int32_t *cu_q_lens, int num_chunks, const void *k_cache,
                           const void *v_cache, const int32_t *block_tables, int max_blocks_per_seq,
                           const int32_t *context_lens, int num_q_heads, int num_kv_heads, int head_dim,
                           int64_t num_blocks, int block_size, float scale, int kv_dtype, const float *k_scale,
                           const float *v_scale, int max_q_len, int max_context_len, const int32_t *host_cu_q_lens,
                           const int32_t *host_context_lens, void *workspace, size_t workspace_bytes,
                           pa_stream_t stream) {
  if (num_chunks < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || num_blocks <= 0 || max_blocks_per_seq <= 0)
    return PA_EINVAL;
  if (!block_size_ok(block_size)) return PA_EUNSUPPORTED;
  if (num_q_heads % num_kv_heads != 0) return PA_EINVAL;
  if (head_dim != 128 && head_dim != 64) return PA_EUNSUPPORTED;
  if (kv_dtype != PA_KV_BF16 && kv_dtype != PA_KV_FP8_E4M3 && kv_dtype != PA_KV_INT8) return PA_EUNSUPPORTED;
  if (kv_dtype != PA_KV_BF16 && head_dim != 128) return PA_EUNSUPPORTED;
  if (max_q_len < 0 || max_context_len < 0) return PA_EINVAL;
  if (!(scale == scale) || isinf(scale)) return PA_EINVAL;
  if ((host_cu_q_lens == nullptr) != (host_context_lens == nullptr)) return PA_EINVAL;
  if (num_chunks == 0 || max_q_len == 0) return PA_OK;
  if (!out || !q || !cu_q_lens || !k_cache || !v_cache || !block_tables || !context_lens) return PA_EINVAL;
  if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache)) return PA_EINVAL;
  if (kv_dtype != PA_KV_BF16 && (!k_scale || !v_scale)) return PA_EINVAL;
  pa::PrefillPlanHost &plan = g_prefill_plan;
  const bool planned = prefill_plan_for(num_chunks, host_cu_q_lens, host_context_lens, num_q_heads, num_kv_heads,
                                        max_blocks_per_seq, block_size, max_q_len, max_context_len, plan);
  if (planned) {
    const int group = num_q_heads / num_kv_heads;
    const int hpr = (group <= 128 && 128 % group == 0) ? group : 1;
    const size_t need = pa::prefill_plan_workspace(plan, num_q_heads / hpr, head_dim);
    if (need > 0 && (!workspace || workspace_bytes < need || !aligned16(workspace))) return PA_EWORKSPACE;
  }
  const int r = pa::launch_prefill(out, q, cu_q_lens, num_chunks, k_cache, v_cache, block_tables, max_blocks_per_seq,
                                   context_lens, num_q_heads, num_kv_heads, head_dim, num_blocks, block_size, scale,
                                   kv_dtype, k_scale, v_scale, max_q_len, max_context_len,
                                   planned ? &plan : nullptr, workspace, reinterpret_cast<cudaStream_t>(stream));
  if (r == -1) return PA_EINVAL;
  if (r == -2) return PA_EUNSUPPORTED;
  if (r != 0) {
    (void)launch_status();   // reports the CUDA error, if any
    return PA_ECUDA;
  }
  return launch_status();
}

}  // extern "C"

// ---------------------------------------------------------------------------------------------
// pa_paged_attention_noalloc: the decode call for callers that cannot allocate device memory.
// Its split-K partials live in this file-scope array instead of a caller workspace.  Host code
// must not pass `g_noalloc_scratch` itself to a kernel (on the host that name is only a stand-in
// for the device symbol); it passes the device address looked up once per device below.
static __device__ __align__(256) float g_noalloc_scratch[PA_NOALLOC_SCRATCH_BYTES / sizeof(float)];

namespace {
std::atomic<void *> g_noalloc_addr[kMaxDevices];

// Device address of g_noalloc_scratch on the current device (looked up on the first call per device).
void *noalloc_scratch_address() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  void *p = g_noalloc_addr[dev].load(std::memory_order_acquire);
  if (p == nullptr) {
    void *addr = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&addr, g_noalloc_scratch);
    if (e != cudaSuccess || addr == nullptr) {
      fprintf(stderr, "pagedattn: cudaGetSymbolAddress(scratch) failed: %s\n", cudaGetErrorString(e));
      return nullptr;
    }
    g_noalloc_addr[dev].store(addr, std::memory_order_release);
    p = addr;
  }
  return p;
}
}  // namespace

extern "C" pa_status pa_paged_attention_noalloc(void *out, const void *q, const void *k_cache, const void *v_cache,
                                                const int32_t *block_tables, int max_blocks_per_seq,
                                                const int32_t *context_lens, int num_seqs, int num_q_heads,
                                                int num_kv_heads, int head_dim, int64_t num_blocks, float scale,
                                                int kv_dtype, const float *k_scale, const float *v_scale,
                                                int max_context_len, int split_tokens, pa_stream_t stream) {
  const size_t cap = PA_NOALLOC_SCRATCH_BYTES;
  int S = split_tokens;
  if (S == 0 && num_seqs > 0 && num_q_heads > 0 && num_kv_heads > 0 && max_context_len > 0) {
    S = pa_paged_attention_auto_split(num_seqs, num_q_heads, num_kv_heads, head_dim, max_context_len, kv_dtype);
    while (pa_paged_attention_workspace_size(num_seqs, num_q_heads, head_dim, max_context_len, S) > cap)
      S = static_cast<int>(ceil_div64(2 * (int64_t)S, 16) * 16);
  }
  const size_t need = S > 0 ? pa_paged_attention_workspace_size(num_seqs, num_q_heads, head_dim, max_context_len, S) : 0;
  if (need > cap) {
    fprintf(stderr, "pagedattn: pa_paged_attention_noalloc needs %zu bytes of split partials, more than the "
            "%zu-byte static scratch; use a longer split_tokens (or 0)\n", need, cap);
    return PA_EWORKSPACE;
  }
  void *ws = nullptr;
  if (need > 0 && num_seqs > 0) {
    ws = noalloc_scratch_address();
    if (ws == nullptr) return PA_ECUDA;
  }
  return pa_paged_attention(out, q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens, num_seqs,
                            num_q_heads, num_kv_heads, head_dim, num_blocks, PA_BLOCK_SIZE, scale, kv_dtype, k_scale,
                            v_scale, max_context_len, S, nullptr, ws, ws ? cap : 0, stream);
}
