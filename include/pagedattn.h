/*
 * pagedattn.h -- C ABI of libpagedattn.so, the B200 (sm_100a) PagedAttention hot path.
 *
 * Pages this follows (cited by title and section):
 *   [Core Concepts]    "3、核心概念：LLM推理原理、KV Cache、PagedAttention、连续批处理（Continuous
 *                      Batching）机制", §3.1 (decode step: only the new token's K/V are computed,
 *                      its query attends over the cached K/V) and §3.2 (KV cache cut into fixed
 *                      blocks of 16 or 32 tokens; a block table maps logical to physical blocks;
 *                      prefill writes the prompt's K/V into blocks; each decode step writes the new
 *                      token at the end of the current block, taking a new block when it is full;
 *                      the attention kernel reads the non-contiguous K/V through the block table).
 *   [vLLM overview]    uml.org.cn vLLM page, section 二 "PagedAttention" (16-token pages, one page
 *                      table per request, pages stitched together for attention), "Prefix Sharing"
 *                      (shared pages, copy-on-write on divergence), "Continuous Batching" (prefill
 *                      and decode requests in one batch).
 *   [KV Cache to vLLM] "从KV Cache到vLLM：大模型推理提速与显存优化实战", §1.2 (new query against all
 *                      cached keys), §2.1 (KV size formula), §2.2 (1-byte KV elements; GQA: several
 *                      query heads share one KV head).
 *
 * Common conventions
 *   - Block size bs is 16 (PA_BLOCK_SIZE) or 32 tokens [Core Concepts §3.2: "usually 16 or 32"], passed
 *     as `block_size`.  A KV cache is two device arrays, K and V, each laid out
 *     [num_blocks][num_kv_heads][bs][head_dim] ("HND"): one (block, KV head) tile is bs*head_dim
 *     contiguous elements.  Elements are bf16 (PA_KV_BF16), OCP FP8 E4M3
 *     (PA_KV_FP8_E4M3) or signed INT8 (PA_KV_INT8, codes -127..127); the one-byte formats carry one
 *     fp32 scale per KV head for K and one for V: value = code * scale.
 *   - head_dim is 64 or 128.  num_q_heads must be a multiple of num_kv_heads; query head h uses
 *     KV head h / (num_q_heads / num_kv_heads) (any group size).
 *   - bf16 tensors (q, k, v, out) are row-major with the last dimension contiguous.
 *   - A block table is int32 [num_seqs][max_blocks_per_seq]: entry i is the physical block holding
 *     tokens bs*i .. bs*i+bs-1 of that sequence; entries past ceil(context_len/bs) are never read.
 *   - All pointers are DEVICE pointers unless stated; all buffers are owned by the caller; the
 *     library never allocates device memory.  Every call is asynchronous on `stream` (0 = the
 *     legacy default stream) and returns after launching.
 *   - Device pointers must be 16-byte aligned.
 *
 * Errors
 *   Arguments are checked on the host before anything is launched; a bad one returns PA_EINVAL
 *   or PA_EUNSUPPORTED and launches nothing.  A failed launch returns PA_ECUDA.  Values that only
 *   the device sees (a block id outside [0, num_blocks), a slot outside the pool, a context length
 *   beyond the table or beyond max_context_len) are not trusted: the kernel clamps the access into
 *   the pool, sets a per-device error word and carries on; pa_get_device_error() reports it.  No
 *   kernel traps, asserts or waits without a bound.
 */
#ifndef PAGEDATTN_H
#define PAGEDATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *pa_stream_t; /* same handle as cudaStream_t */
typedef int pa_status;

#define PA_OK 0
#define PA_EINVAL (-1)        /* malformed argument (size, null pointer, misalignment) */
#define PA_EUNSUPPORTED (-2)  /* valid but not built: head_dim, group size, dtype */
#define PA_ECUDA (-3)         /* a CUDA launch or query failed */
#define PA_EDEVICE_OOB (-4)   /* a kernel met a block id / slot / length outside its bounds */
#define PA_EWORKSPACE (-5)    /* workspace missing or smaller than required */
#define PA_ENOMEM (-6)        /* block manager: not enough free blocks (nothing was changed) */

#define PA_BLOCK_SIZE 16      /* the default block size; 32 is also supported */
#define PA_KV_BF16 0
#define PA_KV_FP8_E4M3 1
#define PA_KV_INT8 2

/*
 * pa_kv_append -- write new tokens' K and V into their slots [Core Concepts §3.2: each new token is
 * written at the end of its sequence's current block; prefill writes all prompt tokens].
 *   k_cache, v_cache : the cache (see conventions), written in place.
 *   k, v             : bf16 [num_tokens][num_kv_heads][head_dim], the new tokens.
 *   slot_mapping     : int64 [num_tokens]; token n goes to block slot/bs, offset slot%bs.  A negative
 *                      slot means "padding, write nothing".  Slots must be distinct.
 *   kv_dtype         : PA_KV_BF16 (bit copy), PA_KV_FP8_E4M3: code = E4M3(x / scale[h]), the
 *                      binary32 quotient rounded to nearest even and saturated to +-448, or
 *                      PA_KV_INT8: code = clamp(round-half-even(x / scale[h]), -127, 127)
 *                      [KV Cache to vLLM §2.2: INT8 or FP8 KV at one byte per element].
 *   k_scale, v_scale : fp32 [num_kv_heads] device arrays; read for the one-byte formats, may be NULL
 *                      for bf16.
 * num_tokens == 0 launches nothing and returns PA_OK.
 */
pa_status pa_kv_append(void *k_cache, void *v_cache, const void *k, const void *v,
                       const int64_t *slot_mapping, int64_t num_tokens, int num_kv_heads,
                       int head_dim, int64_t num_blocks, int block_size, int kv_dtype,
                       const float *k_scale, const float *v_scale, pa_stream_t stream);

/*
 * pa_copy_blocks -- copy-on-write fork [vLLM overview, Prefix Sharing: after divergence the new token
 * is written into a copied page; the shared page stays unchanged].  For each pair p the whole physical
 * block src_dst_pairs[2p] (all KV heads, bs slots, K and V) is copied to block src_dst_pairs[2p+1].
 *   src_dst_pairs : int32 [num_pairs][2] on the device.  Preconditions: destinations are distinct and
 *                   no destination is also a source in the same call (copies run concurrently).
 */
pa_status pa_copy_blocks(void *k_cache, void *v_cache, const int32_t *src_dst_pairs, int num_pairs,
                         int num_kv_heads, int head_dim, int64_t num_blocks, int block_size,
                         int kv_dtype, pa_stream_t stream);

/*
 * pa_swap_blocks -- move whole blocks between two pools [vLLM overview, section 三: when GPU memory
 * runs short KV pages are swapped out to CPU memory, and swapped back in when the request resumes].
 * For each pair p, block src_dst_pairs[2p] of the source pool (all KV heads, bs slots, K and V) is
 * copied into block src_dst_pairs[2p+1] of the destination pool.  Both pools have the cache layout
 * and the same num_kv_heads, head_dim, block_size and kv_dtype; each may live in device memory or in pinned,
 * mapped host memory (cudaHostAlloc / cudaHostRegister): the kernel reads and writes host memory
 * directly over the host link.  src_dst_pairs must be device-accessible as well.  Pageable host
 * memory is rejected with PA_EINVAL.  Destinations must be distinct and must not overlap sources.
 */
pa_status pa_swap_blocks(void *dst_k, void *dst_v, int64_t dst_num_blocks, const void *src_k,
                         const void *src_v, int64_t src_num_blocks, const int32_t *src_dst_pairs,
                         int num_pairs, int num_kv_heads, int head_dim, int block_size, int kv_dtype,
                         pa_stream_t stream);

/*
 * pa_paged_attention_workspace_size -- bytes of fp32 scratch pa_paged_attention needs for the given
 * split.  0 when every sequence fits one split (no workspace needed).  split_tokens as below.
 */
size_t pa_paged_attention_workspace_size(int num_seqs, int num_q_heads, int head_dim,
                                         int max_context_len, int split_tokens);

/*
 * pa_paged_attention_auto_split -- the split length pa_paged_attention picks for split_tokens == 0.
 */
int pa_paged_attention_auto_split(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                                  int max_context_len, int kv_dtype);

/*
 * pa_paged_attention_uses_tensor_cores -- 1 when pa_paged_attention runs its products on the tensor
 * cores for this shape (a group of at most 16 heads or a multiple of 16, and either a bf16 cache with at
 * least 4 query heads per KV head or a one-byte cache at head_dim 128), 0 when it uses the CUDA-core
 * kernel (smaller bf16 groups, one-byte caches at head_dim 64), -1 for an invalid shape.  Both kernels
 * compute the same function; this only names the one that runs.
 */
int pa_paged_attention_uses_tensor_cores(int num_q_heads, int num_kv_heads, int head_dim, int kv_dtype);

/*
 * pa_paged_attention -- decode attention over the paged cache [Core Concepts §3.2: the kernel reads
 * non-contiguous K/V through the block table; KV Cache to vLLM §1.2: the new token's query attends
 * over all cached keys and takes the weighted sum of values; §2.2 GQA].  For every sequence b and
 * query head h:  out[b][h] = softmax_t(scale * q[b][h] . K_b[t]) . V_b[t]  over t < context_lens[b],
 * K_b[t] = k_cache[block_tables[b][t/bs]][h/G][t%bs].  context_lens counts the newest token (append
 * first, then attend).  A context length of 0 gives a zero row.
 *   out          : bf16 [num_seqs][num_q_heads][head_dim]
 *   q            : bf16 [num_seqs][num_q_heads][head_dim]
 *   block_tables : int32 [num_seqs][max_blocks_per_seq];  context_lens : int32 [num_seqs]
 *   max_context_len : host-side upper bound of context_lens (sizes the launch and the workspace).
 *   split_tokens : tokens per split-K partition (a multiple of 16); 0 = pa_paged_attention_auto_split.
 *                  When a sequence spans several splits each writes a partial (max, sum, unnormalised
 *                  output) to the workspace and a log-sum-exp reduce combines them.
 *   host_context_lens : optional host copy of context_lens (int32 [num_seqs]), or NULL.  When given,
 *                  the (sequence, split) work items are launched longest first (a counting sort on
 *                  the host), so the launch ends on short items instead of idling on a long one.
 *                  Every split up to max_context_len is launched whatever these values are: they
 *                  decide only the order, never the result.  Up to 4000 (sequence, split) pairs;
 *                  beyond that the natural order is used.
 *   workspace    : device scratch of at least pa_paged_attention_workspace_size(...) bytes, or NULL
 *                  when that is 0.  Its contents need no initialisation and are clobbered.
 */
pa_status pa_paged_attention(void *out, const void *q, const void *k_cache, const void *v_cache,
                             const int32_t *block_tables, int max_blocks_per_seq,
                             const int32_t *context_lens, int num_seqs, int num_q_heads,
                             int num_kv_heads, int head_dim, int64_t num_blocks, int block_size,
                             float scale, int kv_dtype, const float *k_scale, const float *v_scale,
                             int max_context_len, int split_tokens,
                             const int32_t *host_context_lens, void *workspace,
                             size_t workspace_bytes, pa_stream_t stream);

/*
 * pa_paged_attention_noalloc -- pa_paged_attention for callers that cannot allocate device memory.
 * The pages have no counterpart of this call.  It exists for callers that cannot call cudaMalloc
 * themselves: a plugin inside a serving engine that has already reserved the GPU's memory for its
 * own KV pool and forbids further allocations, or a latency-critical loop that must not take the
 * device-wide synchronisation a cudaMalloc/cudaFree implies.  Arguments and results are those of
 * pa_paged_attention without `workspace`, for 16-token blocks; the caller still passes every input and
 * output buffer.
 *
 * Instead of a caller workspace, the split-K partials go to one library-owned scratch array of
 * PA_NOALLOC_SCRATCH_BYTES (a file-scope __device__ array: every GPU that loads the library holds
 * it until the process exits).  The first call on a device looks up that array's device address
 * (cudaGetSymbolAddress, with that device current); make that first call before any stream capture.
 * All calls on a device share the one array and it keeps the last call's contents; the kernels
 * write every partial they read, so nothing needs clearing between calls, but calls whose work
 * overlaps on the GPU (two streams, two host threads) race on it and must be serialised by the caller.
 * With split_tokens == 0 the split length is the auto choice, lengthened until the partials fit; an
 * explicit split_tokens whose partials would exceed the array returns PA_EWORKSPACE and launches
 * nothing.  Never calls cudaMalloc, cudaFree or any allocating routine.
 */
#define PA_NOALLOC_SCRATCH_BYTES (16u * 1024u * 1024u)
pa_status pa_paged_attention_noalloc(void *out, const void *q, const void *k_cache, const void *v_cache,
                                     const int32_t *block_tables, int max_blocks_per_seq,
                                     const int32_t *context_lens, int num_seqs, int num_q_heads,
                                     int num_kv_heads, int head_dim, int64_t num_blocks, float scale,
                                     int kv_dtype, const float *k_scale, const float *v_scale,
                                     int max_context_len, int split_tokens, pa_stream_t stream);

/*
 * pa_paged_prefill -- causal attention of prefill chunks over their paged history [vLLM overview,
 * Continuous Batching: requests in prefill share the batch with decoding ones; Core Concepts §3.2:
 * prefill writes the prompt's K/V into blocks].  Chunk c owns query rows cu_q_lens[c] ..
 * cu_q_lens[c+1]-1 (C_c rows) and its context_lens[c] = H_c + C_c tokens are in the cache (append the
 * chunk first).  Row i of the chunk is position H_c + i and attends to positions t <= H_c + i.
 *   out, q       : bf16 [cu_q_lens[num_chunks]][num_q_heads][head_dim]
 *   cu_q_lens    : int32 [num_chunks + 1] on the device, non-decreasing, cu_q_lens[0] = 0
 *   block_tables : int32 [num_chunks][max_blocks_per_seq];  context_lens : int32 [num_chunks]
 *   max_q_len    : host-side upper bound of C_c;  max_context_len : upper bound of context_lens.
 *   kv_dtype     : PA_KV_BF16 (head_dim 64 or 128), or PA_KV_FP8_E4M3 / PA_KV_INT8 (head_dim 128), with
 *                  k_scale / v_scale fp32 [num_kv_heads] on the device as for pa_paged_attention (NULL for
 *                  bf16): K[t] = code * k_scale[h/G], V[t] = code * v_scale[h/G]  [KV Cache to vLLM §2.2].
 * A chunk whose C_c exceeds max_q_len, or whose context exceeds max_context_len or its table row,
 * sets the device error word (PA_EDEVICE_OOB from pa_get_device_error) and its rows are not written.
 * All cache types run on the tcgen05 tensor cores (one-byte codes are converted to f16 tiles in shared
 * memory inside the kernel).  A one-byte cache at head_dim 64 returns PA_EUNSUPPORTED.
 *   host_cu_q_lens, host_context_lens : optional host copies of cu_q_lens / context_lens (both or
 *                  neither; they must hold the same values as the device arrays).  With them the call
 *                  plans its launch: work items longest first, and a CTA whose key range is long next to
 *                  the launch's work per SM is cut into pieces whose partial results a second kernel
 *                  merges (the same log-sum-exp merge as the decode's split-K).  The plan changes the
 *                  schedule only, not the result beyond rounding.  Without them the launch is ordered on
 *                  the device by context length and nothing is split.
 *   workspace    : device memory of at least pa_paged_prefill_workspace_size(...) bytes, 16-byte aligned,
 *                  for the pieces' partials (NULL when that size is 0); owned by the caller, reusable
 *                  once the call has completed on the stream.  Too small: PA_EWORKSPACE, nothing launched.
 */
pa_status pa_paged_prefill(void *out, const void *q, const int32_t *cu_q_lens, int num_chunks,
                           const void *k_cache, const void *v_cache, const int32_t *block_tables,
                           int max_blocks_per_seq, const int32_t *context_lens, int num_q_heads,
                           int num_kv_heads, int head_dim, int64_t num_blocks, int block_size,
                           float scale, int kv_dtype, const float *k_scale, const float *v_scale,
                           int max_q_len, int max_context_len, const int32_t *host_cu_q_lens,
                           const int32_t *host_context_lens, void *workspace, size_t workspace_bytes,
                           pa_stream_t stream);

/* pa_paged_prefill_workspace_size -- bytes of workspace a pa_paged_prefill call with these host lengths
 * needs (0: the plan splits nothing, or no host lengths).  Deterministic for given arguments on a given
 * device model (the plan depends on its SM count). */
size_t pa_paged_prefill_workspace_size(int num_chunks, const int32_t *host_cu_q_lens,
                                       const int32_t *host_context_lens, int num_q_heads, int num_kv_heads,
                                       int head_dim, int max_blocks_per_seq, int block_size, int max_q_len,
                                       int max_context_len);

/* ------------------------------------------------------------------------------------------------
 * Host block manager: the control plane that produces block tables, slot mappings and copy-on-write
 * pairs for the kernels above.  Host memory only; not thread-safe (one manager per scheduler thread).
 * [Core Concepts §3.2: blocks are taken on demand, a new one when the current block is full;
 *  vLLM overview, Prefix Sharing: shared pages, copy-on-write on the first write after a fork;
 *  vLLM overview, Continuous Batching: a finished request's pages return to the pool at once.]
 * Sequences are named by caller-chosen int64 ids.
 */
typedef struct pa_block_manager pa_block_manager;

/* pa_bm_create -- pool of num_blocks physical blocks of block_size tokens (16 or 32).  shuffle_seed != 0
 * hands blocks out in a seeded random order (a long-running server's scattered placement); 0 hands them
 * out in order.  NULL on bad arguments or out of host memory. */
pa_block_manager *pa_bm_create(int64_t num_blocks, int block_size, uint64_t shuffle_seed);
void pa_bm_destroy(pa_block_manager *bm);
/* pa_bm_block_size -- tokens per block of the manager (-1 for a NULL manager). */
int pa_bm_block_size(const pa_block_manager *bm);
/* pa_bm_num_free -- blocks available for new contents: free ones and, with prefix caching, cached
 * evictable ones (-1 for a NULL manager). */
int64_t pa_bm_num_free(const pa_block_manager *bm);
/* pa_bm_add -- register an empty sequence.  PA_EINVAL if the id exists. */
pa_status pa_bm_add(pa_block_manager *bm, int64_t seq_id);
/*
 * pa_bm_add_prompt -- register a new sequence with a prompt of n_tokens token ids, sharing the blocks of
 * any earlier prompt that starts alike [vLLM overview, Prefix Sharing].  Full prompt blocks whose K/V
 * have been committed (pa_bm_commit) form a prefix tree keyed by (previous block, token ids); the
 * longest chain of blocks that exactly match a node is shared (reference counts + 1), and *reused_out
 * is its length in tokens (a multiple of the block size).  The block holding the prompt's last token is
 * never shared, so at least one token stays new: its query is what the next token depends on.  The
 * remaining n_tokens - *reused_out tokens get slots in new blocks, written to slots_out[0 ..] in order:
 * only those need their K/V appended; the shared ones are already in the cache.  The prompt's own full
 * blocks join the tree when pa_bm_commit reports them written, never before.  A node lives while some
 * sequence holds its block (or, with prefix caching on, until it is evicted).
 * PA_EINVAL if the id exists; PA_ENOMEM (nothing changed) if the pool is short.
 */
pa_status pa_bm_add_prompt(pa_block_manager *bm, int64_t seq_id, const int32_t *tokens, int64_t n_tokens,
                           int64_t *slots_out, int64_t *reused_out);
/*
 * pa_bm_commit -- report that the K/V of the first tokens_written tokens of seq_id are in the cache (for
 * a prompt prefilled in chunks: call it after each chunk's append).  Every full prompt block within them
 * joins the prefix tree and can be shared by later prompts from then on.  A sequence freed before its
 * blocks are committed leaves nothing in the tree.  PA_EINVAL if the id is unknown or tokens_written is
 * negative or beyond the tokens reserved for it.
 */
pa_status pa_bm_commit(pa_block_manager *bm, int64_t seq_id, int64_t tokens_written);
/*
 * pa_bm_set_prefix_caching -- keep_freed != 0: a committed prompt block whose last holder leaves stays
 * in the prefix tree as a cached, evictable block (counted by pa_bm_num_free), so that a later prompt
 * that starts alike can take it back without recomputing its K/V.  Allocation uses free blocks first,
 * then evicts the least recently freed cached block that no other node builds on.  keep_freed == 0
 * (the default) drops the cache at once: cached blocks become free.
 */
pa_status pa_bm_set_prefix_caching(pa_block_manager *bm, int keep_freed);
/* pa_bm_prefix_stats -- blocks currently in the prefix tree, and prompt tokens served from it so far. */
pa_status pa_bm_prefix_stats(const pa_block_manager *bm, int64_t *cached_blocks, int64_t *tokens_reused);
/* pa_bm_fork -- child shares every block of parent (reference counts + 1), same length.  Prompt blocks
 * still waiting for pa_bm_commit are committed through the parent only. */
pa_status pa_bm_fork(pa_block_manager *bm, int64_t parent, int64_t child);
/*
 * pa_bm_append -- reserve slots for n_tokens new tokens at the end of seq_id and write them to
 * slots_out[n_tokens] (slot = block*block_size + offset, ready for pa_kv_append).  If the block that receives
 * the first new token is shared, it is first replaced by a private copy: the (src, dst) pair goes to
 * cow_pairs_out[2] (run pa_copy_blocks on it before the append) and *num_cow_out = 1, else 0.
 * PA_ENOMEM if the pool cannot supply the blocks; then nothing changes.
 */
pa_status pa_bm_append(pa_block_manager *bm, int64_t seq_id, int32_t n_tokens, int64_t *slots_out,
                       int32_t *cow_pairs_out, int32_t *num_cow_out);
/* pa_bm_free -- drop a sequence; blocks no other sequence holds return to the free list. */
pa_status pa_bm_free(pa_block_manager *bm, int64_t seq_id);
/* pa_bm_length -- tokens reserved for seq_id, i.e. slots handed out (-1 if unknown). */
int64_t pa_bm_length(const pa_block_manager *bm, int64_t seq_id);
/* pa_bm_tables -- block tables int32 [n][max_blocks_per_seq] (padded with -1) and lengths int32 [n] of
 * the given sequences, in host memory.  PA_EINVAL if an id is unknown or a table does not fit. */
pa_status pa_bm_tables(const pa_block_manager *bm, const int64_t *seq_ids, int32_t n, int32_t *tables_out,
                       int32_t max_blocks_per_seq, int32_t *lens_out);
/* pa_bm_stats -- tokens held by the pool (shared blocks counted once), blocks in use, blocks held by
 * more than one sequence, copy-on-write copies made so far.  Any output pointer may be NULL. */
pa_status pa_bm_stats(const pa_block_manager *bm, int64_t *tokens_stored, int64_t *blocks_used,
                      int64_t *blocks_shared, int64_t *cow_copies);

/*
 * pa_get_device_error -- synchronise `stream`, then return PA_EDEVICE_OOB if any kernel of this library
 * on the current device has met an out-of-range block id, slot or length since the last call (and
 * clear the flag), else PA_OK (or PA_ECUDA if the synchronisation failed).
 */
pa_status pa_get_device_error(pa_stream_t stream);

/*
 * pa_selftest_bounded_wait -- launch one thread on `stream` that waits on an mbarrier nothing ever
 * completes.  Every wait in this library's kernels is bounded: after 0.2 s the wait gives up, sets the
 * device error word (read by pa_get_device_error as PA_EDEVICE_OOB) and the kernel returns, so the
 * context stays usable.  This call exists to show that on a device (the tests use it); it launches
 * nothing else and touches no caller memory.
 */
pa_status pa_selftest_bounded_wait(pa_stream_t stream);

/* pa_status_string -- static text for a status code. */
const char *pa_status_string(pa_status status);

/*
 * pa_kv_cache_bytes -- bytes of a KV cache [KV Cache to vLLM §2.1]:
 *   2 (K and V) * layers * kv_heads * head_dim * seq_len * batch * elem_bytes.  -1 on negative input.
 */
int64_t pa_kv_cache_bytes(int64_t layers, int64_t kv_heads, int64_t head_dim, int64_t seq_len,
                          int64_t batch, int64_t elem_bytes);

/* pa_version -- library version string. */
const char *pa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* PAGEDATTN_H */
