// block_manager.cpp -- host-side manager of the paged KV pool (the control plane that feeds the
// kernels' block tables, slot mappings and copy-on-write pairs).  Plain C++, no device code.
//
// Pages followed:
//   Core Concepts §3.2 ("PagedAttention 如何工作"): blocks are handed out on demand; each decode
//     step writes the new token at the end of the sequence's current block and takes a new
//     physical block from the pool when that block is full.  The batch size is bounded by the
//     number of free blocks, not by a per-request maximum length.
//   vLLM overview, section 二 "Prefix Sharing": requests with a common prefix share its physical
//     pages; when a request writes after the shared part, the page it writes into is copied first
//     (copy-on-write) so the shared page stays unchanged for the others.  Also used for parallel
//     sampling (a fork shares every page of its parent).
//   vLLM overview, section "Continuous Batching": finished requests leave the batch and their pages
//     return to the pool at once.
//
// Structure: a free list (FIFO; optionally shuffled once with a seeded generator, so that physical
// placement is scattered as in a long-running server), a reference count per block, and per
// sequence its block table and length.  Blocks hold 16 or 32 tokens (Core Concepts §3.2: "usually 16
// or 32"), fixed per manager.
//
// Prefix tree (vLLM overview, "Prefix Sharing": requests whose prompts start alike share the pages of
// the common part).  A full prompt block becomes a node keyed by (parent node, its token ids) once the
// caller confirms, with pa_bm_commit, that its K/V are written; a new prompt walks the tree block by
// block and shares every node it matches exactly, so only its remaining tokens need K/V written.  A
// prompt never shares its last token: that position's query must still be computed.  Nodes are looked
// up through a hash of the whole prefix and then compared exactly (parent block and token ids), so a
// hash collision can never share a wrong block.  By default a node lives while some sequence holds its
// block.  With prefix caching on (pa_bm_set_prefix_caching), a node whose last holder leaves stays in
// the tree as a cached block; a later prompt can revive it, and allocation takes truly free blocks
// first, then evicts the least recently freed cached block that no other node builds on (kept in an
// ordered set, so an eviction costs O(log cached blocks)).  So a cached node's parent is never reused
// under it.  Every other call is O(blocks touched).
#include <stdint.h>
#include <string.h>

#include <algorithm>
#include <deque>
#include <new>
#include <random>
#include <set>
#include <unordered_map>
#include <vector>

#include "../../include/pagedattn.h"

namespace {

constexpr int kMaxBlockSize = 32;

struct Seq {
  std::vector<int32_t> blocks;  // logical block i -> physical block
  int64_t len = 0;              // tokens reserved (slots handed out)
  // prompt blocks that join the prefix tree once pa_bm_commit says their K/V are written
  std::vector<int32_t> prompt;  // token ids of the prompt's full blocks (cleared once all are in the tree)
  std::vector<uint64_t> keys;   // prefix key of each full prompt block
  int64_t tree_blocks = 0;      // leading prompt blocks already in the tree (shared or committed)
};

// A full prompt block in the prefix tree.
struct PrefixNode {
  bool live = false;
  int32_t parent = -1;             // block of the previous tokens (-1: the prompt's first block)
  uint64_t key = 0;                // hash of the whole prefix up to and including this block
  int32_t tokens[kMaxBlockSize];   // the block's token ids, compared exactly on every match
};

uint64_t prefix_key(uint64_t parent_key, const int32_t *tokens, int bs) {
  // FNV-1a over the parent's key and the block's token ids, then a splitmix64 finaliser
  uint64_t h = 1469598103934665603ull ^ parent_key;
  for (int i = 0; i < bs; ++i) {
    h ^= static_cast<uint32_t>(tokens[i]);
    h *= 1099511628211ull;
  }
  h ^= h >> 30;
  h *= 0xbf58476d1ce4e5b9ull;
  h ^= h >> 27;
  h *= 0x94d049bb133111ebull;
  return h ^ (h >> 31);
}

}  // namespace

struct pa_block_manager {
  int64_t num_blocks = 0;
  int bs = PA_BLOCK_SIZE;           // tokens per block (16 or 32)
  std::deque<int32_t> free_list;
  std::vector<int32_t> refcount;
  std::unordered_map<int64_t, Seq> seqs;
  int64_t forks = 0;  // copy-on-write copies handed out so far
  // prefix tree: key -> blocks whose prefix hashes to it (exact match decides), node per block
  std::unordered_multimap<uint64_t, int32_t> prefix_index;
  std::vector<PrefixNode> nodes;
  std::vector<int32_t> children;  // live nodes whose parent is this block
  int64_t prefix_tokens_reused = 0;
  // prefix caching: blocks with a live node and no holder ("cached"); the ones no other node builds on
  // are ordered by the time they lost their last holder, oldest first
  bool keep_freed = false;
  uint64_t clock = 0;
  std::vector<uint64_t> freed_at;
  std::vector<char> in_ev;
  int64_t n_evictable = 0;
  std::set<std::pair<uint64_t, int32_t>> ev_leaves;
};

namespace {

// the live node for (parent block, 16 tokens), or -1
int32_t prefix_find(const pa_block_manager *bm, int32_t parent, uint64_t key, const int32_t *tokens) {
  auto range = bm->prefix_index.equal_range(key);
  for (auto it = range.first; it != range.second; ++it) {
    const PrefixNode &nd = bm->nodes[it->second];
    if (nd.live && nd.parent == parent && memcmp(nd.tokens, tokens, sizeof(int32_t) * bm->bs) == 0)
      return it->second;
  }
  return -1;
}

void prefix_forget(pa_block_manager *bm, int32_t b) {
  PrefixNode &nd = bm->nodes[b];
  if (!nd.live) return;
  if (nd.parent >= 0 && --bm->children[nd.parent] == 0 && bm->in_ev[nd.parent])
    bm->ev_leaves.emplace(bm->freed_at[nd.parent], nd.parent);   // the parent became an evictable leaf
  auto range = bm->prefix_index.equal_range(nd.key);
  for (auto it = range.first; it != range.second; ++it)
    if (it->second == b) {
      bm->prefix_index.erase(it);
      break;
    }
  nd.live = false;
}

int64_t available(const pa_block_manager *bm) {
  return static_cast<int64_t>(bm->free_list.size()) + bm->n_evictable;
}

// a cached block leaves the cache (revived by a prompt, or evicted)
void unlist_evictable(pa_block_manager *bm, int32_t b) {
  if (bm->children[b] == 0) bm->ev_leaves.erase({bm->freed_at[b], b});
  bm->in_ev[b] = 0;
  --bm->n_evictable;
}

// A block for new contents (the caller has checked available() first): a free one, else the least
// recently freed cached block on which no other node builds.  One exists whenever a block is cached:
// a sequence that holds a node also holds its parent, so the nodes built on a cached block are cached
// too, and chains end.
int32_t take_block(pa_block_manager *bm) {
  int32_t b;
  if (!bm->free_list.empty()) {
    b = bm->free_list.front();
    bm->free_list.pop_front();
  } else {
    b = bm->ev_leaves.begin()->second;
    unlist_evictable(bm, b);
    prefix_forget(bm, b);   // its contents are about to be overwritten
  }
  bm->refcount[b] = 1;
  return b;
}

void release_block(pa_block_manager *bm, int32_t b) {
  if (--bm->refcount[b] == 0) {
    if (bm->keep_freed && bm->nodes[b].live) {
      bm->in_ev[b] = 1;
      bm->freed_at[b] = ++bm->clock;
      ++bm->n_evictable;
      if (bm->children[b] == 0) bm->ev_leaves.emplace(bm->freed_at[b], b);
    } else {
      prefix_forget(bm, b);   // its contents may be overwritten from now on
      bm->free_list.push_back(b);
    }
  }
}

}  // namespace

extern "C" {

pa_block_manager *pa_bm_create(int64_t num_blocks, int block_size, uint64_t shuffle_seed) {
  if (num_blocks <= 0 || num_blocks > INT32_MAX / kMaxBlockSize) return nullptr;
  if (block_size != 16 && block_size != 32) return nullptr;
  pa_block_manager *bm = new (std::nothrow) pa_block_manager();
  if (!bm) return nullptr;
  bm->num_blocks = num_blocks;
  bm->bs = block_size;
  std::vector<int32_t> order(static_cast<size_t>(num_blocks));
  for (int64_t i = 0; i < num_blocks; ++i) order[i] = static_cast<int32_t>(i);
  if (shuffle_seed != 0) {
    std::mt19937_64 rng(shuffle_seed);
    for (int64_t i = num_blocks - 1; i > 0; --i) {
      std::uniform_int_distribution<int64_t> pick(0, i);
      std::swap(order[i], order[pick(rng)]);
    }
  }
  bm->free_list.assign(order.begin(), order.end());
  bm->refcount.assign(static_cast<size_t>(num_blocks), 0);
  bm->nodes.resize(static_cast<size_t>(num_blocks));
  bm->children.assign(static_cast<size_t>(num_blocks), 0);
  bm->freed_at.assign(static_cast<size_t>(num_blocks), 0);
  bm->in_ev.assign(static_cast<size_t>(num_blocks), 0);
  return bm;
}

int pa_bm_block_size(const pa_block_manager *bm) { return bm ? bm->bs : -1; }

void pa_bm_destroy(pa_block_manager *bm) { delete bm; }

int64_t pa_bm_num_free(const pa_block_manager *bm) { return bm ? available(bm) : -1; }

pa_status pa_bm_set_prefix_caching(pa_block_manager *bm, int keep_freed) {
  if (!bm) return PA_EINVAL;
  bm->keep_freed = keep_freed != 0;
  if (!bm->keep_freed && bm->n_evictable > 0) {   // drop the cache: every cached block becomes free
    std::vector<int32_t> cached;
    for (int64_t b = 0; b < bm->num_blocks; ++b)
      if (bm->in_ev[b]) {
        bm->in_ev[b] = 0;
        cached.push_back(static_cast<int32_t>(b));
      }
    bm->n_evictable = 0;
    bm->ev_leaves.clear();
    for (int32_t b : cached) {
      prefix_forget(bm, b);
      bm->free_list.push_back(b);
    }
  }
  return PA_OK;
}

pa_status pa_bm_add(pa_block_manager *bm, int64_t seq_id) {
  if (!bm) return PA_EINVAL;
  if (bm->seqs.count(seq_id)) return PA_EINVAL;
  bm->seqs.emplace(seq_id, Seq());
  return PA_OK;
}

pa_status pa_bm_add_prompt(pa_block_manager *bm, int64_t seq_id, const int32_t *tokens, int64_t n_tokens,
                           int64_t *slots_out, int64_t *reused_out) {
  if (!bm || n_tokens < 0 || (n_tokens > 0 && (!tokens || !slots_out)) || !reused_out) return PA_EINVAL;
  if (bm->seqs.count(seq_id)) return PA_EINVAL;
  const int bs = bm->bs;
  // walk the tree over the prompt's full blocks; the block holding the last token is never shared
  const int64_t full = n_tokens / bs;
  const int64_t shareable = n_tokens > 0 ? (n_tokens - 1) / bs : 0;
  std::vector<int32_t> shared;
  std::vector<uint64_t> keys;
  int32_t parent = -1;
  uint64_t key = 0;
  for (int64_t i = 0; i < full; ++i) {
    key = prefix_key(key, tokens + i * bs, bs);
    keys.push_back(key);
    if (static_cast<int64_t>(shared.size()) == i && i < shareable) {
      const int32_t b = prefix_find(bm, parent, key, tokens + i * bs);
      if (b >= 0) {
        shared.push_back(b);
        parent = b;
      }
    }
  }
  const int64_t reused = static_cast<int64_t>(shared.size()) * bs;
  const int64_t need = (n_tokens + bs - 1) / bs - static_cast<int64_t>(shared.size());
  int64_t revived = 0;   // cached blocks this prompt takes back out of the cache
  for (int32_t b : shared) revived += bm->in_ev[b];
  if (need > available(bm) - revived) return PA_ENOMEM;  // nothing changed
  Seq s;
  for (int32_t b : shared) {
    if (bm->in_ev[b]) unlist_evictable(bm, b);
    ++bm->refcount[b];
    s.blocks.push_back(b);
  }
  for (int64_t i = 0; i < need; ++i) s.blocks.push_back(take_block(bm));
  // the prompt's own full blocks join the tree when pa_bm_commit reports their K/V written
  s.tree_blocks = static_cast<int64_t>(shared.size());
  if (full > s.tree_blocks) {
    s.prompt.assign(tokens, tokens + full * bs);
    s.keys = std::move(keys);
  }
  for (int64_t t = reused; t < n_tokens; ++t)
    slots_out[t - reused] = static_cast<int64_t>(s.blocks[t / bs]) * bs + t % bs;
  s.len = n_tokens;
  bm->seqs.emplace(seq_id, std::move(s));
  bm->prefix_tokens_reused += reused;
  *reused_out = reused;
  return PA_OK;
}

pa_status pa_bm_commit(pa_block_manager *bm, int64_t seq_id, int64_t tokens_written) {
  if (!bm) return PA_EINVAL;
  auto it = bm->seqs.find(seq_id);
  if (it == bm->seqs.end()) return PA_EINVAL;
  Seq &s = it->second;
  if (tokens_written < 0 || tokens_written > s.len) return PA_EINVAL;
  const int bs = bm->bs;
  const int64_t upto = std::min<int64_t>(tokens_written / bs, static_cast<int64_t>(s.keys.size()));
  for (int64_t i = s.tree_blocks; i < upto; ++i) {
    const int32_t b = s.blocks[i];
    PrefixNode &nd = bm->nodes[b];
    nd.live = true;
    nd.parent = i > 0 ? s.blocks[i - 1] : -1;
    nd.key = s.keys[i];
    memcpy(nd.tokens, s.prompt.data() + i * bs, sizeof(int32_t) * bs);
    bm->prefix_index.emplace(nd.key, b);
    if (nd.parent >= 0 && bm->children[nd.parent]++ == 0 && bm->in_ev[nd.parent])
      bm->ev_leaves.erase({bm->freed_at[nd.parent], nd.parent});
  }
  if (upto > s.tree_blocks) s.tree_blocks = upto;
  if (s.tree_blocks >= static_cast<int64_t>(s.keys.size())) {
    std::vector<int32_t>().swap(s.prompt);
    std::vector<uint64_t>().swap(s.keys);
  }
  return PA_OK;
}

pa_status pa_bm_prefix_stats(const pa_block_manager *bm, int64_t *cached_blocks, int64_t *tokens_reused) {
  if (!bm) return PA_EINVAL;
  if (cached_blocks) *cached_blocks = static_cast<int64_t>(bm->prefix_index.size());
  if (tokens_reused) *tokens_reused = bm->prefix_tokens_reused;
  return PA_OK;
}

pa_status pa_bm_fork(pa_block_manager *bm, int64_t parent, int64_t child) {
  if (!bm) return PA_EINVAL;
  auto it = bm->seqs.find(parent);
  if (it == bm->seqs.end() || bm->seqs.count(child)) return PA_EINVAL;
  Seq c;  // same physical blocks, same length; the parent alone registers its prompt blocks
  c.blocks = it->second.blocks;
  c.len = it->second.len;
  for (int32_t b : c.blocks) ++bm->refcount[b];
  bm->seqs.emplace(child, std::move(c));
  return PA_OK;
}

pa_status pa_bm_append(pa_block_manager *bm, int64_t seq_id, int32_t n_tokens, int64_t *slots_out,
                       int32_t *cow_pairs_out, int32_t *num_cow_out) {
  if (!bm || n_tokens < 0 || (n_tokens > 0 && !slots_out) || !num_cow_out) return PA_EINVAL;
  auto it = bm->seqs.find(seq_id);
  if (it == bm->seqs.end()) return PA_EINVAL;
  Seq &s = it->second;
  const int bs = bm->bs;
  *num_cow_out = 0;
  if (n_tokens == 0) return PA_OK;
  // blocks this append needs: new blocks past the table, plus one copy if the current last block
  // is shared and gets written
  const int64_t first = s.len, last = s.len + n_tokens - 1;
  const int64_t have = static_cast<int64_t>(s.blocks.size());
  const int64_t need_blocks = last / bs + 1;
  int64_t needed = need_blocks > have ? need_blocks - have : 0;
  const int64_t first_blk = first / bs;
  const bool cow = first_blk < have && bm->refcount[s.blocks[first_blk]] > 1;
  if (cow) {
    if (!cow_pairs_out) return PA_EINVAL;
    ++needed;
  }
  if (needed > available(bm)) return PA_ENOMEM;  // nothing changed
  if (cow) {
    const int32_t src = s.blocks[first_blk];
    const int32_t dst = take_block(bm);
    --bm->refcount[src];
    s.blocks[first_blk] = dst;
    cow_pairs_out[0] = src;
    cow_pairs_out[1] = dst;
    *num_cow_out = 1;
    ++bm->forks;
  }
  while (static_cast<int64_t>(s.blocks.size()) < need_blocks) s.blocks.push_back(take_block(bm));
  for (int64_t t = first; t <= last; ++t)
    slots_out[t - first] = static_cast<int64_t>(s.blocks[t / bs]) * bs + t % bs;
  s.len = last + 1;
  return PA_OK;
}

pa_status pa_bm_free(pa_block_manager *bm, int64_t seq_id) {
  if (!bm) return PA_EINVAL;
  auto it = bm->seqs.find(seq_id);
  if (it == bm->seqs.end()) return PA_EINVAL;
  // last block first: a prompt's deeper blocks reach the cache before their parents
  const std::vector<int32_t> &blocks = it->second.blocks;
  for (size_t i = blocks.size(); i-- > 0;) release_block(bm, blocks[i]);
  bm->seqs.erase(it);
  return PA_OK;
}

int64_t pa_bm_length(const pa_block_manager *bm, int64_t seq_id) {
  if (!bm) return -1;
  auto it = bm->seqs.find(seq_id);
  return it == bm->seqs.end() ? -1 : it->second.len;
}

pa_status pa_bm_tables(const pa_block_manager *bm, const int64_t *seq_ids, int32_t n, int32_t *tables_out,
                       int32_t max_blocks_per_seq, int32_t *lens_out) {
  if (!bm || n < 0 || (n > 0 && (!seq_ids || !tables_out || !lens_out)) || max_blocks_per_seq <= 0) return PA_EINVAL;
  for (int32_t i = 0; i < n; ++i) {
    auto it = bm->seqs.find(seq_ids[i]);
    if (it == bm->seqs.end()) return PA_EINVAL;
    if (static_cast<int64_t>(it->second.blocks.size()) > max_blocks_per_seq) return PA_EINVAL;
  }
  for (int32_t i = 0; i < n; ++i) {
    const Seq &s = bm->seqs.find(seq_ids[i])->second;
    int32_t *row = tables_out + static_cast<int64_t>(i) * max_blocks_per_seq;
    const size_t nb = s.blocks.size();
    if (nb) memcpy(row, s.blocks.data(), nb * sizeof(int32_t));
    for (int32_t k = static_cast<int32_t>(nb); k < max_blocks_per_seq; ++k) row[k] = -1;
    lens_out[i] = static_cast<int32_t>(s.len);
  }
  return PA_OK;
}

pa_status pa_bm_stats(const pa_block_manager *bm, int64_t *tokens_stored, int64_t *blocks_used,
                      int64_t *blocks_shared, int64_t *cow_copies) {
  if (!bm) return PA_EINVAL;
  int64_t used = 0, shared = 0, toks = 0;
  for (int32_t rc : bm->refcount) {
    used += rc > 0;
    shared += rc > 1;
  }
  // tokens held by the pool: per physical block the largest fill any of its holders reached
  std::vector<int32_t> fill(static_cast<size_t>(bm->num_blocks), 0);
  for (const auto &kv : bm->seqs) {
    const Seq &s = kv.second;
    for (size_t i = 0; i < s.blocks.size(); ++i) {
      const int64_t f = s.len - static_cast<int64_t>(i) * bm->bs;
      const int32_t fi = static_cast<int32_t>(f > bm->bs ? bm->bs : (f < 0 ? 0 : f));
      if (fi > fill[s.blocks[i]]) fill[s.blocks[i]] = fi;
    }
  }
  for (int32_t f : fill) toks += f;
  if (tokens_stored) *tokens_stored = toks;
  if (blocks_used) *blocks_used = used;
  if (blocks_shared) *blocks_shared = shared;
  if (cow_copies) *cow_copies = bm->forks;
  return PA_OK;
}

}  // extern "C"
