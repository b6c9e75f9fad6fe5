"""The host block manager (C++, through the C ABI), on the CPU.

Pins: the append rule of the Core Concepts page §3.2 (write at the end of the current block, a
new block when it is full), copy-on-write of the vLLM overview's Prefix Sharing (a fork shares
pages; the first write into a shared page goes to a copy; the last holder writes in place), and
Continuous Batching's release of a finished request's pages.  A randomised run checks the
manager against a simulated cache: applying its slots and copy pairs to a token-id array, every
sequence must read back exactly its own tokens through its table.  Block sizes 16 and 32 (Core Concepts
§3.2: blocks of 16 or 32 tokens).
"""
import math

import numpy as np
import pytest

from pagedattention_block_table_b200 import binding as B


@pytest.fixture(params=[16, 32])
def bm(request):
    B.lib()
    h = B.pa_bm_create(64, request.param, 0)
    yield h
    B.pa_bm_destroy(h)


def test_append_fills_the_current_block_then_takes_a_new_one(bm):
    bs = B.pa_bm_block_size(bm)
    B.pa_bm_add(bm, 1)
    slots, cow = B.pa_bm_append(bm, 1, bs + 1)             # bs fill block 0, the next one opens block 1
    assert cow is None
    assert list(slots[:bs]) == list(range(bs)) and slots[bs] == bs
    slots, _ = B.pa_bm_append(bm, 1, 1)
    assert slots[0] == bs + 1                               # end of the current block
    assert B.pa_bm_length(bm, 1) == bs + 2
    assert B.pa_bm_num_free(bm) == 62


def test_fork_then_write_copies_the_shared_page(bm):
    bs = B.pa_bm_block_size(bm)
    B.pa_bm_add(bm, 1)
    B.pa_bm_append(bm, 1, bs + 4)                           # blocks 0 (full), 1 (4 tokens)
    B.pa_bm_fork(bm, 1, 2)
    t1, _ = B.pa_bm_tables(bm, [1], 4)
    slots, cow = B.pa_bm_append(bm, 2, 1)                   # child writes into shared block 1
    assert cow is not None and cow[0] == t1[0, 1]
    t2, l2 = B.pa_bm_tables(bm, [2], 4)
    assert t2[0, 0] == t1[0, 0]                             # full block stays shared
    assert t2[0, 1] == cow[1] != t1[0, 1]                   # partial block replaced by its copy
    assert slots[0] == cow[1] * bs + 4 and l2[0] == bs + 5
    s, cow2 = B.pa_bm_append(bm, 1, 1)                      # parent is now the only holder: in place
    assert cow2 is None and s[0] == t1[0, 1] * bs + 4
    st = B.pa_bm_stats(bm)
    assert st["blocks_shared"] == 1 and st["cow_copies"] == 1


def test_free_returns_blocks_only_when_no_holder_is_left(bm):
    bs = B.pa_bm_block_size(bm)
    B.pa_bm_add(bm, 1)
    B.pa_bm_append(bm, 1, 2 * bs + 8)                       # 3 blocks
    B.pa_bm_fork(bm, 1, 2)
    assert B.pa_bm_num_free(bm) == 61
    B.pa_bm_free(bm, 1)
    assert B.pa_bm_num_free(bm) == 61                       # still held by 2
    B.pa_bm_free(bm, 2)
    assert B.pa_bm_num_free(bm) == 64


def test_block_size_must_be_16_or_32():
    B.lib()
    for bad in (0, 8, 24, 64):
        with pytest.raises(B.PagedAttnError):
            B.pa_bm_create(16, bad, 0)


def test_exhausted_pool_changes_nothing():
    h = B.pa_bm_create(4, 16, 0)
    try:
        B.pa_bm_add(h, 1)
        B.pa_bm_append(h, 1, 60)
        with pytest.raises(B.PagedAttnError) as e:
            B.pa_bm_append(h, 1, 10)                        # needs a 5th block
        assert e.value.status == B.PA_ENOMEM
        assert B.pa_bm_length(h, 1) == 60 and B.pa_bm_num_free(h) == 0
        B.pa_bm_append(h, 1, 4)                             # still fits in block 3
    finally:
        B.pa_bm_destroy(h)


def test_bad_ids_are_rejected(bm):
    with pytest.raises(B.PagedAttnError):
        B.pa_bm_append(bm, 99, 1)
    B.pa_bm_add(bm, 5)
    with pytest.raises(B.PagedAttnError):
        B.pa_bm_add(bm, 5)
    with pytest.raises(B.PagedAttnError):
        B.pa_bm_fork(bm, 5, 5)
    assert B.pa_bm_length(bm, 1234) == -1


@pytest.mark.parametrize("bs", [16, 32])
def test_random_operations_read_back_each_sequences_tokens(bs):
    """Random adds, forks, appends and frees; a simulated cache of token ids written through the
    manager's slots and copy pairs must read back every live sequence's own token ids."""
    rng = np.random.default_rng(12)
    nb = 400 * 16 // bs
    h = B.pa_bm_create(nb, bs, 77)
    cache = np.full(nb * bs, -1, np.int64)       # token id stored in each slot
    seqs = {}                                    # id -> list of token ids (the truth)
    next_id, next_tok = 0, 0
    try:
        for step in range(3000):
            op = rng.random()
            live = list(seqs)
            if op < 0.15 or not live:
                B.pa_bm_add(h, next_id)
                seqs[next_id] = []
                next_id += 1
            elif op < 0.25:
                p = live[rng.integers(len(live))]
                B.pa_bm_fork(h, p, next_id)
                seqs[next_id] = list(seqs[p])
                next_id += 1
            elif op < 0.35 and len(live) > 3:
                s = live[rng.integers(len(live))]
                B.pa_bm_free(h, s)
                del seqs[s]
            else:
                s = live[rng.integers(len(live))]
                n = int(rng.integers(1, 40))
                try:
                    slots, cow = B.pa_bm_append(h, s, n)
                except B.PagedAttnError as e:
                    assert e.status == B.PA_ENOMEM
                    continue
                if cow is not None:                  # copy the page first, as pa_copy_blocks would
                    cache[cow[1] * bs:(cow[1] + 1) * bs] = cache[cow[0] * bs:(cow[0] + 1) * bs]
                toks = list(range(next_tok, next_tok + n))
                next_tok += n
                cache[slots] = toks
                seqs[s].extend(toks)
            if step % 100 == 0 or step == 2999:
                ids = list(seqs)
                if not ids:
                    continue
                mbs = max(1, max(math.ceil(len(v) / bs) for v in seqs.values()))
                tables, lens = B.pa_bm_tables(h, ids, mbs)
                for i, sid in enumerate(ids):
                    L = lens[i]
                    assert L == len(seqs[sid])
                    t = np.arange(L)
                    assert np.array_equal(cache[tables[i, t // bs] * bs + t % bs], np.array(seqs[sid], np.int64))
                st = B.pa_bm_stats(h)
                held = set(int(b) for i in range(len(ids)) for b in tables[i] if b >= 0)
                assert st["blocks_used"] == len(held) == nb - B.pa_bm_num_free(h)
    finally:
        B.pa_bm_destroy(h)


@pytest.mark.parametrize("bs", [16, 32])
def test_paged_vs_reserved_memory_utilisation(bs):
    """Continuous batching over a synthetic trace: requests with lognormal prompt and output lengths
    arrive, grow one token per step and leave.  Paged allocation holds only ceil(len/bs) blocks per
    request; a contiguous scheme reserves the maximum length (2048) per request.  The pages report
    ~50% -> >90% utilisation and >70% waste for reservation (KV Cache to vLLM §2.3, §3.2)."""
    rng = np.random.default_rng(3)
    h = B.pa_bm_create(200000 * 16 // bs, bs, 5)
    try:
        live = {}
        util_paged, util_reserved = [], []
        rid = 0
        for step in range(600):
            for _ in range(rng.poisson(2.0)):
                prompt = int(min(1500, max(16, rng.lognormal(math.log(300), 0.8))))
                out = int(min(2048 - prompt, max(8, rng.lognormal(math.log(150), 0.8))))
                B.pa_bm_add(h, rid)
                B.pa_bm_append(h, rid, prompt)
                live[rid] = out
                rid += 1
            for r in list(live):
                B.pa_bm_append(h, r, 1)
                live[r] -= 1
                if live[r] == 0:
                    B.pa_bm_free(h, r)
                    del live[r]
            if step >= 100 and live:
                st = B.pa_bm_stats(h)
                util_paged.append(st["tokens_stored"] / (bs * st["blocks_used"]))
                util_reserved.append(st["tokens_stored"] / (2048 * len(live)))
        assert np.mean(util_paged) > 0.9
        assert np.mean(util_reserved) < 0.5
    finally:
        B.pa_bm_destroy(h)


# ----------------------------------------------------------------------------- prefix tree

def _read_back(h, cache, ids, mbs, bs=16):
    tables, lens = B.pa_bm_tables(h, ids, mbs)
    return [cache[tables[i, np.arange(lens[i]) // bs] * bs + np.arange(lens[i]) % bs] for i in range(len(ids))]


def test_prompts_that_start_alike_share_their_full_blocks():
    """vLLM overview, Prefix Sharing: a second prompt with the same first 40 tokens shares the two full
    blocks (32 tokens) of the first; only its other tokens get new slots, and every sequence reads back
    exactly its own prompt through its table."""
    h = B.pa_bm_create(64, 16, 3)
    try:
        rng = np.random.default_rng(1)
        common = rng.integers(0, 32000, 40)
        p1 = np.concatenate([common, rng.integers(0, 32000, 9)])
        p2 = np.concatenate([common, rng.integers(0, 32000, 30)])
        cache = np.full(64 * 16, -1, np.int64)
        s1, r1 = B.pa_bm_add_prompt(h, 1, p1)
        assert r1 == 0 and len(s1) == len(p1)
        cache[s1] = p1
        B.pa_bm_commit(h, 1, len(p1))
        free_before = B.pa_bm_num_free(h)
        s2, r2 = B.pa_bm_add_prompt(h, 2, p2)
        assert r2 == 32 and len(s2) == len(p2) - 32
        cache[s2] = p2[32:]
        B.pa_bm_commit(h, 2, len(p2))
        assert free_before - B.pa_bm_num_free(h) == -(-(len(p2) - 32) // 16)   # only the unshared blocks
        t, _ = B.pa_bm_tables(h, [1, 2], 8)
        assert list(t[0, :2]) == list(t[1, :2]) and t[0, 2] != t[1, 2]        # block 2 holds 40 != 40 tokens
        got1, got2 = _read_back(h, cache, [1, 2], 8)
        assert np.array_equal(got1, p1) and np.array_equal(got2, p2)
        st = B.pa_bm_prefix_stats(h)
        assert st["tokens_reused"] == 32 and st["cached_blocks"] == 3 + 2      # full blocks of p1 and p2's own
        assert B.pa_bm_stats(h)["blocks_shared"] == 2
    finally:
        B.pa_bm_destroy(h)


def test_prompt_blocks_are_shared_only_once_committed():
    """A prompt prefilled in chunks: until pa_bm_commit reports a block's K/V written, a matching prompt
    must not share it (it would attend to K/V that is not in the cache yet); a sequence freed before it
    committed leaves nothing behind, even with prefix caching on."""
    h = B.pa_bm_create(32, 16, 0)
    try:
        B.pa_bm_set_prefix_caching(h, True)
        p = np.arange(100, 180, dtype=np.int32)                    # 5 full blocks
        B.pa_bm_add_prompt(h, 1, p)                                # chunk 1 (tokens 0..39) not yet written
        assert B.pa_bm_add_prompt(h, 2, p)[1] == 0
        B.pa_bm_commit(h, 1, 40)                                   # chunk 1 written: blocks 0 and 1 complete
        assert B.pa_bm_add_prompt(h, 3, p)[1] == 32
        B.pa_bm_commit(h, 1, 80)                                   # the rest written
        assert B.pa_bm_add_prompt(h, 4, p)[1] == 64                # the block of the last token stays new
        assert B.pa_bm_prefix_stats(h)["cached_blocks"] == 5
        B.pa_bm_add_prompt(h, 5, np.arange(500, 548, dtype=np.int32))
        B.pa_bm_free(h, 5)                                         # never committed: nothing cached
        assert B.pa_bm_prefix_stats(h)["cached_blocks"] == 5
        assert B.pa_bm_add_prompt(h, 6, np.arange(500, 548, dtype=np.int32))[1] == 0
        with pytest.raises(B.PagedAttnError):
            B.pa_bm_commit(h, 6, 49)                               # beyond the reserved tokens
        with pytest.raises(B.PagedAttnError):
            B.pa_bm_commit(h, 77, 1)                               # unknown sequence
    finally:
        B.pa_bm_destroy(h)


@pytest.mark.parametrize("bs", [16, 32])
def test_a_whole_prompt_match_leaves_its_last_token_new(bs):
    """A prompt whose every block matches still gets its last token's block as new: the query of the last
    prompt position is what the next token depends on (vLLM overview, Prefix Sharing: shared pages save
    recomputing K/V, not that query)."""
    h = B.pa_bm_create(32, bs, 0)
    try:
        p = np.arange(2 * bs, dtype=np.int32)                      # exactly two full blocks
        B.pa_bm_add_prompt(h, 1, p)
        B.pa_bm_commit(h, 1, len(p))
        slots, r = B.pa_bm_add_prompt(h, 2, p)
        assert r == bs and len(slots) == bs                        # one block shared, the last one new
        slots, r = B.pa_bm_add_prompt(h, 3, np.arange(2 * bs + 1, dtype=np.int32))
        assert r == 2 * bs and len(slots) == 1                     # one more token: both blocks shared
        slots, r = B.pa_bm_add_prompt(h, 4, p[:bs])
        assert r == 0 and len(slots) == bs                         # a one-block prompt shares nothing
    finally:
        B.pa_bm_destroy(h)


def test_prefix_nodes_live_while_a_holder_does():
    h = B.pa_bm_create(32, 16, 0)
    try:
        p = np.arange(49, dtype=np.int32)                          # three full blocks and one token
        B.pa_bm_add_prompt(h, 1, p)
        B.pa_bm_commit(h, 1, 49)
        B.pa_bm_add_prompt(h, 2, p[:40])                           # shares two, owns one partial block
        B.pa_bm_free(h, 1)                                         # 2 still holds the first two blocks
        _, r = B.pa_bm_add_prompt(h, 3, p)
        assert r == 32                                             # block 3 of p went back to the pool
        B.pa_bm_free(h, 2)
        B.pa_bm_free(h, 3)
        assert B.pa_bm_num_free(h) == 32 and B.pa_bm_prefix_stats(h)["cached_blocks"] == 0
        _, r = B.pa_bm_add_prompt(h, 4, p)                         # nothing held: nothing to share
        assert r == 0
    finally:
        B.pa_bm_destroy(h)


def test_prefix_sharing_stops_at_the_first_block_that_differs():
    h = B.pa_bm_create(32, 16, 0)
    try:
        p = np.arange(64, dtype=np.int32)
        q = p.copy()
        q[20] = -7                                                 # second block differs
        B.pa_bm_add_prompt(h, 1, p)
        B.pa_bm_commit(h, 1, 64)
        _, r = B.pa_bm_add_prompt(h, 2, q)
        assert r == 16
        r3 = B.pa_bm_add_prompt(h, 3, p[16:])[1]                   # same tokens, other position: no match
        assert r3 == 0
        B.pa_bm_append(h, 2, 5)                                    # the shared block is full: no copy
        assert B.pa_bm_stats(h)["cow_copies"] == 0
    finally:
        B.pa_bm_destroy(h)


def test_prompt_that_does_not_fit_changes_nothing():
    h = B.pa_bm_create(4, 16, 0)
    try:
        B.pa_bm_add_prompt(h, 1, np.arange(48, dtype=np.int32))       # 3 blocks
        B.pa_bm_commit(h, 1, 48)
        with pytest.raises(B.PagedAttnError) as e:
            B.pa_bm_add_prompt(h, 2, np.arange(100, 140, dtype=np.int32))   # 3 more blocks, 1 free
        assert e.value.status == B.PA_ENOMEM
        assert B.pa_bm_num_free(h) == 1 and B.pa_bm_length(h, 2) == -1
        _, r = B.pa_bm_add_prompt(h, 2, np.arange(60, dtype=np.int32))      # shares 3 blocks, needs 1
        assert r == 48 and B.pa_bm_num_free(h) == 0
    finally:
        B.pa_bm_destroy(h)


def _random_prompt_run(bs, caching, seed, nb, steps, n_sys, sys_len, tail_len):
    """Prompts built from a few 'system' prefixes plus random tails, prefilled in one to three chunks over
    later steps (each chunk written to the simulated cache, then committed), with decode appends and frees
    in between.  Right after pa_bm_add_prompt the shared part must already read back exactly (a block is
    shared only once its K/V are written), and every live sequence reads back its written tokens."""
    rng = np.random.default_rng(seed)
    h = B.pa_bm_create(nb, bs, 9)
    try:
        B.pa_bm_set_prefix_caching(h, caching)
        systems = [rng.integers(0, 32000, int(rng.integers(*sys_len))) for _ in range(n_sys)]
        cache = np.full(nb * bs, -1, np.int64)
        seqs, pending, nid, reused_total, tok = {}, {}, 0, 0, 10 ** 6
        for step in range(steps):
            # one chunk of every pending prefill is written and committed
            for sid in list(pending):
                p, slots, r, done, cuts = pending[sid]
                hi = cuts.pop(0)
                cache[slots[done - r:hi - r]] = p[done:hi]
                B.pa_bm_commit(h, sid, hi)
                seqs[sid] = list(p[:hi])
                if cuts:
                    pending[sid] = (p, slots, r, hi, cuts)
                else:
                    del pending[sid]
            u = rng.random()
            if u < 0.45 or len(seqs) + len(pending) < 3:
                p = np.concatenate([systems[rng.integers(n_sys)], rng.integers(0, 32000, int(rng.integers(*tail_len)))])
                try:
                    slots, r = B.pa_bm_add_prompt(h, nid, p)
                except B.PagedAttnError as e:
                    assert e.status == B.PA_ENOMEM
                    continue
                assert r < len(p)
                got = _read_back(h, cache, [nid], -(-len(p) // bs), bs)[0][:r]
                assert np.array_equal(got, p[:r]), "a shared block was not written yet"
                k = int(rng.integers(1, 4))
                cuts = sorted(set(int(x) for x in rng.integers(r + 1, len(p) + 1, k - 1)) | {len(p)})
                pending[nid] = (p, slots, r, r, cuts)
                seqs[nid] = list(p[:r])
                reused_total += r
                nid += 1
            elif u < 0.7:
                ready = [s for s in seqs if s not in pending]
                if not ready:
                    continue
                s = ready[rng.integers(len(ready))]
                try:
                    slots, cow = B.pa_bm_append(h, s, 3)
                except B.PagedAttnError as e:
                    assert e.status == B.PA_ENOMEM
                    continue
                if cow is not None:
                    cache[cow[1] * bs:(cow[1] + 1) * bs] = cache[cow[0] * bs:(cow[0] + 1) * bs]
                cache[slots] = np.arange(tok, tok + 3)
                seqs[s] += list(range(tok, tok + 3))
                tok += 3
            else:
                s = list(seqs)[rng.integers(len(seqs))]
                B.pa_bm_free(h, s)                                  # also mid-prefill (an aborted request)
                del seqs[s]
                pending.pop(s, None)
            for sid in seqs:
                n = len(seqs[sid])
                got = _read_back(h, cache, [sid], max(1, -(-B.pa_bm_length(h, sid) // bs)), bs)[0][:n]
                assert np.array_equal(got, np.array(seqs[sid], np.int64))
        assert reused_total > 0 and B.pa_bm_prefix_stats(h)["tokens_reused"] == reused_total
    finally:
        B.pa_bm_destroy(h)


@pytest.mark.parametrize("bs", [16, 32])
def test_random_prompts_with_shared_system_prefixes(bs):
    _random_prompt_run(bs, False, 5, 2000 * 16 // bs, 400, 4, (20, 200), (0, 60))


# ----------------------------------------------------------------------------- prefix caching

def test_prefix_caching_keeps_freed_prompt_blocks_for_later_prompts():
    h = B.pa_bm_create(16, 16, 0)
    try:
        B.pa_bm_set_prefix_caching(h, True)
        p = np.arange(53, dtype=np.int32)                          # 3 full blocks + 5 tokens
        B.pa_bm_add_prompt(h, 1, p)
        B.pa_bm_commit(h, 1, 53)
        B.pa_bm_free(h, 1)
        assert B.pa_bm_num_free(h) == 16                           # cached blocks count as available
        assert B.pa_bm_prefix_stats(h)["cached_blocks"] == 3
        slots, r = B.pa_bm_add_prompt(h, 2, p)
        assert r == 48 and len(slots) == 5                         # only the partial block is new
        assert B.pa_bm_num_free(h) == 16 - 4
        B.pa_bm_set_prefix_caching(h, False)                       # held blocks stay, nothing cached
        B.pa_bm_free(h, 2)
        assert B.pa_bm_prefix_stats(h)["cached_blocks"] == 0 and B.pa_bm_num_free(h) == 16
    finally:
        B.pa_bm_destroy(h)


def test_prefix_cache_evicts_least_recently_freed_leaves_first():
    h = B.pa_bm_create(8, 16, 0)
    try:
        B.pa_bm_set_prefix_caching(h, True)
        a = np.arange(48, dtype=np.int32)                          # three full blocks A0 <- A1 <- A2
        B.pa_bm_add_prompt(h, 1, a)
        B.pa_bm_commit(h, 1, 48)
        B.pa_bm_free(h, 1)                                         # all three cached, five free
        b = np.arange(1000, 1096, dtype=np.int32)                  # 6 blocks: 5 free + the leaf A2 evicted
        B.pa_bm_add_prompt(h, 2, b)
        B.pa_bm_commit(h, 2, 96)
        assert B.pa_bm_num_free(h) == 2 and B.pa_bm_prefix_stats(h)["cached_blocks"] == 6 + 2
        _, r = B.pa_bm_add_prompt(h, 3, a[:32])                    # A0 revives; A1, now a leaf, is evicted
        assert r == 16 and B.pa_bm_num_free(h) == 0
        assert B.pa_bm_prefix_stats(h)["cached_blocks"] == 6 + 1
        with pytest.raises(B.PagedAttnError) as e:                 # 1 block needed, none available
            B.pa_bm_add_prompt(h, 4, np.arange(2000, 2016, dtype=np.int32))
        assert e.value.status == B.PA_ENOMEM
        B.pa_bm_free(h, 3)                                         # A0 cached again, its uncommitted block free
        assert B.pa_bm_num_free(h) == 2
        _, r = B.pa_bm_add_prompt(h, 5, np.arange(3000, 3032, dtype=np.int32))  # the free block, then A0
        assert r == 0 and B.pa_bm_prefix_stats(h)["cached_blocks"] == 6
        B.pa_bm_free(h, 2)                                         # b's six blocks cached, deepest first
        _, r = B.pa_bm_add_prompt(h, 6, b[:81])                    # 5 shared (the last token's block is not)
        assert r == 80
    finally:
        B.pa_bm_destroy(h)


@pytest.mark.parametrize("bs", [16, 32])
def test_random_prompts_with_prefix_caching_and_eviction(bs):
    """Same as the random system-prompt run, with caching on and a pool small enough to evict: a revived
    block still holds the K/V it was given, an evicted one is never shared again."""
    _random_prompt_run(bs, True, 6, 120 * 16 // bs, 600, 5, (20, 120), (0, 40))
