"""Seeded synthetic workloads for the paged KV cache (inputs only, no attention math).

This module is the one place both the CUDA path and the CPU oracle get their inputs
from.  It draws token K/V and queries (N(0,1) rounded to bf16), context lengths with
the distributions of the workloads, a seeded random placement of logical blocks
in the physical pool, the slot of every token, and -- for the prefix-sharing step --
which blocks are shared and which copy-on-write pairs a fork needs.  It holds none
of the method's arithmetic: no attention, no quantisation, no copying of caches.

Cache layout used throughout: ``[num_blocks][num_kv_heads][bs][head_dim]`` with block size
bs = 16 (default) or 32; a token at logical position ``t`` of a sequence lives in physical
block ``block_table[t // bs]`` at offset ``t % bs``, so its slot is
``block_table[t // bs] * bs + t % bs`` (Core Concepts page, section 3.2: the block table
maps logical blocks to physical blocks, blocks of 16 or 32 tokens; vLLM overview page,
section 二: pages of 16 tokens).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Dict, List, Optional

import numpy as np
import torch

BLOCK = 16
E4M3_MAX = 448.0
INT8_MAX = 127.0

# The workloads.  Lengths given here are HISTORIES (tokens already cached);
# every decode sequence then appends one token, so it attends over history + 1.
WORKLOADS: Dict[str, dict] = {
    "tiny_decode": dict(num_seqs=4, num_q_heads=8, num_kv_heads=2, head_dim=64,
                        hist=("fixed", [17, 33, 64, 100]), num_blocks=64),
    "llama3_8b_decode": dict(num_seqs=64, num_q_heads=32, num_kv_heads=8, head_dim=128,
                             hist=("uniform", 512, 4096)),
    "mixed_step": dict(num_seqs=256, num_q_heads=32, num_kv_heads=8, head_dim=128,
                       hist=("lognormal", 800.0, 1.0, 16, 8192),
                       share_group=8, share_prefix=1024,
                       prefill_chunks=4, chunk_len=(512, 2048), chunk_hist=(1, 4095)),
    "long_context_decode": dict(num_seqs=8, num_q_heads=32, num_kv_heads=8, head_dim=128,
                                hist=("fixed", [32767] * 8), split_tokens=512),
    "mha_fp8_decode": dict(num_seqs=32, num_q_heads=64, num_kv_heads=64, head_dim=128,
                           hist=("uniform", 2048, 8192), kv_dtype="fp8"),
    # eight query heads per KV head (the 64 / 8 head layout of a 70B-class model): a decode CTA takes
    # four query heads, so each KV tile is fetched by two CTAs; measures whether the second fetch hits L2
    "gqa8_decode": dict(num_seqs=32, num_q_heads=64, num_kv_heads=8, head_dim=128,
                        hist=("uniform", 512, 4096)),
    # the Llama-3-8B decode batch over an FP8 E4M3 cache: four query heads meet every dequantised byte
    "llama3_8b_fp8_decode": dict(num_seqs=64, num_q_heads=32, num_kv_heads=8, head_dim=128,
                                 hist=("uniform", 512, 4096), kv_dtype="fp8"),
    # the continuous-batching mixed step over an FP8 E4M3 cache (prefill and decode both read one-byte K/V)
    "mixed_step_fp8": dict(num_seqs=256, num_q_heads=32, num_kv_heads=8, head_dim=128,
                           hist=("lognormal", 800.0, 1.0, 16, 8192),
                           share_group=8, share_prefix=1024,
                           prefill_chunks=4, chunk_len=(512, 2048), chunk_hist=(1, 4095), kv_dtype="fp8"),
    # chunked prefill of a long prompt: two 512-token chunks, one starting a prompt and one 32,256 tokens
    # into it (Llama-3-8B heads); 64 query-tile pairs x head groups, far fewer CTAs than SMs unless the
    # long key ranges are split
    "chunked_prefill_long": dict(num_seqs=2, num_q_heads=32, num_kv_heads=8, head_dim=128,
                                 hist=("fixed", [100, 200]), prefill_chunks=2, chunk_len=(512, 512),
                                 chunk_hist=(32256, 32256)),
}
WORKLOAD_SEED = {name: 1001 + i for i, name in enumerate(WORKLOADS)}


def _gen(device, *key) -> torch.Generator:
    """A torch generator on ``device`` seeded from an integer key tuple."""
    s = np.random.SeedSequence([int(k) for k in key]).generate_state(2, dtype=np.uint32)
    g = torch.Generator(device=device)
    g.manual_seed(int(s[0]) << 32 | int(s[1]))
    return g


def randn_bf16(shape, device, *key) -> torch.Tensor:
    """N(0,1) fp32 draws rounded to bf16 (round-to-nearest-even), deterministic in ``key``."""
    g = _gen(device, *key)
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)


@dataclass
class PagedBatch:
    """One step of a batch over a paged KV cache.

    Sequences ``0 .. num_decode-1`` are decoding (one new token each); sequences
    ``num_decode .. num_seqs-1`` are prefill chunks (``new_lens`` new tokens each).
    """

    name: str
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    num_blocks: int
    scale: float
    kv_dtype: int                       # 0 = bf16 cache, 1 = fp8 E4M3 cache, 2 = int8 cache
    block_size: int                     # tokens per physical block (16 or 32)
    num_decode: int
    hist_lens: np.ndarray               # int32 [S] tokens cached before the step
    new_lens: np.ndarray                # int32 [S] tokens appended by the step
    block_tables: np.ndarray            # int32 [S][MBS], after the step's forks; -1 padding
    setup_slots: np.ndarray             # int64 [T_all] slot of every token for the setup fill (-1 skip)
    step_slots: np.ndarray              # int64 [T_new] slot of every appended token
    cow_pairs: np.ndarray               # int32 [P][2] (src, dst) blocks the step's forks copy
    shared_blocks: np.ndarray           # int32 [*] physical blocks shared by several sequences
    tok_k: torch.Tensor                 # bf16 [T_all][Hkv][D]: every token of every sequence
    tok_v: torch.Tensor
    tok_offsets: np.ndarray             # int64 [S+1] row offsets of each sequence in tok_k/tok_v
    q_decode: torch.Tensor              # bf16 [num_decode][Hq][D]
    q_prefill: torch.Tensor             # bf16 [sum new_lens of chunks][Hq][D]
    k_scale: Optional[torch.Tensor] = None   # fp32 [Hkv] (one-byte caches only)
    v_scale: Optional[torch.Tensor] = None
    split_tokens: int = 0
    info: dict = field(default_factory=dict)

    # ------------------------------------------------------------------ derived views
    @property
    def num_seqs(self) -> int:
        return int(self.hist_lens.shape[0])

    @property
    def context_lens(self) -> np.ndarray:
        return (self.hist_lens + self.new_lens).astype(np.int32)

    @property
    def max_blocks_per_seq(self) -> int:
        return int(self.block_tables.shape[1])

    @property
    def decode_tables(self) -> np.ndarray:
        return np.ascontiguousarray(self.block_tables[: self.num_decode])

    @property
    def prefill_tables(self) -> np.ndarray:
        return np.ascontiguousarray(self.block_tables[self.num_decode:])

    @property
    def cu_q_lens(self) -> np.ndarray:
        c = self.new_lens[self.num_decode:].astype(np.int64)
        return np.concatenate([[0], np.cumsum(c)]).astype(np.int32)

    def step_rows(self) -> np.ndarray:
        """Row indices (into tok_k/tok_v) of the tokens appended by the step, in step order."""
        rows = []
        for s in range(self.num_seqs):
            lo = self.tok_offsets[s] + self.hist_lens[s]
            rows.append(np.arange(lo, lo + self.new_lens[s], dtype=np.int64))
        return np.concatenate(rows) if rows else np.zeros(0, np.int64)

    def seq_rows(self, s: int) -> np.ndarray:
        return np.arange(self.tok_offsets[s], self.tok_offsets[s + 1], dtype=np.int64)

    def to(self, device) -> "PagedBatch":
        d = dict(self.__dict__)
        for k in ("tok_k", "tok_v", "q_decode", "q_prefill", "k_scale", "v_scale"):
            if d[k] is not None:
                d[k] = d[k].to(device)
        return PagedBatch(**d)


# ---------------------------------------------------------------------- lengths

def _draw_hist(spec, n, rng: np.random.Generator) -> np.ndarray:
    kind = spec[0]
    if kind == "fixed":
        return np.array(spec[1], dtype=np.int32)
    if kind == "uniform":
        return rng.integers(spec[1], spec[2] + 1, size=n).astype(np.int32)
    if kind == "lognormal":
        median, sigma, lo, hi = spec[1:]
        x = np.rint(rng.lognormal(math.log(median), sigma, size=n))
        return np.clip(x, lo, hi).astype(np.int32)
    raise ValueError(kind)


class _Pool:
    """Seeded placement of logical blocks: blocks are handed out in the order of a
    random permutation of the pool (a FIFO free list after shuffling)."""

    def __init__(self, num_blocks: int, rng: Optional[np.random.Generator]):
        # rng None: identity placement (logical order == physical order, a contiguous layout)
        self.order = (np.arange(num_blocks) if rng is None else rng.permutation(num_blocks)).astype(np.int32)
        self.next = 0

    def take(self, n: int) -> np.ndarray:
        if self.next + n > self.order.shape[0]:
            raise ValueError("physical block pool exhausted")
        out = self.order[self.next:self.next + n]
        self.next += n
        return out


def _nblk(n, bs=BLOCK) -> int:
    return (int(n) + bs - 1) // bs


# ---------------------------------------------------------------------- builder

def make_batch(name: str, *, seed: Optional[int] = None, device="cpu", perm_seed: Optional[int] = None,
               overrides: Optional[dict] = None) -> PagedBatch:
    """Build workload ``name`` (a key of WORKLOADS), optionally with fields overridden.

    ``perm_seed`` changes only the physical placement of blocks (the logical data
    stays the same), which is how block-table invariance is tested; ``perm_seed=-1``
    places blocks in allocation order (each sequence's blocks contiguous).
    """
    spec = dict(WORKLOADS[name])
    if overrides:
        spec.update(overrides)
    seed = WORKLOAD_SEED.get(name, 1000) if seed is None else seed
    rng = np.random.default_rng([seed, 0])
    prng = None if perm_seed == -1 else np.random.default_rng([seed if perm_seed is None else perm_seed, 1])

    bs = int(spec.get("block_size", BLOCK))
    if bs not in (16, 32):
        raise ValueError("block_size must be 16 or 32")
    B = int(spec["num_seqs"])
    hq, hkv, D = int(spec["num_q_heads"]), int(spec["num_kv_heads"]), int(spec["head_dim"])
    hist_dec = _draw_hist(spec["hist"], B, rng)
    if hist_dec.shape[0] != B:
        raise ValueError("fixed length list does not match num_seqs")

    n_chunks = int(spec.get("prefill_chunks", 0))
    if n_chunks:
        clo, chi = spec["chunk_len"]
        hlo, hhi = spec["chunk_hist"]
        c_len = rng.integers(clo, chi + 1, size=n_chunks).astype(np.int32)
        c_hist = np.concatenate([[0], rng.integers(hlo, hhi + 1, size=n_chunks - 1)]).astype(np.int32)
    else:
        c_len = np.zeros(0, np.int32)
        c_hist = np.zeros(0, np.int32)

    hist = np.concatenate([hist_dec, c_hist]).astype(np.int32)
    new = np.concatenate([np.ones(B, np.int32), c_len]).astype(np.int32)
    S = B + n_chunks
    ctx = hist + new

    group = int(spec.get("share_group", 0))
    prefix = int(spec.get("share_prefix", 0))

    # ---- block placement ------------------------------------------------------
    # shared prefix blocks per group: enough to cover the longest member's share
    need_private = []
    shared_cover = np.zeros(S, np.int64)      # tokens of seq s living in its group's shared blocks
    if group:
        for s in range(B):
            shared_cover[s] = min(int(hist[s]), prefix)
    n_groups = (B + group - 1) // group if group else 0
    group_blocks_needed = []
    for gi in range(n_groups):
        mem = range(gi * group, min(B, (gi + 1) * group))
        group_blocks_needed.append(max(_nblk(shared_cover[s], bs) for s in mem))
    for s in range(S):
        # private blocks: logical blocks not covered by the shared prefix, plus one spare
        # for a copy-on-write fork of the last shared block
        nb_total = _nblk(ctx[s], bs)
        nb_shared = _nblk(shared_cover[s], bs)
        need_private.append(nb_total - nb_shared + (1 if nb_shared else 0))
    need = sum(group_blocks_needed) + sum(need_private)
    num_blocks = int(spec.get("num_blocks") or math.ceil(1.25 * need))
    if num_blocks < need:
        raise ValueError("pool smaller than the workload needs")
    pool = _Pool(num_blocks, prng)

    mbs = max(_nblk(c, bs) for c in ctx) if S else 1
    tables = np.full((S, mbs), -1, np.int32)
    group_blocks = [pool.take(n) for n in group_blocks_needed]
    refcount: Dict[int, int] = {}
    for s in range(S):
        nb_shared = _nblk(shared_cover[s], bs)
        if nb_shared:
            gb = group_blocks[s // group]
            tables[s, :nb_shared] = gb[:nb_shared]
            for b in gb[:nb_shared]:
                refcount[int(b)] = refcount.get(int(b), 0) + 1
        nb_hist = _nblk(hist[s], bs)
        if nb_hist > nb_shared:
            tables[s, nb_shared:nb_hist] = pool.take(nb_hist - nb_shared)
    shared_blocks = np.array(sorted(b for b, c in refcount.items() if c > 1), np.int32)

    # ---- the step: forks (copy-on-write) then new blocks for appended tokens ----
    pairs: List[List[int]] = []
    for s in range(S):
        for t in range(int(hist[s]), int(ctx[s])):
            lb = t // bs
            if tables[s, lb] < 0:
                tables[s, lb] = pool.take(1)[0]
                refcount[int(tables[s, lb])] = 1
                continue
            blk = int(tables[s, lb])
            if refcount.get(blk, 1) > 1:
                # the page is shared: write into a copy instead (copy-on-write)
                dst = int(pool.take(1)[0])
                pairs.append([blk, dst])
                refcount[blk] -= 1
                refcount[dst] = 1
                tables[s, lb] = dst
    cow_pairs = np.array(pairs, np.int32).reshape(-1, 2)

    # ---- token data ---------------------------------------------------------------
    offsets = np.concatenate([[0], np.cumsum(ctx.astype(np.int64))]).astype(np.int64)
    T_all = int(offsets[-1])
    tok_k = torch.empty((T_all, hkv, D), dtype=torch.bfloat16, device=device)
    tok_v = torch.empty((T_all, hkv, D), dtype=torch.bfloat16, device=device)
    group_data = {}
    for s in range(S):
        lo = int(offsets[s])
        n_sh = int(shared_cover[s])
        if n_sh:
            gi = s // group
            if gi not in group_data:
                n_g = max(int(shared_cover[m]) for m in range(gi * group, min(B, (gi + 1) * group)))
                group_data[gi] = (randn_bf16((n_g, hkv, D), device, seed, 2, gi),
                                  randn_bf16((n_g, hkv, D), device, seed, 3, gi))
            gk, gv = group_data[gi]
            tok_k[lo:lo + n_sh] = gk[:n_sh]
            tok_v[lo:lo + n_sh] = gv[:n_sh]
        n_own = int(ctx[s]) - n_sh
        tok_k[lo + n_sh:lo + n_sh + n_own] = randn_bf16((n_own, hkv, D), device, seed, 4, s)
        tok_v[lo + n_sh:lo + n_sh + n_own] = randn_bf16((n_own, hkv, D), device, seed, 5, s)

    # ---- slots ----------------------------------------------------------------------
    setup_slots = np.full(T_all, -1, np.int64)
    written = set()
    # history tokens are written through the tables as they were before the step's forks
    pre_tables = tables.copy()
    for (src, dst) in pairs:
        pre_tables[pre_tables == dst] = src
    for s in range(S):
        t = np.arange(int(hist[s]), dtype=np.int64)
        phys = pre_tables[s, t // bs].astype(np.int64)
        slots = phys * bs + t % bs
        if shared_cover[s]:
            # shared-prefix tokens are written once, by the first member that covers them
            keep = np.array([int(x) not in written for x in slots], dtype=bool)
            written.update(int(x) for x in slots[t < shared_cover[s]])
            slots = np.where(keep, slots, -1)
        setup_slots[offsets[s]:offsets[s] + hist[s]] = slots
    step_slots = []
    for s in range(S):
        t = np.arange(int(hist[s]), int(ctx[s]), dtype=np.int64)
        step_slots.append(tables[s, t // bs].astype(np.int64) * bs + t % bs)
    step_slots = np.concatenate(step_slots) if step_slots else np.zeros(0, np.int64)

    q_dec = randn_bf16((B, hq, D), device, seed, 6)
    q_pre = randn_bf16((int(c_len.sum()), hq, D), device, seed, 7)

    kv_dtype = {"fp8": 1, "int8": 2}.get(spec.get("kv_dtype"), 0)
    k_scale = v_scale = None
    if kv_dtype:
        # one fp32 scale per KV head (and per K/V tensor): absmax of the seeded data / largest code
        top = E4M3_MAX if kv_dtype == 1 else INT8_MAX
        # (abs and max are exact in bf16, so the absmax is taken before widening to fp32)
        k_scale = (tok_k.abs().amax(dim=(0, 2)).float() / top).to(torch.float32)
        v_scale = (tok_v.abs().amax(dim=(0, 2)).float() / top).to(torch.float32)

    return PagedBatch(
        name=name, num_q_heads=hq, num_kv_heads=hkv, head_dim=D, num_blocks=num_blocks,
        scale=1.0 / math.sqrt(D), kv_dtype=kv_dtype, block_size=bs, num_decode=B,
        hist_lens=hist, new_lens=new, block_tables=tables, setup_slots=setup_slots,
        step_slots=step_slots, cow_pairs=cow_pairs, shared_blocks=shared_blocks,
        tok_k=tok_k, tok_v=tok_v, tok_offsets=offsets, q_decode=q_dec, q_prefill=q_pre,
        k_scale=k_scale, v_scale=v_scale, split_tokens=int(spec.get("split_tokens", 0)),
        info=dict(seed=seed, perm_seed=perm_seed, groups=n_groups),
    )


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> NumPy uint16 bit patterns (host copy)."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def decode_kv_bytes(ctx_lens, num_kv_heads, head_dim, elem_bytes) -> int:
    """Bytes of K and V a decode step must read: every cached token of every sequence,
    for every KV head, K and V."""
    return int(np.sum(np.asarray(ctx_lens, np.int64))) * 2 * num_kv_heads * head_dim * elem_bytes
