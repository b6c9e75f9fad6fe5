"""KV-head sharding of a paged batch across ranks (tensor parallelism).

The KV Cache to vLLM page (§3.4, §4.4) splits a model over several GPUs with tensor parallelism,
which splits the weights and the KV cache.  For attention that means each rank holds the KV heads
[lo, hi) of every block -- its own [num_blocks][hi-lo][16][head_dim] pool -- and the query heads
that use them.  Attention needs no exchange between ranks: every (sequence, KV head) is
independent, so each rank calls pa_paged_attention on its shard and the per-head outputs are the
unsharded ones.  (The collective that follows in a model, the output projection's all-reduce,
sits outside this path.)  Block tables, lengths and slots are the same on every rank.
"""
from __future__ import annotations

import dataclasses

from .inputs import PagedBatch


def kv_head_range(rank: int, world: int, num_kv_heads: int):
    """KV heads [lo, hi) owned by `rank`.  num_kv_heads must be a multiple of world."""
    if world <= 0 or not 0 <= rank < world or num_kv_heads % world:
        raise ValueError("num_kv_heads must split evenly over the ranks")
    per = num_kv_heads // world
    return rank * per, (rank + 1) * per


def q_head_range(rank: int, world: int, num_q_heads: int, num_kv_heads: int):
    """Query heads [lo, hi) that use the rank's KV heads (contiguous GQA groups)."""
    lo, hi = kv_head_range(rank, world, num_kv_heads)
    g = num_q_heads // num_kv_heads
    return lo * g, hi * g


def shard_batch(batch: PagedBatch, rank: int, world: int) -> PagedBatch:
    """The part of `batch` rank `rank` holds: its KV heads of every token and block, its query heads."""
    klo, khi = kv_head_range(rank, world, batch.num_kv_heads)
    qlo, qhi = q_head_range(rank, world, batch.num_q_heads, batch.num_kv_heads)
    return dataclasses.replace(
        batch,
        num_q_heads=qhi - qlo,
        num_kv_heads=khi - klo,
        tok_k=batch.tok_k[:, klo:khi].contiguous(),
        tok_v=batch.tok_v[:, klo:khi].contiguous(),
        q_decode=batch.q_decode[:, qlo:qhi].contiguous(),
        q_prefill=batch.q_prefill[:, qlo:qhi].contiguous(),
        k_scale=None if batch.k_scale is None else batch.k_scale[klo:khi].contiguous(),
        v_scale=None if batch.v_scale is None else batch.v_scale[klo:khi].contiguous(),
        info=dict(batch.info, shard=(rank, world)),
    )
