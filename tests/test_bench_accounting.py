"""The roofline numerators bench.py reports, checked on the CPU.

- Prefill FLOPs (4 * D * Hq * keys attended, causal) against the per-chunk figures worked out from the
  Llama-3-8B shapes: C=512 from scratch is 2.15 GFLOP, C=2048 from scratch 34.4 GFLOP, and C=2048 over a
  4095-token history 171.8 GFLOP.
- Decode bytes: K and V of every context token once (4096 B per token at 8 KV heads x 128 dims x bf16,
  half that for a one-byte cache), plus q, out, table entries and lengths; checked against an
  element-by-element count over the block tables.
- Unique bytes under prefix sharing: the distinct physical slots the tables reach, by brute force.
"""
import math
from types import SimpleNamespace

import numpy as np
import pytest

import bench
from pagedattention_block_table_b200.inputs import make_batch


def _chunk_batch(C, H, hq=32, hkv=8, d=128):
    return SimpleNamespace(num_decode=0, num_seqs=1, new_lens=np.array([C]), context_lens=np.array([H + C]),
                           head_dim=d, num_q_heads=hq, num_kv_heads=hkv)


@pytest.mark.parametrize("C,H,gflop", [(512, 0, 2.15), (2048, 0, 34.4), (2048, 4095, 171.8)])
def test_prefill_flops_per_chunk(C, H, gflop):
    got = bench.prefill_flops(_chunk_batch(C, H))
    assert abs(got / 1e9 - gflop) < 0.05
    # brute force: row i of the chunk attends H + i + 1 keys; QK^T and PV are 2 * D flops per key each
    assert got == sum(4 * 128 * 32 * (H + i + 1) for i in range(C))


@pytest.mark.parametrize("kv", ["bf16", "fp8"])
def test_decode_bytes_count_every_element_once(kv):
    over = dict(num_seqs=5, hist=("fixed", [0, 15, 16, 300, 1000]))
    if kv == "fp8":
        over["kv_dtype"] = "fp8"
    b = make_batch("llama3_8b_decode", seed=3, overrides=over)
    e = 1 if kv == "fp8" else 2
    # element by element: every context token's K and V row of every KV head, through its table entry
    kvb = 0
    entries = 0
    for s in range(b.num_decode):
        L = int(b.context_lens[s])
        used = set()
        for t in range(L):
            used.add(int(b.block_tables[s, t // b.block_size]))
            kvb += 2 * b.num_kv_heads * b.head_dim * e
        entries += math.ceil(L / b.block_size)
        assert len(used) == math.ceil(L / b.block_size)          # distinct blocks of one sequence
    q_out = 2 * b.num_decode * b.num_q_heads * b.head_dim * 2
    assert bench.kv_bytes(b) == kvb
    assert bench.decode_bytes(b) == kvb + q_out + 4 * entries + 4 * b.num_decode
    if kv == "bf16":
        assert kvb == int(b.context_lens.sum()) * 4096            # 2 x 8 heads x 128 dims x 2 bytes


def test_unique_bytes_count_shared_prefix_slots_once():
    b = make_batch("mixed_step", seed=7, overrides=dict(num_seqs=16, share_group=8, share_prefix=1024,
                                                          prefill_chunks=0))
    slots = set()
    for s in range(b.num_decode):
        for t in range(int(b.context_lens[s])):
            slots.add(int(b.block_tables[s, t // b.block_size]) * b.block_size + t % b.block_size)
    per_slot = 2 * b.num_kv_heads * b.head_dim * 2
    assert bench.kv_unique_bytes(b) == len(slots) * per_slot
    assert bench.kv_unique_bytes(b) < bench.kv_bytes(b)          # the shared prefixes are read by several
