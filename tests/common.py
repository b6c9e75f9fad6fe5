"""Helpers shared by the tests: run a PagedBatch step through the CPU oracle, compare results."""
from __future__ import annotations

import numpy as np
import torch

from pagedattention_block_table_b200.inputs import PagedBatch, bf16_bits

ATOL_MAX = 1e-2      # attention max-abs error vs the oracle (bf16 inputs, bf16 output)
ATOL_MEAN = 1e-3     # attention mean-abs error vs the oracle
FP8_MAX = 5e-2       # fp8 cache, vs the oracle on the original bf16 K/V


def oracle_step(batch: PagedBatch, O, keep_pre_step=False):
    """Fill the history, then run the step (forks, append, decode, prefill) in the oracle."""
    nb, hkv, d = batch.num_blocks, batch.num_kv_heads, batch.head_dim
    dt = {0: np.uint16, 1: np.uint8, 2: np.int8}[batch.kv_dtype]
    kc = np.zeros((nb, hkv, batch.block_size, d), dt)
    vc = np.zeros((nb, hkv, batch.block_size, d), dt)
    tk = bf16_bits(batch.tok_k)
    tv = bf16_bits(batch.tok_v)
    ks = None if batch.k_scale is None else batch.k_scale.cpu().numpy()
    vs = None if batch.v_scale is None else batch.v_scale.cpu().numpy()
    O.kv_append(kc, vc, tk, tv, batch.setup_slots, batch.kv_dtype, ks, vs)
    res = {}
    if keep_pre_step:
        res["k_pre"], res["v_pre"] = kc.copy(), vc.copy()
    O.copy_blocks(kc, vc, batch.cow_pairs)
    if keep_pre_step:
        res["k_forked"], res["v_forked"] = kc.copy(), vc.copy()
    rows = batch.step_rows()
    O.kv_append(kc, vc, tk[rows], tv[rows], batch.step_slots, batch.kv_dtype, ks, vs)
    res["k_cache"], res["v_cache"] = kc, vc
    ctx = batch.context_lens
    nd = batch.num_decode
    if nd:
        res["decode"] = O.paged_decode(bf16_bits(batch.q_decode), kc, vc, batch.decode_tables, ctx[:nd],
                                       batch.scale, batch.kv_dtype, ks, vs)
    if batch.num_seqs > nd:
        res["prefill"] = O.paged_prefill(bf16_bits(batch.q_prefill), batch.cu_q_lens, kc, vc, batch.prefill_tables,
                                         ctx[nd:], batch.scale, batch.kv_dtype, ks, vs)
    return res


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def assert_close(got: np.ndarray, ref: np.ndarray, max_tol=ATOL_MAX, mean_tol=ATOL_MEAN, what=""):
    err = np.abs(got - ref)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    mx, mn = float(err.max()) if err.size else 0.0, float(err.mean()) if err.size else 0.0
    assert mx <= max_tol, f"{what}: max abs err {mx:.3e} > {max_tol:.1e}"
    if mean_tol is not None:
        assert mn <= mean_tol, f"{what}: mean abs err {mn:.3e} > {mean_tol:.1e}"
    return mx, mn


def oracle_decode_one(batch: PagedBatch, s: int, O, kv_dtype=None):
    """Oracle decode of sequence s alone (all query heads) from its token rows, in a fresh
    contiguous cache; used to check sampled outputs of full-size runs."""
    kv_dtype = batch.kv_dtype if kv_dtype is None else kv_dtype
    L = int(batch.context_lens[s])
    rows = torch.from_numpy(batch.seq_rows(s)[:L]).to(batch.tok_k.device)
    tk = bf16_bits(batch.tok_k.index_select(0, rows))
    tv = bf16_bits(batch.tok_v.index_select(0, rows))
    nblk = max(1, (L + 15) // 16)
    dt = {0: np.uint16, 1: np.uint8, 2: np.int8}[kv_dtype]
    kc = np.zeros((nblk, batch.num_kv_heads, 16, batch.head_dim), dt)
    vc = np.zeros_like(kc)
    ks = vs = None
    if kv_dtype:
        ks, vs = batch.k_scale.cpu().numpy(), batch.v_scale.cpu().numpy()
    O.kv_append(kc, vc, tk, tv, np.arange(L, dtype=np.int64), kv_dtype, ks, vs)
    q = bf16_bits(batch.q_decode[s:s + 1])
    return O.paged_decode(q, kc, vc, np.arange(nblk, dtype=np.int32)[None], np.array([L], np.int32), batch.scale,
                          kv_dtype, ks, vs)[0]


def oracle_attend_prefix(batch: PagedBatch, s: int, L: int, q_bits: np.ndarray, O):
    """Oracle attention of the given query rows (bf16 bits [n][Hq][D]) over the first L tokens of
    sequence s, from its token rows in a fresh contiguous cache (bf16)."""
    rows = torch.from_numpy(batch.seq_rows(s)[:L]).to(batch.tok_k.device)
    tk = bf16_bits(batch.tok_k.index_select(0, rows))
    tv = bf16_bits(batch.tok_v.index_select(0, rows))
    nblk = max(1, (L + 15) // 16)
    kc = np.zeros((nblk, batch.num_kv_heads, 16, batch.head_dim), np.uint16)
    vc = np.zeros_like(kc)
    O.kv_append(kc, vc, tk, tv, np.arange(L, dtype=np.int64))
    n = q_bits.shape[0]
    tables = np.tile(np.arange(nblk, dtype=np.int32)[None], (n, 1))
    return O.paged_decode(q_bits, kc, vc, tables, np.full(n, L, np.int32), batch.scale)


def oracle_decode_all(batch: PagedBatch, O, kv_dtype=None) -> np.ndarray:
    """Oracle decode of every decoding sequence, [num_decode][Hq][D] fp64, each from its own token rows in
    a fresh contiguous cache (the plain definition: no paging, no sharing, no forks)."""
    return np.stack([oracle_decode_one(batch, s, O, kv_dtype) for s in range(batch.num_decode)])


def oracle_prefill_all(batch: PagedBatch, O) -> np.ndarray:
    """Oracle causal attention of every prefill row, [sum C][Hq][D] fp64: chunk c's rows over its own
    token rows (history + chunk) in a fresh contiguous cache of the batch's element type."""
    cu = batch.cu_q_lens
    ctx = batch.context_lens
    kv_dtype = batch.kv_dtype
    dt = {0: np.uint16, 1: np.uint8, 2: np.int8}[kv_dtype]
    ks = vs = None
    if kv_dtype:
        ks, vs = batch.k_scale.cpu().numpy(), batch.v_scale.cpu().numpy()
    outs = []
    for c in range(batch.num_seqs - batch.num_decode):
        s = batch.num_decode + c
        L = int(ctx[s])
        rows = torch.from_numpy(batch.seq_rows(s)[:L]).to(batch.tok_k.device)
        tk = bf16_bits(batch.tok_k.index_select(0, rows))
        tv = bf16_bits(batch.tok_v.index_select(0, rows))
        nblk = max(1, (L + 15) // 16)
        kc = np.zeros((nblk, batch.num_kv_heads, 16, batch.head_dim), dt)
        vc = np.zeros_like(kc)
        O.kv_append(kc, vc, tk, tv, np.arange(L, dtype=np.int64), kv_dtype, ks, vs)
        C = int(cu[c + 1] - cu[c])
        q = bf16_bits(batch.q_prefill[int(cu[c]):int(cu[c + 1])])
        outs.append(O.paged_prefill(q, np.array([0, C], np.int32), kc, vc, np.arange(nblk, dtype=np.int32)[None],
                                    np.array([L], np.int32), batch.scale, kv_dtype, ks, vs))
    return np.concatenate(outs) if outs else np.zeros((0, batch.num_q_heads, batch.head_dim))
