"""Pins of the CPU oracle to things other than itself (CPU only).

- values the pages print (KV-size formula and its worked example) and the OCP E4M3
  definition (tests/golden/*.json, each with its citation);
- library routines the method reduces to in special cases: torch's fp64
  scaled_dot_product_attention on contiguous K/V (no paging), and torch's float8_e4m3fn cast;
- closed forms: one-token context returns V exactly; identical keys or a zero query return the
  mean of V;
- invariants of paging: physical placement does not change any result; reading a sequence back
  through its block table returns exactly its tokens; copy-on-write leaves every other
  sequence's view of the cache unchanged.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from pagedattention_block_table_b200.inputs import make_batch, bf16_bits
from tests.common import oracle_step

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _bf16_to_f64(bits):
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


# ----------------------------------------------------------------------------- KV size formula

def test_kv_cache_bytes_pages_example(O):
    g = _golden("kv_cache_sizes.json")
    for c in g["cases"]:
        got = O.kv_cache_bytes(c["layers"], c["kv_heads"], c["head_dim"], c["seq_len"], c["batch"], c["elem_bytes"])
        assert got == c["bytes"], c
    a = O.kv_cache_bytes(32, 8, 128, 32768, 1, 2)
    b = O.kv_cache_bytes(32, 8, 128, 4096, 1, 2)
    assert a == g["ratios"][0]["ratio"] * b


def test_kv_cache_bytes_matches_a_built_pool(O):
    """A paged pool holding one 4096-token sequence for 32 layers (256 blocks of 16 per layer, K and V,
    8 heads, 128 dims, 2 bytes) occupies exactly the page's 536,870,912 bytes."""
    blocks_per_layer = 4096 // 16
    one_pool = np.zeros((blocks_per_layer, 8, 16, 128), np.uint16)
    assert 32 * 2 * one_pool.nbytes == O.kv_cache_bytes(32, 8, 128, 4096, 1, 2) == 536870912


# ----------------------------------------------------------------------------- E4M3

def test_e4m3_decode_spec_points(O):
    g = _golden("e4m3_points.json")
    for p in g["decode"]:
        v = O.e4m3_decode([p["code"]])[0]
        assert v == p["value"] and math.copysign(1, v) == math.copysign(1, p["value"]), p
    for c in g["nan_codes"]:
        assert np.isnan(O.e4m3_decode([c])[0])


def test_e4m3_encode_spec_points(O):
    g = _golden("e4m3_points.json")
    for p in g["encode"]:
        assert int(O.e4m3_encode([p["x"]])[0]) == p["code"], p


def test_e4m3_decode_matches_torch(O):
    codes = np.arange(256, dtype=np.uint8)
    mine = O.e4m3_decode(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    finite = ~np.isnan(ref)
    assert np.array_equal(np.isnan(mine), ~finite)
    assert np.array_equal(mine[finite], ref[finite])


def test_e4m3_encode_matches_torch_cast(O):
    """torch's float8_e4m3fn cast rounds to nearest even; clamped to +-448 first it equals the
    saturating encoder.  Inputs: every finite bf16 magnitude in range, divided by a few scales
    (the quotients an FP8 append forms), plus all code midpoints (ties)."""
    bits = np.arange(0, 0x7F80, 7, dtype=np.uint32)
    xs = [(bits << 16).view(np.float32)]
    with np.errstate(over="ignore"):
        for s in (0.0123, 0.5, 1.0 / 448 * 3.7):
            xs.append((xs[0] / np.float32(s)).astype(np.float32))
    vals = O.e4m3_decode(np.arange(0, 0x7F, dtype=np.uint8))
    mids = ((vals[:-1] + vals[1:]) / 2).astype(np.float32)
    x = np.concatenate(xs + [mids, -mids])
    x = x[np.isfinite(x)]
    x = x[::3]
    mine = O.e4m3_encode(x)
    ref = torch.from_numpy(np.clip(x, -448.0, 448.0)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(mine, ref)


def test_e4m3_roundtrip_all_codes(O):
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    vals = O.e4m3_decode(codes).astype(np.float32)
    back = O.e4m3_encode(vals)
    assert np.array_equal(back, codes)


# ----------------------------------------------------------------------------- attention vs library

def _sdpa_decode_reference(batch):
    """Decode attention of every sequence from its token rows (contiguous, never paged), by torch SDPA in fp64."""
    g = batch.num_q_heads // batch.num_kv_heads
    outs = []
    ctx = batch.context_lens
    for s in range(batch.num_decode):
        rows = batch.seq_rows(s)[: ctx[s]]
        k = batch.tok_k[rows].double().permute(1, 0, 2).repeat_interleave(g, 0)  # [Hq][L][D]
        v = batch.tok_v[rows].double().permute(1, 0, 2).repeat_interleave(g, 0)
        q = batch.q_decode[s].double()[:, None, :]                              # [Hq][1][D]
        o = torch.nn.functional.scaled_dot_product_attention(q[None], k[None], v[None], scale=batch.scale)
        outs.append(o[0, :, 0, :].numpy())
    return np.stack(outs)


@pytest.mark.parametrize("hq,hkv,d,bs", [(8, 2, 64, 16), (4, 1, 128, 16), (6, 6, 64, 16), (8, 2, 64, 32)])
def test_decode_matches_sdpa_on_unpaged_kv(O, hq, hkv, d, bs):
    batch = make_batch("tiny_decode", seed=7, overrides=dict(num_q_heads=hq, num_kv_heads=hkv, head_dim=d,
                                                          num_seqs=5, hist=("fixed", [0, 15, 16, 47, 130]),
                                                          num_blocks=40, block_size=bs))
    res = oracle_step(batch, O)
    ref = _sdpa_decode_reference(batch)
    np.testing.assert_allclose(res["decode"], ref, rtol=0, atol=1e-12)


def test_prefill_matches_sdpa_with_causal_offset(O):
    batch = make_batch("mixed_step", seed=11, overrides=dict(
        num_seqs=2, hist=("fixed", [20, 9]), share_group=0, share_prefix=0, num_q_heads=4, num_kv_heads=2,
        head_dim=64, prefill_chunks=3, chunk_len=(5, 37), chunk_hist=(1, 50)))
    res = oracle_step(batch, O)
    g = batch.num_q_heads // batch.num_kv_heads
    cu = batch.cu_q_lens
    ctx = batch.context_lens
    for c in range(batch.num_seqs - batch.num_decode):
        s = batch.num_decode + c
        C = int(batch.new_lens[s])
        H = int(ctx[s]) - C
        rows = batch.seq_rows(s)[: ctx[s]]
        k = batch.tok_k[rows].double().permute(1, 0, 2).repeat_interleave(g, 0)
        v = batch.tok_v[rows].double().permute(1, 0, 2).repeat_interleave(g, 0)
        q = batch.q_prefill[cu[c]:cu[c + 1]].double().permute(1, 0, 2)           # [Hq][C][D]
        mask = torch.arange(H + C)[None, :] <= (H + torch.arange(C))[:, None]   # key t visible to row i
        o = torch.nn.functional.scaled_dot_product_attention(q[None], k[None], v[None], attn_mask=mask,
                                                             scale=batch.scale)
        np.testing.assert_allclose(res["prefill"][cu[c]:cu[c + 1]], o[0].permute(1, 0, 2).numpy(), atol=1e-12, rtol=0)


# ----------------------------------------------------------------------------- closed forms

def _one_seq_cache(k_rows, v_rows, perm):
    """Cache holding one sequence whose logical block i sits in physical block perm[i]."""
    L, hkv, d = k_rows.shape
    nb = len(perm)
    kc = np.zeros((nb, hkv, 16, d), np.uint16)
    vc = np.zeros((nb, hkv, 16, d), np.uint16)
    for t in range(L):
        kc[perm[t // 16], :, t % 16] = k_rows[t]
        vc[perm[t // 16], :, t % 16] = v_rows[t]
    return kc, vc


def test_context_of_one_returns_v(O):
    rng = np.random.default_rng(3)
    k = bf16_bits(torch.randn(1, 2, 64).to(torch.bfloat16))
    v = bf16_bits(torch.randn(1, 2, 64).to(torch.bfloat16))
    q = bf16_bits(torch.randn(1, 8, 64).to(torch.bfloat16))
    kc, vc = _one_seq_cache(k, v, [3, 0, 1, 2])
    out = O.paged_decode(q, kc, vc, np.array([[3, 0, 1, 2]], np.int32), np.array([1], np.int32), 0.125)
    for h in range(8):
        assert np.array_equal(out[0, h], _bf16_to_f64(v[0, h // 4])), h
    del rng


@pytest.mark.parametrize("zero_q", [False, True])
def test_identical_keys_or_zero_query_give_mean_of_v(O, zero_q):
    L = 37
    k1 = bf16_bits(torch.randn(1, 1, 128).to(torch.bfloat16))
    k = np.repeat(k1, L, axis=0) if not zero_q else bf16_bits(torch.randn(L, 1, 128).to(torch.bfloat16))
    v = bf16_bits(torch.randn(L, 1, 128).to(torch.bfloat16))
    q = bf16_bits(torch.randn(1, 4, 128).to(torch.bfloat16))
    if zero_q:
        q[:] = 0
    perm = [5, 2, 0, 4, 1, 3]
    kc, vc = _one_seq_cache(k, v, perm)
    out = O.paged_decode(q, kc, vc, np.array([perm], np.int32), np.array([L], np.int32), 1 / math.sqrt(128))
    mean_v = _bf16_to_f64(v[:, 0]).mean(axis=0)
    for h in range(4):
        np.testing.assert_allclose(out[0, h], mean_v, atol=1e-13, rtol=0)


# ----------------------------------------------------------------------------- paging invariants

def test_physical_placement_does_not_change_results(O):
    kw = dict(seed=21, overrides=dict(num_seqs=6, hist=("uniform", 1, 90), num_blocks=None))
    a = oracle_step(make_batch("tiny_decode", perm_seed=1, **kw), O)
    b = oracle_step(make_batch("tiny_decode", perm_seed=2, **kw), O)
    c = oracle_step(make_batch("tiny_decode", perm_seed=-1, **kw), O)
    assert np.array_equal(a["decode"], b["decode"]) and np.array_equal(a["decode"], c["decode"])


@pytest.mark.parametrize("bs", [16, 32])
def test_tables_read_back_each_sequences_tokens(O, bs):
    """After set-up, forks and append, each sequence read through its table is exactly its tokens."""
    batch = make_batch("mixed_step", seed=5, overrides=dict(
        num_seqs=24, hist=("lognormal", 40.0, 1.0, 1, 200), share_group=8, share_prefix=64,
        prefill_chunks=2, chunk_len=(3, 40), chunk_hist=(1, 60), num_q_heads=4, num_kv_heads=2, head_dim=64,
        block_size=bs))
    assert batch.cow_pairs.shape[0] > 0, "workload must exercise copy-on-write"
    res = oracle_step(batch, O, keep_pre_step=True)
    kc, vc = res["k_cache"], res["v_cache"]
    tk, tv = bf16_bits(batch.tok_k), bf16_bits(batch.tok_v)
    ctx = batch.context_lens
    B = batch.block_size
    for s in range(batch.num_seqs):
        t = np.arange(ctx[s])
        phys = batch.block_tables[s, t // B]
        assert np.all(phys >= 0)
        got_k = kc[phys, :, t % B]
        got_v = vc[phys, :, t % B]
        rows = batch.seq_rows(s)[: ctx[s]]
        assert np.array_equal(got_k, tk[rows]) and np.array_equal(got_v, tv[rows]), s


def test_copy_on_write_copies_and_keeps_parent(O):
    batch = make_batch("mixed_step", seed=9, overrides=dict(
        num_seqs=16, hist=("uniform", 1, 60), share_group=8, share_prefix=48,
        prefill_chunks=0, num_q_heads=4, num_kv_heads=2, head_dim=64))
    assert batch.cow_pairs.shape[0] > 0
    res = oracle_step(batch, O, keep_pre_step=True)
    for src, dst in batch.cow_pairs:
        assert np.array_equal(res["k_forked"][dst], res["k_pre"][src])
        assert np.array_equal(res["v_forked"][dst], res["v_pre"][src])
        assert np.array_equal(res["k_forked"][src], res["k_pre"][src])
    # a forked block's parent is written only by its last holder's own appended token
    appended = set(int(x) // 16 for x in batch.step_slots)
    for src, _ in batch.cow_pairs:
        diff = np.argwhere(np.any(res["k_cache"][src] != res["k_pre"][src], axis=-1))
        if diff.size:
            assert int(src) in appended


def test_prefill_of_one_token_equals_decode(O):
    rng = np.random.default_rng(4)
    L = 53
    k = bf16_bits(torch.randn(L, 2, 64).to(torch.bfloat16))
    v = bf16_bits(torch.randn(L, 2, 64).to(torch.bfloat16))
    perm = list(rng.permutation(6))
    kc, vc = _one_seq_cache(k, v, perm)
    q = bf16_bits(torch.randn(1, 8, 64).to(torch.bfloat16))
    tbl = np.array([perm], np.int32)
    dec = O.paged_decode(q, kc, vc, tbl, np.array([L], np.int32), 0.125)
    pre = O.paged_prefill(q, np.array([0, 1], np.int32), kc, vc, tbl, np.array([L], np.int32), 0.125)
    assert np.array_equal(dec, pre)


def test_prefill_last_row_equals_decode_over_whole_context(O):
    rng = np.random.default_rng(8)
    L, C = 70, 19
    k = bf16_bits(torch.randn(L, 1, 64).to(torch.bfloat16))
    v = bf16_bits(torch.randn(L, 1, 64).to(torch.bfloat16))
    perm = list(rng.permutation(5))
    kc, vc = _one_seq_cache(k, v, perm)
    q = bf16_bits(torch.randn(C, 2, 64).to(torch.bfloat16))
    tbl = np.array([perm], np.int32)
    pre = O.paged_prefill(q, np.array([0, C], np.int32), kc, vc, tbl, np.array([L], np.int32), 0.125)
    for i in range(C):
        dec = O.paged_decode(q[i:i + 1], kc, vc, tbl, np.array([L - C + i + 1], np.int32), 0.125)
        assert np.array_equal(pre[i], dec[0]), i


def test_fp8_append_codes_follow_quotient_rule(O):
    """FP8 append stores E4M3(x / scale) of each element; reading it back through the table and
    multiplying by the scale stays within half an E4M3 step of x."""
    batch = make_batch("mha_fp8_decode", seed=2, overrides=dict(num_seqs=3, num_q_heads=2, num_kv_heads=2,
                                                              hist=("fixed", [5, 17, 40])))
    res = oracle_step(batch, O)
    ks = batch.k_scale.numpy().astype(np.float64)
    tk = _bf16_to_f64(bf16_bits(batch.tok_k))
    ctx = batch.context_lens
    for s in range(batch.num_seqs):
        t = np.arange(ctx[s])
        phys = batch.block_tables[s, t // 16]
        codes = res["k_cache"][phys, :, t % 16]                  # [L][Hkv][D]
        deq = O.e4m3_decode(codes) * ks[None, :, None]
        x = tk[batch.seq_rows(s)[: ctx[s]]]
        # relative half-step of a 3-bit mantissa (1/16), or half the smallest subnormal step
        bound = np.maximum(np.abs(x) / 16, 2.0 ** -10 * ks[None, :, None]) * (1 + 1e-6)
        assert np.all(np.abs(deq - x) <= bound)


# ----------------------------------------------------------------------------- INT8

def test_int8_encode_points(O):
    g = _golden("int8_points.json")
    for p in g["encode"]:
        assert int(O.int8_encode([p["x"]])[0]) == p["code"], p


def test_int8_encode_matches_numpy(O):
    """numpy's rint rounds half to even; clipped to +-127 it is the symmetric INT8 encoder."""
    rng = np.random.default_rng(1)
    x = np.concatenate([rng.normal(0, 60, 20000), np.arange(-130, 130, 0.5)]).astype(np.float32)
    ref = np.clip(np.rint(x), -127, 127).astype(np.int8)
    assert np.array_equal(O.int8_encode(x), ref)


def test_int8_append_and_decode_read_back(O):
    """INT8 append stores round(x/scale); decode of a one-token context returns code * scale exactly."""
    k = bf16_bits(torch.randn(1, 1, 64).to(torch.bfloat16))
    v = bf16_bits(torch.randn(1, 1, 64).to(torch.bfloat16))
    sc = np.array([0.02], np.float32)
    kc = np.zeros((2, 1, 16, 64), np.int8)
    vc = np.zeros_like(kc)
    O.kv_append(kc, vc, k, v, np.array([17], np.int64), 2, sc, sc)
    xv = _bf16_to_f64(v[0, 0]).astype(np.float32)
    codes = np.clip(np.rint(xv / np.float32(0.02)), -127, 127)
    assert np.array_equal(vc[1, 0, 1], codes.astype(np.int8))
    q = bf16_bits(torch.randn(1, 2, 64).to(torch.bfloat16))
    # the token sits at slot 17 = block 1, offset 1; a table whose block 0 is physical block 1 and a
    # context of 2 reads (zero row, token)
    out = O.paged_decode(q, kc, vc, np.array([[1]], np.int32), np.array([2], np.int32), 0.125, 2, sc, sc)
    assert np.all(np.isfinite(out))
    # the two-token result is a convex combination of the two dequantised rows
    rows = np.stack([vc[1, 0, 0].astype(np.float64), vc[1, 0, 1].astype(np.float64)]) * np.float64(np.float32(0.02))
    lo, hi = rows.min(axis=0) - 1e-12, rows.max(axis=0) + 1e-12
    assert np.all((out[0] >= lo) & (out[0] <= hi))


# ----------------------------------------------------------------------------- one-byte caches: dequantisation

def _dequant_reference(codes, kv_dtype, scale):
    """Values of one-byte cache codes [..][Hkv][bs][D] with one scale per KV head, from the library
    routines: torch's float8_e4m3fn reinterpretation (FP8) or the integer itself (INT8), times the scale."""
    c = torch.from_numpy(np.ascontiguousarray(codes))
    v = c.view(torch.float8_e4m3fn).to(torch.float64) if kv_dtype == 1 else c.to(torch.float64)
    return v * torch.from_numpy(np.asarray(scale, np.float32)).to(torch.float64)[None, :, None, None]


def _one_byte_case(kv_dtype, bs, seed):
    """A shuffled pool of random one-byte codes (no NaN codes), two KV heads with four different scales."""
    rng = np.random.default_rng(seed)
    nb, hkv, d = 24, 2, 64
    if kv_dtype == 1:
        codes = rng.integers(0, 256, size=(2, nb, hkv, bs, d)).astype(np.uint8)
        codes[(codes & 0x7F) == 0x7F] = 0x3C                 # the NaN codes never come out of the encoder
    else:
        codes = rng.integers(-127, 128, size=(2, nb, hkv, bs, d)).astype(np.int8)
    k_scale = np.array([0.013, 0.041], np.float32)             # every scale different: K vs V and per head
    v_scale = np.array([0.37, 0.0029], np.float32)
    return codes[0], codes[1], k_scale, v_scale, rng


def _gather(pool, table, L, bs):
    """Rows 0..L-1 of one sequence, [Hkv][L][D], read from a [NB][Hkv][bs][D] tensor through its table."""
    t = torch.arange(L)
    return pool[torch.from_numpy(table.astype(np.int64))[t // bs], :, t % bs].permute(1, 0, 2)


@pytest.mark.parametrize("kv_dtype", [1, 2])
@pytest.mark.parametrize("bs", [16, 32])
def test_one_byte_decode_matches_sdpa_on_dequantised_kv(O, kv_dtype, bs):
    """Decode over an FP8 / INT8 cache equals torch fp64 SDPA on code * scale, with K and V dequantised by
    their own per-head scales (KV Cache to vLLM §2.2: one byte per element with a scale)."""
    kc, vc, ks, vs, rng = _one_byte_case(kv_dtype, bs, 31 + kv_dtype)
    hq, hkv, d = 6, 2, 64
    kf, vf = _dequant_reference(kc, kv_dtype, ks), _dequant_reference(vc, kv_dtype, vs)
    lens = np.array([1, 29, bs * 3, 150], np.int32)
    mbs = (int(lens.max()) + bs - 1) // bs
    tables = np.stack([rng.permutation(kc.shape[0])[:mbs] for _ in lens]).astype(np.int32)
    q = bf16_bits(torch.randn(len(lens), hq, d, generator=torch.Generator().manual_seed(5)).to(torch.bfloat16))
    got = O.paged_decode(q, kc, vc, tables, lens, 0.125, kv_dtype, ks, vs)
    qf = torch.from_numpy(_bf16_to_f64(q))
    for b, L in enumerate(lens):
        k = _gather(kf, tables[b], int(L), bs).repeat_interleave(hq // hkv, 0)
        v = _gather(vf, tables[b], int(L), bs).repeat_interleave(hq // hkv, 0)
        ref = torch.nn.functional.scaled_dot_product_attention(qf[b][None, :, None, :], k[None], v[None], scale=0.125)
        np.testing.assert_allclose(got[b], ref[0, :, 0].numpy(), atol=1e-12, rtol=1e-12)


@pytest.mark.parametrize("kv_dtype", [1, 2])
def test_one_byte_prefill_matches_sdpa_on_dequantised_kv(O, kv_dtype):
    """Causal chunks over an FP8 / INT8 cache equal torch fp64 SDPA (causal offset mask) on code * scale."""
    bs = 16
    kc, vc, ks, vs, rng = _one_byte_case(kv_dtype, bs, 41 + kv_dtype)
    hq, hkv, d = 4, 2, 64
    kf, vf = _dequant_reference(kc, kv_dtype, ks), _dequant_reference(vc, kv_dtype, vs)
    C = np.array([7, 19], np.int32)
    ctx = np.array([7, 60], np.int32)                          # chunk 0 starts a request, chunk 1 has H = 41
    cu = np.concatenate([[0], np.cumsum(C)]).astype(np.int32)
    mbs = (int(ctx.max()) + bs - 1) // bs
    tables = np.stack([rng.permutation(kc.shape[0])[:mbs] for _ in C]).astype(np.int32)
    q = bf16_bits(torch.randn(int(cu[-1]), hq, d, generator=torch.Generator().manual_seed(6)).to(torch.bfloat16))
    got = O.paged_prefill(q, cu, kc, vc, tables, ctx, 0.1, kv_dtype, ks, vs)
    qf = torch.from_numpy(_bf16_to_f64(q))
    for c in range(len(C)):
        L, H = int(ctx[c]), int(ctx[c] - C[c])
        k = _gather(kf, tables[c], L, bs).repeat_interleave(hq // hkv, 0)
        v = _gather(vf, tables[c], L, bs).repeat_interleave(hq // hkv, 0)
        mask = torch.arange(L)[None, :] <= (H + torch.arange(int(C[c])))[:, None]
        ref = torch.nn.functional.scaled_dot_product_attention(qf[cu[c]:cu[c + 1]].permute(1, 0, 2)[None], k[None],
                                                               v[None], attn_mask=mask, scale=0.1)
        np.testing.assert_allclose(got[cu[c]:cu[c + 1]], ref[0].permute(1, 0, 2).numpy(), atol=1e-12, rtol=1e-12)


# ----------------------------------------------------------------------------- swap

@pytest.mark.parametrize("dtype,bs", [(np.uint16, 16), (np.uint8, 32)])
def test_swap_reads_back_each_moved_block(O, dtype, bs):
    """After a swap (vLLM overview, section 三: KV pages move to CPU memory and back), block dst of the
    destination pool equals block src of the source pool, for K and for V separately; every other
    destination block and the whole source pool are unchanged."""
    rng = np.random.default_rng(17)
    hkv, d, nsrc, ndst = 2, 64, 30, 20
    hi = np.iinfo(dtype).max
    src_k, src_v = (rng.integers(0, hi, size=(nsrc, hkv, bs, d)).astype(dtype) for _ in range(2))
    dst_k, dst_v = (rng.integers(0, hi, size=(ndst, hkv, bs, d)).astype(dtype) for _ in range(2))
    pairs = np.stack([rng.permutation(nsrc)[:9], rng.permutation(ndst)[:9]], 1).astype(np.int32)
    before = [a.copy() for a in (src_k, src_v, dst_k, dst_v)]
    O.swap_blocks(dst_k, dst_v, src_k, src_v, pairs)
    assert np.array_equal(src_k, before[0]) and np.array_equal(src_v, before[1])
    for s, t in pairs:
        assert np.array_equal(dst_k[t], before[0][s]) and np.array_equal(dst_v[t], before[1][s])
    untouched = np.setdiff1d(np.arange(ndst), pairs[:, 1])
    assert np.array_equal(dst_k[untouched], before[2][untouched])
    assert np.array_equal(dst_v[untouched], before[3][untouched])
