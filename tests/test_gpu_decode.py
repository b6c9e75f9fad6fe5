"""GPU parity of paged decode attention (bf16 and FP8 caches, split-K) against the oracle."""
import numpy as np
import pytest
import torch

from pagedattention_block_table_b200.inputs import make_batch
from tests.common import ATOL_MAX, ATOL_MEAN, FP8_MAX, assert_close, oracle_decode_one, oracle_step, to_f64

pytestmark = pytest.mark.gpu


def _gpu_decode(batch, split_tokens=None):
    from pagedattention_block_table_b200.runner import DeviceStep
    st = DeviceStep(batch, split_tokens=split_tokens)
    st.fill_history()
    st.step()
    torch.cuda.synchronize()
    return st


SMALL = {
    # the tiny workload exactly as specified
    "tiny": ("tiny_decode", {}),
    # 8B shapes, ragged lengths spanning several tiles, splits and a ragged tail
    "gqa4_d128": ("llama3_8b_decode", dict(num_seqs=6, hist=("fixed", [0, 15, 16, 511, 1023, 1700]))),
    "gqa8_d128": ("llama3_8b_decode", dict(num_seqs=3, num_q_heads=64, num_kv_heads=8, hist=("uniform", 30, 900))),
    "gqa2_d64": ("tiny_decode", dict(num_seqs=5, num_q_heads=4, num_kv_heads=2, hist=("uniform", 1, 700),
                                     num_blocks=None)),
    "mha_d64": ("tiny_decode", dict(num_seqs=3, num_q_heads=3, num_kv_heads=3, hist=("uniform", 200, 600),
                                    num_blocks=None)),
    "gqa3_d128": ("llama3_8b_decode", dict(num_seqs=2, num_q_heads=6, num_kv_heads=2, hist=("uniform", 40, 300))),
    # 32-token blocks (Core Concepts §3.2: blocks of 16 or 32 tokens)
    "gqa4_d128_bs32": ("llama3_8b_decode", dict(num_seqs=5, hist=("fixed", [0, 31, 32, 700, 1500]), block_size=32)),
    "gqa2_d64_bs32": ("tiny_decode", dict(num_seqs=4, num_q_heads=4, num_kv_heads=2, hist=("uniform", 1, 400),
                                          num_blocks=None, block_size=32)),
    # groups of 8 or more query heads per KV head take the tensor-core kernel: 8 rows, 16 rows, a group
    # split over two CTAs (32 heads), head_dim 64, 32-token blocks; lengths 0, 1, block edges and splits
    "gqa8_d128_edges": ("llama3_8b_decode", dict(num_seqs=6, num_q_heads=32, num_kv_heads=4,
                                                 hist=("fixed", [0, 1, 15, 16, 17, 1301]))),
    "gqa16_d128": ("llama3_8b_decode", dict(num_seqs=4, num_q_heads=32, num_kv_heads=2, hist=("uniform", 1, 900))),
    "gqa32_d128": ("llama3_8b_decode", dict(num_seqs=2, num_q_heads=32, num_kv_heads=1, hist=("fixed", [5, 333]))),
    "gqa8_d64": ("tiny_decode", dict(num_seqs=4, num_q_heads=16, num_kv_heads=2, hist=("uniform", 1, 700),
                                     num_blocks=None)),
    "gqa8_d128_bs32": ("llama3_8b_decode", dict(num_seqs=4, num_q_heads=64, num_kv_heads=8, block_size=32,
                                                hist=("fixed", [31, 32, 33, 777]))),
}


@pytest.mark.parametrize("case", sorted(SMALL))
@pytest.mark.parametrize("split", [None, 64, 256])
def test_decode_bf16_matches_oracle(O, cuda_lib, case, split):
    name, ov = SMALL[case]
    batch = make_batch(name, seed=41, overrides=ov)
    ref = oracle_step(batch, O)["decode"]
    st = _gpu_decode(batch, split)
    assert cuda_lib.pa_get_device_error() == cuda_lib.PA_OK
    assert_close(to_f64(st.out_dec), ref, what=f"{case} split={split}")


@pytest.mark.parametrize("d,bs", [(64, 16), (128, 16), (128, 32)])
@pytest.mark.parametrize("split", [None, 128])
def test_decode_fp8_matches_oracle(O, cuda_lib, d, bs, split):
    batch = make_batch("mha_fp8_decode", seed=42, overrides=dict(num_seqs=4, num_q_heads=8, num_kv_heads=8,
                                                               head_dim=d, hist=("uniform", 1, 700), block_size=bs))
    st = _gpu_decode(batch, split)
    got = to_f64(st.out_dec)
    # against the oracle on the dequantised cache: kernel arithmetic only
    assert_close(got, oracle_step(batch, O)["decode"], what="fp8 vs dequantised")
    # against the oracle on the original bf16 K/V: includes the quantisation error
    b16 = make_batch("mha_fp8_decode", seed=42, overrides=dict(num_seqs=4, num_q_heads=8, num_kv_heads=8,
                                                             head_dim=d, hist=("uniform", 1, 700), kv_dtype=None,
                                                             block_size=bs))
    assert_close(got, oracle_step(b16, O)["decode"], max_tol=FP8_MAX, mean_tol=None, what="fp8 vs bf16")


def test_decode_fp8_with_gqa(O, cuda_lib):
    batch = make_batch("mha_fp8_decode", seed=43, overrides=dict(num_seqs=3, num_q_heads=16, num_kv_heads=4,
                                                               hist=("uniform", 10, 400)))
    assert_close(to_f64(_gpu_decode(batch).out_dec), oracle_step(batch, O)["decode"], what="fp8 gqa4")


# one-byte caches take the tensor-core kernel at head_dim 128 (f16 products on codes converted in
# registers; up to 8 heads the products are transposed, tokens on M): groups of 1, 2, 4, 8, 16, a group
# split over two CTAs, 32-token blocks, lengths at block edges, several splits
ONE_BYTE_MMA = {
    "g1": dict(num_seqs=4, num_q_heads=8, num_kv_heads=8, hist=("fixed", [2, 16, 500, 2100])),
    "g2": dict(num_seqs=4, num_q_heads=16, num_kv_heads=8, hist=("fixed", [1, 16, 17, 1200])),
    "g4": dict(num_seqs=5, num_q_heads=32, num_kv_heads=8, hist=("fixed", [0, 15, 16, 700, 1500])),
    "g8": dict(num_seqs=3, num_q_heads=64, num_kv_heads=8, hist=("uniform", 30, 900)),
    "g16": dict(num_seqs=3, num_q_heads=32, num_kv_heads=2, hist=("uniform", 1, 900)),
    "g32": dict(num_seqs=2, num_q_heads=32, num_kv_heads=1, hist=("fixed", [5, 333])),
    "g4_bs32": dict(num_seqs=4, num_q_heads=32, num_kv_heads=8, hist=("fixed", [31, 32, 33, 777]), block_size=32),
}


@pytest.mark.parametrize("kv", ["fp8", "int8"])
@pytest.mark.parametrize("case", sorted(ONE_BYTE_MMA))
@pytest.mark.parametrize("split", [None, 128])
def test_one_byte_gqa_decode_on_tensor_cores(O, cuda_lib, kv, case, split):
    from pagedattention_block_table_b200 import binding as B
    ov = dict(ONE_BYTE_MMA[case], kv_dtype=kv)
    batch = make_batch("mha_fp8_decode", seed=71, overrides=ov)
    assert B.pa_paged_attention_uses_tensor_cores(batch.num_q_heads, batch.num_kv_heads, 128, batch.kv_dtype) == 1
    got = to_f64(_gpu_decode(batch, split).out_dec)
    assert cuda_lib.pa_get_device_error() == cuda_lib.PA_OK
    assert_close(got, oracle_step(batch, O)["decode"], what=f"{kv} {case} vs dequantised")
    # against the original bf16 K/V: the quantisation error of a one-byte code (up to 2^-4 relative for
    # E4M3) averages out only over many tokens, so sequences of at least 64 tokens
    b16 = make_batch("mha_fp8_decode", seed=71, overrides=dict(ov, kv_dtype=None))
    long_ = batch.context_lens[:batch.num_decode] >= 64
    assert long_.any()
    assert_close(got[long_], oracle_step(b16, O)["decode"][long_], max_tol=FP8_MAX, mean_tol=None,
                 what=f"{kv} {case} vs bf16")


@pytest.mark.parametrize("e", [-20, 20, 0])
def test_one_byte_gqa_decode_any_query_magnitude(O, cuda_lib, e):
    """The tensor-core path rounds q to f16 after scaling each row by a power of two into [1, 2): q * 2^e
    with the softmax scale * 2^-e gives the same scores far outside f16's range (2^20 overflows it, 2^-20
    is below its normal range), and the output still matches the oracle."""
    import math
    batch = make_batch("mha_fp8_decode", seed=72, overrides=dict(num_seqs=3, num_q_heads=32, num_kv_heads=8,
                                                               hist=("uniform", 100, 900)))
    batch.q_decode = (batch.q_decode.float() * 2.0 ** e).to(torch.bfloat16)    # exact: a power of two
    batch.scale = 1.0 / math.sqrt(batch.head_dim) * 2.0 ** -e
    got = to_f64(_gpu_decode(batch, 256).out_dec)
    assert cuda_lib.pa_get_device_error() == cuda_lib.PA_OK
    assert_close(got, oracle_step(batch, O)["decode"], what=f"fp8 gqa, q * 2^{e}")


GROUPS = {"g4": dict(num_q_heads=32, num_kv_heads=8), "g8": dict(num_q_heads=64, num_kv_heads=8),
          "g16": dict(num_q_heads=32, num_kv_heads=2)}


@pytest.mark.parametrize("grp", sorted(GROUPS))
def test_placement_invariance_bit_identical(cuda_lib, grp):
    kw = dict(seed=44, overrides=dict(num_seqs=5, hist=("uniform", 100, 1200), **GROUPS[grp]))
    outs = [_gpu_decode(make_batch("llama3_8b_decode", perm_seed=p, **kw), 256).out_dec for p in (1, 2, -1)]
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[0], outs[2])


def test_split_and_unsplit_agree(O, cuda_lib):
    batch = make_batch("llama3_8b_decode", seed=45, overrides=dict(num_seqs=4, hist=("uniform", 1000, 3000)))
    ref = oracle_step(batch, O)["decode"]
    a = to_f64(_gpu_decode(batch, 4096).out_dec)
    b = to_f64(_gpu_decode(batch, 512).out_dec)
    assert_close(a, ref, what="unsplit")
    assert_close(b, ref, what="split 512")
    assert_close(a, b, max_tol=ATOL_MAX, mean_tol=ATOL_MEAN, what="split vs unsplit")


@pytest.mark.parametrize("grp", sorted(GROUPS))
def test_one_token_context_returns_v_exactly(cuda_lib, grp):
    batch = make_batch("llama3_8b_decode", seed=46, overrides=dict(num_seqs=3, hist=("fixed", [0, 0, 0]),
                                                                   **GROUPS[grp]))
    st = _gpu_decode(batch)
    g = batch.num_q_heads // batch.num_kv_heads
    for s in range(3):
        v0 = st.v_new[s]                                   # the only token: [Hkv][D]
        assert torch.equal(st.out_dec[s], v0.repeat_interleave(g, 0))


@pytest.mark.parametrize("grp", sorted(GROUPS))
def test_zero_length_sequence_gives_zero_row(cuda_lib, grp):
    from pagedattention_block_table_b200 import binding as B
    batch = make_batch("llama3_8b_decode", seed=47, overrides=dict(num_seqs=3, hist=("fixed", [5, 40, 9]),
                                                                   **GROUPS[grp]))
    from pagedattention_block_table_b200.runner import DeviceStep
    st = DeviceStep(batch)
    st.fill_history()
    st.append()
    lens = st.dec_lens.clone()
    lens[1] = 0
    out = torch.full_like(st.out_dec, 7.0)
    B.pa_paged_attention(out, st.q_dec, st.k_cache, st.v_cache, st.dec_tables, lens, batch.scale, st.dec_max_len)
    torch.cuda.synchronize()
    assert torch.count_nonzero(out[1]) == 0
    assert torch.isfinite(out.float()).all()


@pytest.mark.parametrize("hq", [8, 16])
def test_bad_block_id_is_flagged_and_stays_in_pool(cuda_lib, hq):
    from pagedattention_block_table_b200 import binding as B
    batch = make_batch("tiny_decode", seed=48, overrides=dict(num_q_heads=hq))
    from pagedattention_block_table_b200.runner import DeviceStep
    st = DeviceStep(batch)
    st.fill_history()
    st.append()
    bad = st.dec_tables.clone()
    bad[2, 1] = batch.num_blocks + 1000
    B.pa_paged_attention(st.out_dec, st.q_dec, st.k_cache, st.v_cache, bad, st.dec_lens, batch.scale, st.dec_max_len)
    assert B.pa_get_device_error() == B.PA_EDEVICE_OOB
    lens = st.dec_lens.clone()
    lens[0] = batch.max_blocks_per_seq * 16 + 5                     # beyond the table row
    B.pa_paged_attention(st.out_dec, st.q_dec, st.k_cache, st.v_cache, st.dec_tables, lens, batch.scale,
                         batch.max_blocks_per_seq * 16 + 5)
    assert B.pa_get_device_error() == B.PA_EDEVICE_OOB
    assert B.pa_get_device_error() == B.PA_OK


def test_one_byte_decode_at_head_dim_64_on_cuda_cores(O, cuda_lib):
    """One-byte caches at head_dim 64 stay on the CUDA-core kernel (FP8 here; INT8 below)."""
    from pagedattention_block_table_b200 import binding as B
    assert B.pa_paged_attention_uses_tensor_cores(4, 2, 64, B.PA_KV_FP8_E4M3) == 0
    ov = dict(num_seqs=4, num_q_heads=4, num_kv_heads=2, head_dim=64, hist=("uniform", 1, 700), kv_dtype="fp8")
    batch = make_batch("mha_fp8_decode", seed=48, overrides=ov)
    assert_close(to_f64(_gpu_decode(batch, 256).out_dec), oracle_step(batch, O)["decode"], what="fp8 d64")


@pytest.mark.parametrize("d,hq,hkv", [(128, 8, 8), (128, 16, 4), (64, 4, 2)])
def test_decode_int8_matches_oracle(O, cuda_lib, d, hq, hkv):
    ov = dict(num_seqs=4, num_q_heads=hq, num_kv_heads=hkv, head_dim=d, hist=("uniform", 1, 700), kv_dtype="int8")
    batch = make_batch("mha_fp8_decode", seed=49, overrides=ov)
    got = to_f64(_gpu_decode(batch, 256).out_dec)
    assert_close(got, oracle_step(batch, O)["decode"], what="int8 vs dequantised")
    b16 = make_batch("mha_fp8_decode", seed=49, overrides=dict(ov, kv_dtype=None))
    assert_close(got, oracle_step(b16, O)["decode"], max_tol=FP8_MAX, mean_tol=None, what="int8 vs bf16")


def test_kv_head_shards_reproduce_the_unsharded_call(O, cuda_lib):
    """Tensor-parallel KV-head shards (KV Cache to vLLM §4.4: tensor parallelism splits the KV cache), run
    one after the other on one GPU (no rank waits on another): each shard's output matches the oracle on
    that shard, and together they are bit-identical to the unsharded call at the same split."""
    from pagedattention_block_table_b200 import sharding
    batch = make_batch("llama3_8b_decode", seed=50, overrides=dict(num_seqs=5, hist=("uniform", 100, 1500)))
    full = _gpu_decode(batch, 256).out_dec
    parts = []
    for r in range(4):
        shard = sharding.shard_batch(batch, r, 4)
        out = _gpu_decode(shard, 256).out_dec
        assert_close(to_f64(out), oracle_step(shard, O)["decode"], what=f"shard {r} of 4")
        parts.append(out)
    assert torch.equal(torch.cat(parts, dim=1), full)


@pytest.mark.parametrize("graphs", [True, False])
def test_host_pipeline_delivers_the_step_outputs(cuda_lib, graphs):
    """The double-buffered host-fed pipeline (inputs copied in and outputs copied out every step,
    overlapped with compute; CUDA graphs per slot or eager launches) returns the same outputs to the
    host as a plain device step, and a step run after new inputs were written to the host buffer uses
    those inputs."""
    from pagedattention_block_table_b200.runner import DeviceStep, HostPipeline
    # no shared prefixes: a repeated step is then idempotent (with forks, re-copying a page that its
    # last holder already appended into would change the copy)
    ov = dict(num_seqs=6, hist=("uniform", 20, 300), share_group=0, share_prefix=0, prefill_chunks=2,
              chunk_len=(30, 150), chunk_hist=(1, 100), num_q_heads=8, num_kv_heads=2)
    batch = make_batch("mixed_step", seed=53, overrides=ov)
    ref = _gpu_decode(batch, 64)
    st = DeviceStep(batch, split_tokens=64)
    st.fill_history()
    pipe = HostPipeline(st, use_graphs=graphs)
    assert (pipe.graphs[0] is not None) == graphs
    for _ in range(5):
        pipe.step()
    pipe.finish()
    torch.cuda.synchronize()
    for s in range(2):
        assert torch.equal(pipe.host_out[s][0], ref.out_dec.cpu())
        assert torch.equal(pipe.host_out[s][1], ref.out_pre.cpu())
    # new queries through the host buffer (negated: exact).  The next step's inputs are already on the
    # device, so the two steps after it (one per slot) are the first to read the new ones
    batch2 = make_batch("mixed_step", seed=53, overrides=ov)
    batch2.q_decode = -batch2.q_decode
    ref2 = _gpu_decode(batch2, 64)
    pipe.host_in["q_dec"].copy_(batch2.q_decode)
    for _ in range(3):
        pipe.step()
    pipe.finish()
    torch.cuda.synchronize()
    for s in range(2):
        assert torch.equal(pipe.host_out[s][0], ref2.out_dec.cpu())
        assert torch.equal(pipe.host_out[s][1], ref.out_pre.cpu())
    assert not torch.equal(ref2.out_dec, ref.out_dec)


@pytest.mark.parametrize("grp", ["g4", "g8"])
@pytest.mark.parametrize("split", [64, 256])
def test_longest_first_order_changes_nothing_but_the_order(O, cuda_lib, split, grp):
    """The host copy of the context lengths only orders the launch (longest (sequence, split) first):
    natural order, the true lengths and deliberately wrong ones all give bit-identical outputs, and
    they match the oracle."""
    from pagedattention_block_table_b200 import binding as B
    batch = make_batch("llama3_8b_decode", seed=61, overrides=dict(num_seqs=9, hist=("uniform", 0, 1500),
                                                                   **GROUPS[grp]))
    st = _gpu_decode(batch, split)
    ref = oracle_step(batch, O)["decode"]
    outs = {}
    true_lens = st.dec_lens_host
    for name, host in (("natural", None), ("true", true_lens), ("reversed", np.ascontiguousarray(true_lens[::-1])),
                       ("zeros", np.zeros_like(true_lens)), ("huge", np.full_like(true_lens, 1 << 30)),
                       ("cpu tensor", torch.from_numpy(true_lens.copy()))):
        out = torch.full_like(st.out_dec, float("nan"))
        B.pa_paged_attention(out, st.q_dec, st.k_cache, st.v_cache, st.dec_tables, st.dec_lens, batch.scale,
                             st.dec_max_len, split_tokens=split, workspace=st.workspace, host_context_lens=host)
        torch.cuda.synchronize()
        outs[name] = out
    assert B.pa_get_device_error() == B.PA_OK
    for name, out in outs.items():
        assert torch.equal(out, outs["natural"]), name
    assert_close(to_f64(outs["true"]), ref, what=f"ordered launch, split {split}")
    with pytest.raises(ValueError):
        B.pa_paged_attention(st.out_dec, st.q_dec, st.k_cache, st.v_cache, st.dec_tables, st.dec_lens, batch.scale,
                             st.dec_max_len, split_tokens=split, workspace=st.workspace,
                             host_context_lens=true_lens[:-1])


@pytest.mark.parametrize("grp", ["g4", "g8"])
def test_many_splits_and_a_reused_workspace(O, cuda_lib, grp):
    """79 and 313 splits of one sequence (the reduce kernel loops over more than 32 partials per lane
    group), a second call on the same workspace, and sampled rows against the oracle."""
    from pagedattention_block_table_b200 import binding as B
    batch = make_batch("llama3_8b_decode", seed=62, overrides=dict(num_seqs=3, hist=("fixed", [20000, 7000, 300]),
                                                                   **GROUPS[grp]))
    for split in (256, 64):
        st = _gpu_decode(batch, split)
        first = st.out_dec.clone()
        st.decode()
        torch.cuda.synchronize()
        assert torch.equal(st.out_dec, first), f"second call on the same workspace, split {split}"
        got = to_f64(st.out_dec)
        for s in range(3):
            assert_close(got[s], oracle_decode_one(batch, s, O), what=f"seq {s}, split {split}")
    assert B.pa_get_device_error() == B.PA_OK


@pytest.mark.parametrize("e", [-20, 20, 0])
def test_decode_fp8_any_query_magnitude(O, cuda_lib, e):
    """Scores do not depend on how q and the softmax scale share a power of two: q * 2^e with the scale
    * 2^-e gives the same scores (the FP8 decode folds the scale and the K scale into q in fp32), far
    outside bf16's usual range of q, and the output still matches the oracle."""
    import math
    batch = make_batch("mha_fp8_decode", seed=63, overrides=dict(num_seqs=3, num_q_heads=8, num_kv_heads=4,
                                                               hist=("uniform", 100, 900)))
    batch.q_decode = (batch.q_decode.float() * 2.0 ** e).to(torch.bfloat16)    # exact: a power of two
    batch.scale = 1.0 / math.sqrt(batch.head_dim) * 2.0 ** -e
    got = to_f64(_gpu_decode(batch, 256).out_dec)
    assert cuda_lib.pa_get_device_error() == cuda_lib.PA_OK
    assert_close(got, oracle_step(batch, O)["decode"], what=f"fp8, q * 2^{e}")
