"""The full-size workloads against the oracle, every output element.

Each runs on the GPU exactly as bench.py times it (same inputs, same split choice, longest-first launch
order): the Llama-3-8B-shaped decode batch (64 sequences, 32/8 heads, contexts 513..4097), the
continuous-batching mixed step (256 prefix-sharing decode sequences with copy-on-write forks plus four
causal prefill chunks of 512..2048 tokens), the long-context batch (8 x 32768 tokens, split 512), the
MHA batch over an FP8 E4M3 cache (32 sequences, 64/64 heads, contexts 2049..8193), a GQA batch with
eight query heads per KV head (32 sequences, 64/8 heads, contexts 513..4097) and the Llama-3-8B batch over
an FP8 cache, and the mixed step over an FP8 cache.  The oracle computes every sequence from its own token rows in a fresh contiguous cache (no
paging, sharing or forks), so the comparison also checks that paging, prefix sharing and copy-on-write
change nothing.
Tolerances: attention max-abs <= 1e-2 and mean-abs <= 1e-3 against the oracle on the same bf16 inputs
(for the FP8 cache: on the same dequantised codes), and <= 5e-2 max against the oracle on the original
bf16 K/V for the FP8 cache.
"""
import numpy as np
import pytest
import torch

from pagedattention_block_table_b200.inputs import make_batch
from tests.common import FP8_MAX, assert_close, oracle_decode_all, oracle_prefill_all, to_f64

pytestmark = pytest.mark.gpu


def _run(batch):
    from pagedattention_block_table_b200.runner import DeviceStep
    st = DeviceStep(batch, split_tokens=None)
    st.fill_history()
    st.step()
    torch.cuda.synchronize()
    return st


@pytest.mark.parametrize("name", ["llama3_8b_decode", "long_context_decode", "mha_fp8_decode", "gqa8_decode",
                                  "llama3_8b_fp8_decode"])
def test_full_size_decode_every_element(O, cuda_lib, name):
    batch = make_batch(name, device="cuda")
    st = _run(batch)
    assert cuda_lib.pa_get_device_error() == cuda_lib.PA_OK
    if name == "long_context_decode":
        assert st.split_tokens == 512 and st.dec_max_len == 32768          # 64 splits per sequence
    got = to_f64(st.out_dec)
    assert_close(got, oracle_decode_all(batch, O), what=name)
    if batch.kv_dtype:
        assert_close(got, oracle_decode_all(batch, O, kv_dtype=0), max_tol=FP8_MAX, mean_tol=None,
                     what=f"{name} vs the bf16 K/V")


@pytest.mark.parametrize("name", ["mixed_step", "mixed_step_fp8"])
def test_full_size_mixed_step_every_element(O, cuda_lib, name):
    batch = make_batch(name, device="cuda")
    assert batch.cow_pairs.shape[0] > 0 and batch.shared_blocks.shape[0] > 0
    st = _run(batch)
    assert cuda_lib.pa_get_device_error() == cuda_lib.PA_OK
    assert_close(to_f64(st.out_dec), oracle_decode_all(batch, O), what=f"{name}: 256 decode rows")
    assert_close(to_f64(st.out_pre), oracle_prefill_all(batch, O), what=f"{name}: every prefill row")


def test_full_size_chunked_long_prompt_every_element(O, cuda_lib):
    """Chunked prefill of a long prompt (a 512-token chunk 32,256 tokens into a prompt, beside one that
    starts a prompt): far fewer query-tile CTAs than SMs, so the planned launch splits the long key
    ranges and merges them; every prefill row equals the oracle."""
    batch = make_batch("chunked_prefill_long", device="cuda")
    st = _run(batch)
    assert st.pre_workspace is not None, "the long key ranges were expected to be split"
    assert cuda_lib.pa_get_device_error() == cuda_lib.PA_OK
    got, ref = to_f64(st.out_pre), oracle_prefill_all(batch, O)
    cu = batch.cu_q_lens
    # the chunk 32,256 tokens in (its key ranges split and merged): the default tolerance
    assert_close(got[cu[1]:cu[2]], ref[cu[1]:cu[2]], what="chunk over the long history")
    # the chunk that starts a prompt: its first rows see a handful of keys, so the bf16 roundings are not
    # averaged away: P rounded to bf16 (relative 2^-9 per weight, weights summing to 1) moves out by at
    # most 2^-9 max|v|, and the bf16 output by half an ulp, 2^-9 |out|
    vmax = float(batch.tok_v.float().abs().max())
    bound = 2.0 ** -9 * (vmax + float(np.abs(ref).max())) + 1e-3
    assert_close(got[:cu[1]], ref[:cu[1]], max_tol=bound, what="chunk starting a prompt")
