"""pa_paged_attention_noalloc: the decode call for callers that cannot allocate device memory
(for example a plugin inside a serving engine that has reserved the GPU's memory for its own KV
pool, or a latency-critical loop that must not take cudaMalloc's device-wide synchronisation).
Its split partials live in a static per-device scratch array inside the library instead of a
caller workspace.  Checked through the C ABI against pa_paged_attention with a caller workspace,
on two calls in a row (the second finds the first call's partials still in the scratch).

This file is named to be collected last; it builds all of its own inputs, so it also passes
when run alone in a fresh process.
"""
import pytest
import torch

from pagedattention_block_table_b200.inputs import make_batch
from tests.common import ATOL_MAX, ATOL_MEAN, assert_close, to_f64

pytestmark = pytest.mark.gpu


def _prepared(seed, seqs, hist, split):
    from pagedattention_block_table_b200.runner import DeviceStep
    batch = make_batch("llama3_8b_decode", seed=seed, overrides=dict(num_seqs=seqs, hist=hist))
    st = DeviceStep(batch, split_tokens=split)
    st.fill_history()
    st.append()
    return batch, st


def _with_workspace(B, batch, st, split):
    ref = torch.empty_like(st.out_dec)
    S = split or B.pa_paged_attention_auto_split(batch.num_decode, batch.num_q_heads, batch.num_kv_heads,
                                                 batch.head_dim, st.dec_max_len)
    ws_bytes = B.pa_paged_attention_workspace_size(batch.num_decode, batch.num_q_heads, batch.head_dim,
                                                   st.dec_max_len, S)
    ws = torch.empty(ws_bytes // 4 + 4, dtype=torch.float32, device="cuda") if ws_bytes else None
    B.pa_paged_attention(ref, st.q_dec, st.k_cache, st.v_cache, st.dec_tables, st.dec_lens, batch.scale,
                         st.dec_max_len, split_tokens=split, workspace=ws)
    return ref


def _no_alloc(B, batch, st, split):
    out = torch.full_like(st.out_dec, float("nan"))
    B.pa_paged_attention_noalloc(out, st.q_dec, st.k_cache, st.v_cache, st.dec_tables, st.dec_lens, batch.scale,
                                 st.dec_max_len, split_tokens=split)
    return out


@pytest.mark.parametrize("split", [512, 0])
def test_noalloc_matches_workspace_call_twice(cuda_lib, split):
    B = cuda_lib
    batch, st = _prepared(71, 6, ("uniform", 600, 3000), 512)
    ref = _with_workspace(B, batch, st, split)
    for call in range(2):
        out = _no_alloc(B, batch, st, split)
        torch.cuda.synchronize()
        assert B.pa_get_device_error() == B.PA_OK
        assert_close(to_f64(out), to_f64(ref), max_tol=ATOL_MAX, mean_tol=ATOL_MEAN, what=f"call {call}")


def test_noalloc_second_workload_sees_no_stale_partials(cuda_lib):
    B = cuda_lib
    for seed, seqs, hist in ((72, 5, ("uniform", 1500, 4000)), (73, 3, ("uniform", 520, 1100))):
        batch, st = _prepared(seed, seqs, hist, 256)
        ref = _with_workspace(B, batch, st, 256)
        out = _no_alloc(B, batch, st, 256)
        torch.cuda.synchronize()
        assert_close(to_f64(out), to_f64(ref), what=f"seed {seed}")


def test_noalloc_rejects_partials_beyond_the_scratch(cuda_lib):
    B = cuda_lib
    batch, st = _prepared(74, 64, ("uniform", 4000, 4096), 512)
    need = B.pa_paged_attention_workspace_size(64, 32, 128, st.dec_max_len, 16)
    assert need > 16 * 1024 * 1024
    out = torch.empty_like(st.out_dec)
    with pytest.raises(B.PagedAttnError) as e:
        B.pa_paged_attention_noalloc(out, st.q_dec, st.k_cache, st.v_cache, st.dec_tables, st.dec_lens,
                                     batch.scale, st.dec_max_len, split_tokens=16)
    assert e.value.status == B.PA_EWORKSPACE


def test_noalloc_lengthens_an_auto_split_that_overflows_the_scratch(cuda_lib):
    """split_tokens = 0 where the auto split's partials would not fit the static scratch: the call lengthens
    the split until they do, and gives exactly what the workspace call gives at that split."""
    from pagedattention_block_table_b200.runner import DeviceStep
    B = cuda_lib
    cap = 16 * 1024 * 1024
    batch = make_batch("llama3_8b_decode", seed=75, device="cuda",
                       overrides=dict(num_seqs=64, num_q_heads=128, num_kv_heads=8, hist=("uniform", 6200, 8000)))
    st = DeviceStep(batch, split_tokens=512)
    st.fill_history()
    st.append()
    args = (batch.num_decode, batch.num_q_heads, batch.head_dim, st.dec_max_len)
    S = B.pa_paged_attention_auto_split(batch.num_decode, batch.num_q_heads, batch.num_kv_heads, batch.head_dim,
                                        st.dec_max_len)
    assert B.pa_paged_attention_workspace_size(*args, S) > cap, "the case must overflow at the auto split"
    while B.pa_paged_attention_workspace_size(*args, S) > cap:
        S = -(-2 * S // 16) * 16
    ref = _with_workspace(B, batch, st, S)
    for call in range(2):
        out = _no_alloc(B, batch, st, 0)
        torch.cuda.synchronize()
        assert B.pa_get_device_error() == B.PA_OK
        assert torch.equal(out, ref), f"call {call}"
