"""GPU parity of the paged prefill (tcgen05 for bf16 caches, warp-level tensor cores for one-byte caches) and
of the whole mixed step against the oracle."""
import numpy as np
import pytest
import torch

from pagedattention_block_table_b200.inputs import make_batch
from tests.common import assert_close, oracle_step, to_f64

pytestmark = pytest.mark.gpu


def _run(batch):
    from pagedattention_block_table_b200.runner import DeviceStep
    st = DeviceStep(batch)
    st.fill_history()
    st.step()
    torch.cuda.synchronize()
    return st


def _chunks(**ov):
    base = dict(num_seqs=1, hist=("fixed", [3]), share_group=0, share_prefix=0, num_q_heads=8, num_kv_heads=2,
                head_dim=128, prefill_chunks=3, chunk_len=(1, 300), chunk_hist=(1, 400))
    base.update(ov)
    return base


CASES = {
    "gqa4_d128": _chunks(),
    "gqa4_d128_long": _chunks(prefill_chunks=2, chunk_len=(300, 700), chunk_hist=(500, 900)),
    "mha_d128": _chunks(num_q_heads=4, num_kv_heads=4, chunk_len=(100, 260)),
    "gqa2_d64": _chunks(head_dim=64, num_q_heads=4, num_kv_heads=2),
    "tiny_chunks": _chunks(prefill_chunks=5, chunk_len=(1, 17), chunk_hist=(1, 40)),
    "gqa8_d128": _chunks(num_q_heads=16, num_kv_heads=2, chunk_len=(20, 150)),
    "gqa3_d128": _chunks(num_q_heads=6, num_kv_heads=2, chunk_len=(60, 200)),
    "gqa16_d64": _chunks(num_q_heads=16, num_kv_heads=1, head_dim=64, chunk_len=(5, 90)),
    "gqa4_d128_bs32": _chunks(block_size=32, chunk_len=(40, 300), chunk_hist=(1, 300)),
}


@pytest.mark.parametrize("case", sorted(CASES))
def test_prefill_matches_oracle(O, cuda_lib, case):
    batch = make_batch("mixed_step", seed=51, overrides=CASES[case])
    ref = oracle_step(batch, O)
    st = _run(batch)
    assert cuda_lib.pa_get_device_error() == cuda_lib.PA_OK
    assert_close(to_f64(st.out_pre), ref["prefill"], what=f"prefill {case}")
    assert_close(to_f64(st.out_dec), ref["decode"], what=f"decode {case}")


def test_prefill_chunk_starting_a_request(O, cuda_lib):
    """H = 0: row 0 sees only key 0, so its output is exactly V[0]."""
    batch = make_batch("mixed_step", seed=52, overrides=_chunks(prefill_chunks=1, chunk_len=(200, 200)))
    st = _run(batch)
    ref = oracle_step(batch, O)["prefill"]
    assert_close(to_f64(st.out_pre), ref, what="H=0 chunk")
    g = batch.num_q_heads // batch.num_kv_heads
    # appended tokens: the decoding sequence's first, then the chunk's; chunk row 0 is step token 1
    assert torch.equal(st.out_pre[0], st.v_new[1].repeat_interleave(g, 0))


def test_prefill_placement_invariance(cuda_lib):
    kw = dict(seed=53, overrides=_chunks(prefill_chunks=2, chunk_len=(130, 300), chunk_hist=(17, 300)))
    a = _run(make_batch("mixed_step", perm_seed=1, **kw)).out_pre
    b = _run(make_batch("mixed_step", perm_seed=2, **kw)).out_pre
    assert torch.equal(a, b)


@pytest.mark.parametrize("scale", [2.5, -2.5])
def test_prefill_large_and_negative_scale(O, cuda_lib, scale):
    """Scores with a standard deviation of ~40 in log2 units: the running max of a row climbs by more
    than 2^8 several times along the history, so the kernel moves its reference and rescales O in TMEM.
    A negative scale turns the tile max into the min of the raw scores."""
    batch = make_batch("mixed_step", seed=54, overrides=_chunks(prefill_chunks=2, chunk_len=(200, 400),
                                                                chunk_hist=(600, 1200)))
    batch.scale = scale
    ref = oracle_step(batch, O)
    st = _run(batch)
    assert cuda_lib.pa_get_device_error() == cuda_lib.PA_OK
    # Near one-hot rows make out ~ one V row (|v| up to ~4.5), so the bf16 roundings are not averaged
    # away: P rounded to bf16 (relative 2^-9 per weight, weights summing to 1) moves out by at most
    # 2^-9 max|v|, and the bf16 output by half an ulp, 2^-9 |out|.
    vmax = float(batch.tok_v.float().abs().max())
    for name in ("prefill", "decode"):
        got = to_f64(st.out_pre if name == "prefill" else st.out_dec)
        bound = 2.0 ** -9 * (vmax + float(np.abs(ref[name]).max())) + 1e-3
        assert_close(got, ref[name], max_tol=bound, mean_tol=bound / 4, what=f"{name}, scale {scale}")


def test_prefill_chunk_longer_than_max_q_is_flagged(cuda_lib):
    """A chunk longer than the max_q_len the call was given is reported, not silently cut short."""
    from pagedattention_block_table_b200.runner import DeviceStep
    batch = make_batch("mixed_step", seed=55, overrides=_chunks(prefill_chunks=2, chunk_len=(300, 300)))
    st = DeviceStep(batch)
    st.fill_history()
    st.append()
    torch.cuda.synchronize()
    assert cuda_lib.pa_get_device_error() == cuda_lib.PA_OK
    cuda_lib.pa_paged_prefill(st.out_pre, st.q_pre, st.cu_q, st.k_cache, st.v_cache, st.pre_tables, st.pre_lens,
                              batch.scale, 100, st.pre_max_len)
    assert cuda_lib.pa_get_device_error() == cuda_lib.PA_EDEVICE_OOB
    assert cuda_lib.pa_get_device_error() == cuda_lib.PA_OK          # reading the word clears it


ONE_BYTE = {k: CASES[k] for k in ("gqa4_d128", "gqa4_d128_long", "mha_d128", "tiny_chunks", "gqa8_d128", "gqa3_d128",
                                  "gqa4_d128_bs32")}
ONE_BYTE["gqa16_d128"] = _chunks(num_q_heads=16, num_kv_heads=1, chunk_len=(5, 90))


@pytest.mark.parametrize("kv", ["fp8", "int8"])
@pytest.mark.parametrize("case", sorted(ONE_BYTE))
def test_one_byte_prefill_matches_oracle(O, cuda_lib, case, kv):
    """Prefill over FP8 / INT8 caches (f16 products on codes converted in registers) against the oracle on
    the same codes and scales; the step's decode rows ride along."""
    batch = make_batch("mixed_step", seed=54, overrides=dict(ONE_BYTE[case], kv_dtype=kv))
    ref = oracle_step(batch, O)
    st = _run(batch)
    assert cuda_lib.pa_get_device_error() == cuda_lib.PA_OK
    assert_close(to_f64(st.out_pre), ref["prefill"], what=f"{kv} prefill {case}")
    assert_close(to_f64(st.out_dec), ref["decode"], what=f"{kv} decode {case}")


def test_one_byte_prefill_long_chunk_over_long_history(O, cuda_lib):
    """1000-row FP8 chunks with GQA 4, one starting a request and one over a 2000-token history: many row
    tiles, every key unit, the causal edge inside the last units."""
    ov = _chunks(prefill_chunks=2, chunk_len=(1000, 1000), chunk_hist=(2000, 2000), kv_dtype="fp8")
    batch = make_batch("mixed_step", seed=55, overrides=ov)
    ref = oracle_step(batch, O)["prefill"]
    st = _run(batch)
    assert cuda_lib.pa_get_device_error() == cuda_lib.PA_OK
    assert_close(to_f64(st.out_pre), ref, what="fp8 long chunk")


# ---------------------------------------------------------------------------------------------- planned launches
# With host copies of the lengths the call plans its launch: longest work first, and a CTA whose key range
# is long next to the launch's work per SM runs as pieces whose partials a merge kernel combines.

PLAN_CASES = {
    # two long histories in a small launch: the long CTAs are cut into pieces
    "long_histories": _chunks(prefill_chunks=2, chunk_len=(300, 600), chunk_hist=(3000, 5000)),
    # one chunk starting a request next to a long one: uneven CTAs
    "uneven": _chunks(prefill_chunks=3, chunk_len=(64, 900), chunk_hist=(1, 6000)),
    "gqa8_bs32": _chunks(num_q_heads=16, num_kv_heads=2, block_size=32, prefill_chunks=2, chunk_len=(100, 400),
                         chunk_hist=(2000, 4000)),
    "mha_d64": _chunks(num_q_heads=4, num_kv_heads=4, head_dim=64, prefill_chunks=2, chunk_len=(200, 300),
                       chunk_hist=(2500, 3500)),
}


def _unplanned(st, cuda_lib):
    out = torch.empty_like(st.out_pre)
    cuda_lib.pa_paged_prefill(out, st.q_pre, st.cu_q, st.k_cache, st.v_cache, st.pre_tables, st.pre_lens,
                              st.batch.scale, st.max_q, st.pre_max_len, st.kv_dtype, k_scale=st.k_scale,
                              v_scale=st.v_scale)
    torch.cuda.synchronize()
    return out


@pytest.mark.parametrize("kv", ["bf16", "fp8"])
@pytest.mark.parametrize("case", sorted(PLAN_CASES))
def test_planned_prefill_matches_oracle(O, cuda_lib, case, kv):
    """The planned launch splits key ranges (it asks for workspace) and still equals the oracle, and the
    unplanned launch of the same call, up to the rounding of the merge."""
    ov = dict(PLAN_CASES[case])
    if kv == "fp8":
        if ov["head_dim"] != 128:
            pytest.skip("one-byte caches need head_dim 128")
        ov["kv_dtype"] = "fp8"
    batch = make_batch("mixed_step", seed=57, overrides=ov)
    ref = oracle_step(batch, O)["prefill"]
    st = _run(batch)
    assert st.pre_workspace is not None, "the plan was expected to split this launch"
    assert cuda_lib.pa_get_device_error() == cuda_lib.PA_OK
    assert_close(to_f64(st.out_pre), ref, what=f"planned {kv} prefill {case}")
    plain = _unplanned(st, cuda_lib)
    assert cuda_lib.pa_get_device_error() == cuda_lib.PA_OK
    assert_close(to_f64(plain), ref, what=f"unplanned {kv} prefill {case}")
    d = (st.out_pre.float() - plain.float()).abs()
    assert float(d.max()) <= 2e-2 and float(d.mean()) <= 1e-3


def _planned_call(st, cuda_lib, host_cu, host_ctx, max_q, max_ctx):
    ws_bytes = cuda_lib.pa_paged_prefill_workspace_size(host_cu, host_ctx, st.batch.num_q_heads,
                                                        st.batch.num_kv_heads, st.batch.head_dim,
                                                        st.pre_tables.shape[1], st.batch.block_size, max_q, max_ctx)
    ws = torch.empty(ws_bytes // 4 + 4, dtype=torch.float32, device="cuda") if ws_bytes else None
    out = torch.zeros_like(st.out_pre)
    cuda_lib.pa_paged_prefill(out, st.q_pre, st.cu_q, st.k_cache, st.v_cache, st.pre_tables, st.pre_lens,
                              st.batch.scale, max_q, max_ctx, st.kv_dtype, k_scale=st.k_scale, v_scale=st.v_scale,
                              host_cu_q_lens=host_cu, host_context_lens=host_ctx, workspace=ws)
    torch.cuda.synchronize()
    return out, ws_bytes


def test_planned_prefill_with_longer_host_histories(O, cuda_lib):
    """Host lengths longer than the device's (within the table rows): the plan has pieces past the device's
    keys, which leave empty partials, and the output still equals the oracle for the device lengths."""
    batch = make_batch("mixed_step", seed=58, overrides=_chunks(prefill_chunks=2, chunk_len=(300, 300),
                                                                chunk_hist=(1000, 4000)))
    st = _run(batch)
    ref = oracle_step(batch, O)["prefill"]
    cap = st.pre_tables.shape[1] * batch.block_size
    host_ctx = np.minimum(st.pre_lens_host + 2500, cap).astype(np.int32)
    out, ws_bytes = _planned_call(st, cuda_lib, st.pre_cu_host, host_ctx, st.max_q, int(host_ctx.max()))
    assert ws_bytes > 0
    assert cuda_lib.pa_get_device_error() == cuda_lib.PA_OK
    # Rows near the start of the chunk that starts a request see a handful of keys, so the bf16 roundings
    # are not averaged away: P rounded to bf16 (relative 2^-9 per weight, weights summing to 1) moves out
    # by at most 2^-9 max|v|, and the bf16 output by half an ulp, 2^-9 |out|.
    vmax = float(batch.tok_v.float().abs().max())
    bound = 2.0 ** -9 * (vmax + float(np.abs(ref).max())) + 1e-3
    assert_close(to_f64(out), ref, max_tol=bound, what="planned with longer host histories")
    # the same arithmetic as the launch planned for the true lengths, up to the merge's rounding
    d = (out.float() - st.out_pre.float()).abs()
    assert float(d.max()) <= 2e-2 and float(d.mean()) <= 1e-4


def test_planned_prefill_with_shorter_host_chunk_is_flagged(cuda_lib):
    """Host lengths that give a chunk fewer new tokens than the device's leave query tiles unplanned: the
    call reports it in the device error word instead of silently skipping rows."""
    batch = make_batch("mixed_step", seed=59, overrides=_chunks(prefill_chunks=2, chunk_len=(600, 600),
                                                                chunk_hist=(500, 900)))
    st = _run(batch)
    host_cu = st.pre_cu_host.copy()
    host_cu[1:] -= 300                                 # chunk 0 three hundred rows short on the host
    host_ctx = st.pre_lens_host.copy()
    host_ctx[0] -= 300
    assert cuda_lib.pa_paged_prefill_workspace_size(host_cu, host_ctx, batch.num_q_heads, batch.num_kv_heads,
                                                    batch.head_dim, st.pre_tables.shape[1], batch.block_size,
                                                    st.max_q, st.pre_max_len) > 0   # the call is planned
    _planned_call(st, cuda_lib, host_cu, host_ctx, st.max_q, st.pre_max_len)
    assert cuda_lib.pa_get_device_error() == cuda_lib.PA_EDEVICE_OOB
    assert cuda_lib.pa_get_device_error() == cuda_lib.PA_OK
