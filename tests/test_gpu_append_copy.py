"""GPU parity of kv_append (bf16 and FP8) and copy_blocks against the oracle: bit-exact."""
import numpy as np
import pytest
import torch

from pagedattention_block_table_b200.inputs import make_batch, bf16_bits
from tests.common import oracle_step

pytestmark = pytest.mark.gpu

SMALL_MIXED = dict(num_seqs=40, hist=("lognormal", 60.0, 1.0, 1, 400), share_group=8, share_prefix=96,
                   prefill_chunks=3, chunk_len=(1, 70), chunk_hist=(1, 90), num_q_heads=8, num_kv_heads=2,
                   head_dim=128)


def _cache_np(t):
    if t.dtype == torch.bfloat16:
        return bf16_bits(t)
    return t.cpu().numpy()


def _gpu_step_caches(batch, cuda_lib):
    from pagedattention_block_table_b200.runner import DeviceStep
    st = DeviceStep(batch)
    st.fill_history()
    k_pre, v_pre = _cache_np(st.k_cache), _cache_np(st.v_cache)
    st.fork()
    st.append()
    torch.cuda.synchronize()
    assert cuda_lib.pa_get_device_error() == cuda_lib.PA_OK
    return k_pre, v_pre, _cache_np(st.k_cache), _cache_np(st.v_cache)


@pytest.mark.parametrize("head_dim,bs", [(64, 16), (128, 16), (128, 32)])
def test_append_and_fork_bf16_bit_exact(O, cuda_lib, head_dim, bs):
    batch = make_batch("mixed_step", seed=31, overrides=dict(SMALL_MIXED, head_dim=head_dim, block_size=bs))
    assert batch.cow_pairs.shape[0] > 0
    ref = oracle_step(batch, O, keep_pre_step=True)
    k_pre, v_pre, k, v = _gpu_step_caches(batch, cuda_lib)
    assert np.array_equal(k_pre, ref["k_pre"]) and np.array_equal(v_pre, ref["v_pre"])
    assert np.array_equal(k, ref["k_cache"]) and np.array_equal(v, ref["v_cache"])


def test_append_fp8_bit_exact(O, cuda_lib):
    batch = make_batch("mha_fp8_decode", seed=32, overrides=dict(num_seqs=5, num_q_heads=4, num_kv_heads=4,
                                                               hist=("uniform", 1, 300)))
    ref = oracle_step(batch, O)
    _, _, k, v = _gpu_step_caches(batch, cuda_lib)
    assert np.array_equal(k, ref["k_cache"]) and np.array_equal(v, ref["v_cache"])


def test_fp8_quantiser_all_bf16_inputs(O, cuda_lib):
    """Every finite bf16 value, divided by several scales, encodes to the oracle's E4M3 code."""
    bits = np.arange(0, 1 << 16, dtype=np.uint32)
    finite = ((bits >> 7) & 0xFF) != 0xFF
    bits = bits[finite].astype(np.uint16)
    n = (bits.shape[0] + 63) // 64 * 64
    pad = np.zeros(n, np.uint16)
    pad[: bits.shape[0]] = bits
    tok = pad.reshape(-1, 1, 64)            # [T][Hkv=1][D=64]
    T = tok.shape[0]
    for scale in (1.0, 0.0071, 3.3e-3, 41.5):
        kc = torch.zeros((T // 16 + 1, 1, 16, 64), dtype=torch.uint8, device="cuda")
        vc = torch.zeros_like(kc)
        kt = torch.from_numpy(tok.view(np.int16)).view(torch.bfloat16).cuda()
        s = torch.tensor([scale], dtype=torch.float32, device="cuda")
        slots = torch.arange(T, dtype=torch.int64, device="cuda")
        cuda_lib.pa_kv_append(kc, vc, kt, kt, slots, cuda_lib.PA_KV_FP8_E4M3, s, s)
        okc = np.zeros(tuple(kc.shape), np.uint8)
        ovc = np.zeros_like(okc)
        sc = np.array([scale], np.float32)
        O.kv_append(okc, ovc, tok, tok, np.arange(T, dtype=np.int64), 1, sc, sc)
        got = kc.cpu().numpy()
        assert np.array_equal(got, okc), f"scale {scale}: {(got != okc).sum()} codes differ"


def test_copy_blocks_bit_exact(O, cuda_lib):
    g = torch.Generator().manual_seed(5)
    nb, hkv, d = 50, 4, 128
    k = torch.randn((nb, hkv, 16, d), generator=g).to(torch.bfloat16)
    v = torch.randn((nb, hkv, 16, d), generator=g).to(torch.bfloat16)
    perm = torch.randperm(nb, generator=g).numpy()
    pairs = np.stack([perm[:12], perm[12:24]], axis=1).astype(np.int32)
    kc, vc = k.cuda(), v.cuda()
    cuda_lib.pa_copy_blocks(kc, vc, torch.from_numpy(pairs).cuda())
    ok, ov = bf16_bits(k), bf16_bits(v)
    O.copy_blocks(ok, ov, pairs)
    assert np.array_equal(bf16_bits(kc), ok) and np.array_equal(bf16_bits(vc), ov)


def test_out_of_pool_slot_is_flagged_not_written(cuda_lib):
    kc = torch.zeros((4, 2, 16, 64), dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    k = torch.ones((3, 2, 64), dtype=torch.bfloat16, device="cuda")
    slots = torch.tensor([0, 64, -1], dtype=torch.int64, device="cuda")   # 64 = 4 blocks * 16: outside
    assert cuda_lib.pa_get_device_error() == cuda_lib.PA_OK
    cuda_lib.pa_kv_append(kc, vc, k, k, slots)
    assert cuda_lib.pa_get_device_error() == cuda_lib.PA_EDEVICE_OOB
    assert cuda_lib.pa_get_device_error() == cuda_lib.PA_OK              # cleared
    assert float(kc.float().sum()) == 2 * 64                              # only slot 0 written


@pytest.mark.parametrize("bs", [16, 32])
def test_append_int8_bit_exact(O, cuda_lib, bs):
    batch = make_batch("mha_fp8_decode", seed=33, overrides=dict(num_seqs=5, num_q_heads=4, num_kv_heads=4,
                                                               hist=("uniform", 1, 300), kv_dtype="int8",
                                                               block_size=bs))
    ref = oracle_step(batch, O)
    _, _, k, v = _gpu_step_caches(batch, cuda_lib)
    assert np.array_equal(k, ref["k_cache"]) and np.array_equal(v, ref["v_cache"])


def test_int8_quantiser_all_bf16_inputs(O, cuda_lib):
    """Every finite bf16 value, divided by several scales, quantises to the oracle's INT8 code."""
    bits = np.arange(0, 1 << 16, dtype=np.uint32)
    bits = bits[((bits >> 7) & 0xFF) != 0xFF].astype(np.uint16)
    n = (bits.shape[0] + 63) // 64 * 64
    pad = np.zeros(n, np.uint16)
    pad[: bits.shape[0]] = bits
    tok = pad.reshape(-1, 1, 64)
    T = tok.shape[0]
    for scale in (1.0, 0.0313, 7.5e-4, 3.0):
        kc = torch.zeros((T // 16 + 1, 1, 16, 64), dtype=torch.int8, device="cuda")
        kt = torch.from_numpy(tok.view(np.int16)).view(torch.bfloat16).cuda()
        s = torch.tensor([scale], dtype=torch.float32, device="cuda")
        cuda_lib.pa_kv_append(kc, kc.clone(), kt, kt, torch.arange(T, dtype=torch.int64, device="cuda"),
                              cuda_lib.PA_KV_INT8, s, s)
        okc = np.zeros(tuple(kc.shape), np.int8)
        sc = np.array([scale], np.float32)
        O.kv_append(okc, np.zeros_like(okc), tok, tok, np.arange(T, dtype=np.int64), 2, sc, sc)
        got = kc.cpu().numpy()
        assert np.array_equal(got, okc), f"scale {scale}: {(got != okc).sum()} codes differ"
