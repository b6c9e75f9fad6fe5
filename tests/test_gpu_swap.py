"""GPU parity of pa_swap_blocks (KV eviction to pinned host memory and back) against the oracle:
bit-exact, for bf16 and FP8 pools, in both directions."""
import numpy as np
import pytest
import torch

from pagedattention_block_table_b200.inputs import bf16_bits

pytestmark = pytest.mark.gpu


def _np(t):
    t = t.cpu()
    return bf16_bits(t) if t.dtype == torch.bfloat16 else t.numpy().copy()


@pytest.mark.parametrize("dtype,d,bs", [(torch.bfloat16, 128, 16), (torch.uint8, 128, 16), (torch.bfloat16, 64, 16),
                                        (torch.bfloat16, 128, 32)])
def test_swap_out_and_in_bit_exact(O, cuda_lib, dtype, d, bs):
    B = cuda_lib
    g = torch.Generator().manual_seed(9)
    nb_dev, nb_host, hkv = 40, 24, 8
    kv_dtype = B.PA_KV_BF16 if dtype == torch.bfloat16 else B.PA_KV_FP8_E4M3

    def rnd(n):
        if dtype == torch.bfloat16:
            return torch.randn((n, hkv, bs, d), generator=g).to(dtype)
        return torch.randint(0, 256, (n, hkv, bs, d), generator=g, dtype=torch.uint8)

    dk, dv = rnd(nb_dev).cuda(), rnd(nb_dev).cuda()
    hk, hv = rnd(nb_host).pin_memory(), rnd(nb_host).pin_memory()
    perm_d = torch.randperm(nb_dev, generator=g)[:10].int()
    perm_h = torch.randperm(nb_host, generator=g)[:10].int()
    out_pairs = torch.stack([perm_d, perm_h], 1).contiguous()      # device block -> host block
    in_pairs = torch.stack([perm_h[:6], perm_d[4:10]], 1).contiguous()

    ok_h, ov_h = _np(hk), _np(hv)
    ok_d, ov_d = _np(dk), _np(dv)
    O.swap_blocks(ok_h, ov_h, ok_d, ov_d, out_pairs.numpy())
    B.pa_swap_blocks(hk, hv, dk, dv, out_pairs.cuda(), kv_dtype)
    torch.cuda.synchronize()
    assert np.array_equal(_np(hk), ok_h) and np.array_equal(_np(hv), ov_h)

    O.swap_blocks(ok_d, ov_d, ok_h, ov_h, in_pairs.numpy())
    B.pa_swap_blocks(dk, dv, hk, hv, in_pairs.pin_memory(), kv_dtype)
    torch.cuda.synchronize()
    assert np.array_equal(_np(dk), ok_d) and np.array_equal(_np(dv), ov_d)
    assert B.pa_get_device_error() == B.PA_OK


def test_swap_rejects_pageable_host_memory(cuda_lib):
    import ctypes
    B = cuda_lib
    dk = torch.zeros((4, 2, 16, 64), dtype=torch.bfloat16, device="cuda")
    hk = torch.zeros((4, 2, 16, 64), dtype=torch.bfloat16)              # pageable
    pairs = torch.tensor([[0, 1]], dtype=torch.int32, device="cuda")
    P = ctypes.c_void_p
    st = B.lib().pa_swap_blocks(P(hk.data_ptr()), P(hk.data_ptr()), 4, P(dk.data_ptr()), P(dk.data_ptr()), 4,
                                P(pairs.data_ptr()), 1, 2, 64, 16, 0, None)
    assert st == B.PA_EINVAL


def test_swap_out_of_range_pair_is_flagged(cuda_lib):
    B = cuda_lib
    dk = torch.zeros((4, 2, 16, 64), dtype=torch.bfloat16, device="cuda")
    hk = torch.ones((4, 2, 16, 64), dtype=torch.bfloat16).pin_memory()
    pairs = torch.tensor([[0, 9]], dtype=torch.int32, device="cuda")
    B.pa_swap_blocks(hk, hk, dk, dk, pairs)
    assert B.pa_get_device_error() == B.PA_EDEVICE_OOB
    assert float(hk.float().sum()) == hk.numel()
