"""The oracle's pins catch plausible mistakes.  Each mutant is a copy of oracle.c with one planted
error (on the CPU, in a temporary build); the pin tests of test_oracle_pins.py run against it and at
least one of them must fail.  The real oracle passes them all (test_oracle_pins.py)."""
import ctypes
import os
import subprocess
import tempfile

import numpy as np
import pytest

from oracle import oracle as O
from tests import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle", "oracle.c")

MUTANTS = {
    "scale dropped": ("s[t] = scale * acc;", "s[t] = acc;"),
    "GQA map modulo": ("int g = h / (num_q_heads / num_kv_heads);\n            float ks",
                       "int g = h % num_kv_heads;\n            float ks"),
    "block/offset swapped": ("int64_t phys = table[t / bs];", "int64_t phys = table[t % bs];"),
    "slot offset by one": ("off = slot % bs;", "off = (slot + 1) % bs;"),
    "head/slot transposed": ("int64_t idx = ((phys * num_kv_heads + g) * bs + (t % bs)) * (int64_t)head_dim + d;",
                             "int64_t idx = ((phys * bs + (t % bs)) * num_kv_heads + g) * (int64_t)head_dim + d;"),
    "causal off by one": ("hist + i + 1,", "hist + i,"),
    "softmax not normalised": ("double p = s[t] / sum;", "double p = s[t];"),
    "max not subtracted in sum": ("s[t] = exp(s[t] - mx); sum += s[t];", "s[t] = exp(s[t] - mx); sum += exp(s[t]);"),
    "E4M3 bias 6": ("v = ldexp(1.0 + (double)m / 8.0, e - 7);", "v = ldexp(1.0 + (double)m / 8.0, e - 6);"),
    "E4M3 ties to odd": ("(above == below && (hi & 1) == 0)", "(above == below && (hi & 1) == 1)"),
    "E4M3 no saturation": ("if (a >= 448.0) return (uint8_t)(sign | 0x7E);", "if (a >= 480.0) return (uint8_t)(sign | 0x7F);"),
    "KV bytes without K+V factor": ("return 2 * layers * kv_heads", "return layers * kv_heads"),
    "copy forgets V": ("        memmove((char *)v_cache + d * block_bytes, (char *)v_cache + s * block_bytes, block_bytes);\n", ""),
    "INT8 truncates": ("float r = rintf(x);", "float r = truncf(x);"),
    "INT8 range -128": ("if (r < -127.0f) r = -127.0f;", "if (r < -128.0f) r = -128.0f;"),
    "FP8 dequant drops the scale": ("return oracle_e4m3_decode(((const uint8_t *)cache)[idx]) * (double)scale;",
                                    "return oracle_e4m3_decode(((const uint8_t *)cache)[idx]);"),
    "INT8 dequant drops the scale": ("return (double)((const int8_t *)cache)[idx] * (double)scale;",
                                     "return (double)((const int8_t *)cache)[idx];"),
    "decode V uses k_scale": ("vs = kv_dtype ? v_scale[g] : 1.0f;\n            int r = gather_kv",
                              "vs = kv_dtype ? k_scale[g] : 1.0f;\n            int r = gather_kv"),
    "prefill V uses k_scale": ("vs = kv_dtype ? v_scale[g] : 1.0f;\n            int64_t C",
                               "vs = kv_dtype ? k_scale[g] : 1.0f;\n            int64_t C"),
    "swap copies K into V": ("memcpy((char *)dst_v + d * block_bytes, (const char *)src_v + s * block_bytes",
                             "memcpy((char *)dst_v + d * block_bytes, (const char *)src_k + s * block_bytes"),
}

PIN_TESTS = [
    (pins.test_kv_cache_bytes_pages_example, {}),
    (pins.test_e4m3_decode_spec_points, {}),
    (pins.test_e4m3_encode_spec_points, {}),
    (pins.test_e4m3_encode_matches_torch_cast, {}),
    (pins.test_decode_matches_sdpa_on_unpaged_kv, dict(hq=8, hkv=2, d=64, bs=16)),
    (pins.test_prefill_matches_sdpa_with_causal_offset, {}),
    (pins.test_context_of_one_returns_v, {}),
    (pins.test_tables_read_back_each_sequences_tokens, dict(bs=16)),
    (pins.test_copy_on_write_copies_and_keeps_parent, {}),
    (pins.test_int8_encode_points, {}),
    (pins.test_int8_encode_matches_numpy, {}),
    (pins.test_one_byte_decode_matches_sdpa_on_dequantised_kv, dict(kv_dtype=1, bs=16)),
    (pins.test_one_byte_decode_matches_sdpa_on_dequantised_kv, dict(kv_dtype=2, bs=32)),
    (pins.test_one_byte_prefill_matches_sdpa_on_dequantised_kv, dict(kv_dtype=1)),
    (pins.test_one_byte_prefill_matches_sdpa_on_dequantised_kv, dict(kv_dtype=2)),
    (pins.test_swap_reads_back_each_moved_block, dict(dtype=np.uint16, bs=16)),
]


def _build_mutant(src, tmp):
    c = os.path.join(tmp, "m.c")
    so = os.path.join(tmp, "m.so")
    with open(c, "w") as f:
        f.write(src)
    subprocess.run(["gcc", "-O1", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-fno-fast-math", "-ffp-contract=off",
                    "-o", so, c, "-lm"], check=True)
    return so


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation site for {name!r} not found"
    mutated = src.replace(old, new)
    with tempfile.TemporaryDirectory() as tmp:
        so = _build_mutant(mutated, tmp)
        lib = O.configure(ctypes.CDLL(so))
        saved = O._load()
        O._lib = lib
        failed = []
        try:
            for fn, kw in PIN_TESTS:
                try:
                    fn(O, **kw)
                except Exception as e:  # an assertion, or the mutant crashing a check
                    failed.append(fn.__name__)
        finally:
            O._lib = saved
    assert failed, f"no pin caught mutant {name!r}"
