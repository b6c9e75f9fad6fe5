"""The C-ABI library loads and exports every entry point include/pagedattn.h declares; host-only
calls and host-side argument checks (no kernel is launched, so no GPU is needed)."""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

from pagedattention_block_table_b200 import binding as B
from pagedattention_block_table_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pagedattn.h")


@pytest.fixture(scope="module")
def L():
    build.build()
    return B.lib()


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(pa_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_binding_set():
    assert sorted(B.EXPORTED) == _declared()


def test_library_exports_every_declared_symbol(L):
    out = subprocess.run(["nm", "-D", "--defined-only", B.LIB_PATH], capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r"\sT\s(pa_\w+)", out))
    missing = [s for s in _declared() if s not in exported]
    assert not missing, missing
    for s in _declared():
        assert hasattr(L, s)


def test_library_is_sm100a_only():
    """The build passes exactly one target, sm_100a (no PTX for other archs to JIT)."""
    assert "arch=compute_100a,code=sm_100a" in build.NVCC_FLAGS


def test_kv_cache_bytes_host_function(L):
    assert B.pa_kv_cache_bytes(32, 8, 128, 4096, 1, 2) == 536870912
    assert B.pa_kv_cache_bytes(32, 8, 128, 4096, 8, 1) == 2 * 1024 ** 3
    assert B.pa_kv_cache_bytes(-1, 8, 128, 4096, 8, 1) == -1


def test_status_strings(L):
    for s in (B.PA_OK, B.PA_EINVAL, B.PA_EUNSUPPORTED, B.PA_ECUDA, B.PA_EDEVICE_OOB, B.PA_EWORKSPACE):
        assert B.pa_status_string(s) and B.pa_status_string(s) != "unknown status"
    assert "sm_100a" in B.pa_version()


def test_decode_kernel_choice(L):
    """Groups of 4 or more query heads per KV head decode on the tensor cores over bf16 caches (up to 16 heads
    per CTA, or a multiple of 16), every group over one-byte caches at head_dim 128; the rest on the CUDA
    cores."""
    f = L.pa_paged_attention_uses_tensor_cores
    f.argtypes = [ctypes.c_int] * 4
    assert f(32, 8, 128, 0) == 1 and f(64, 8, 128, 0) == 1 and f(32, 2, 128, 0) == 1 and f(32, 1, 128, 0) == 1
    assert f(32, 8, 64, 0) == 1
    assert f(32, 8, 128, 1) == 1 and f(32, 8, 128, 2) == 1   # FP8 / INT8 caches at head_dim 128
    assert f(16, 8, 128, 1) == 1 and f(16, 8, 128, 2) == 1   # ... two query heads per KV head
    assert f(64, 64, 128, 1) == 1 and f(64, 64, 128, 2) == 1 # ... one query per KV head too
    assert f(32, 8, 64, 1) == 0                              # ... not at head_dim 64
    assert f(8, 8, 128, 0) == 0 and f(4, 2, 128, 0) == 0 and f(6, 2, 128, 0) == 0
    assert f(48, 2, 128, 0) == 0                             # a group of 24: neither <= 16 nor a multiple of 16
    assert f(32, 3, 128, 0) == -1 and f(0, 8, 128, 0) == -1 and f(32, 8, 96, 0) == -1 and f(32, 8, 128, 5) == -1


def test_workspace_size(L):
    assert B.pa_paged_attention_workspace_size(8, 32, 128, 32768, 512) == 8 * 32 * 64 * 130 * 4
    assert B.pa_paged_attention_workspace_size(8, 32, 128, 512, 512) == 0
    assert B.pa_paged_attention_workspace_size(8, 32, 128, 513, 512) == 8 * 32 * 2 * 130 * 4


def _raw_attention(L, **kw):
    args = dict(out=16, q=16, k=16, v=16, bt=16, mbs=4, cl=16, ns=2, hq=8, hkv=2, d=128, nb=10, bs=16, scale=0.1,
                dt=0, ks=None, vs=None, maxl=64, split=0, ws=None, wsb=0)
    args.update(kw)
    P = ctypes.c_void_p
    return L.pa_paged_attention(P(args["out"]), P(args["q"]), P(args["k"]), P(args["v"]), P(args["bt"]), args["mbs"],
                                P(args["cl"]), args["ns"], args["hq"], args["hkv"], args["d"], args["nb"],
                                args["bs"], args["scale"], args["dt"], P(args["ks"]) if args["ks"] else None,
                                P(args["vs"]) if args["vs"] else None, args["maxl"], args["split"], None,
                                P(args["ws"]) if args["ws"] else None, args["wsb"], None)


@pytest.mark.parametrize("bad,status", [
    (dict(hq=7), B.PA_EINVAL),                 # not a multiple of the KV heads
    (dict(d=96), B.PA_EUNSUPPORTED),           # head_dim
    (dict(dt=3), B.PA_EUNSUPPORTED),           # dtype
    (dict(dt=1), B.PA_EINVAL),                 # fp8 without scales
    (dict(split=24), B.PA_EINVAL),             # split not a multiple of 16
    (dict(q=0), B.PA_EINVAL),                  # null pointer
    (dict(out=8), B.PA_EINVAL),                # misaligned
    (dict(maxl=4096, split=512), B.PA_EWORKSPACE),  # needs a workspace, none given
    (dict(nb=0), B.PA_EINVAL),
    (dict(scale=float("nan")), B.PA_EINVAL),
    (dict(bs=8), B.PA_EUNSUPPORTED),           # block size other than 16 / 32
])
def test_attention_rejects_bad_arguments_before_launch(L, bad, status):
    assert _raw_attention(L, **bad) == status


def test_empty_batch_is_a_no_op(L):
    assert _raw_attention(L, ns=0, q=0, out=0) == B.PA_OK
    P = ctypes.c_void_p
    assert L.pa_kv_append(None, None, None, None, None, 0, 8, 128, 10, 16, 0, None, None, None) == B.PA_OK
    assert L.pa_copy_blocks(None, None, None, 0, 8, 128, 10, 16, 0, None) == B.PA_OK
    assert L.pa_kv_append(P(16), P(16), P(16), P(16), P(16), 4, 8, 96, 10, 16, 0, None, None, None) == B.PA_EUNSUPPORTED
    assert L.pa_kv_append(P(16), P(16), P(16), P(16), None, 4, 8, 128, 10, 16, 0, None, None, None) == B.PA_EINVAL
    assert L.pa_kv_append(P(16), P(16), P(16), P(16), P(16), 4, 8, 128, 10, 24, 0, None, None, None) == B.PA_EUNSUPPORTED


def test_prefill_argument_checks(L):
    P = ctypes.c_void_p
    f = L.pa_paged_prefill
    tail = (None, None, None, 0, None)   # host lengths, workspace, workspace bytes, stream
    # one-byte caches: head_dim 128 only, and both scales required
    assert f(P(16), P(16), P(16), 1, P(16), P(16), P(16), 4, P(16), 8, 2, 64, 10, 16, 0.1, 1, P(16), P(16), 16, 64,
             *tail) == B.PA_EUNSUPPORTED
    assert f(P(16), P(16), P(16), 1, P(16), P(16), P(16), 4, P(16), 8, 2, 128, 10, 16, 0.1, 1, None, P(16), 16, 64,
             *tail) == B.PA_EINVAL
    assert f(P(16), P(16), P(16), 1, P(16), P(16), P(16), 4, P(16), 8, 2, 128, 10, 16, 0.1, 5, P(16), P(16), 16, 64,
             *tail) == B.PA_EUNSUPPORTED
    # heads not a multiple of the KV heads
    assert f(P(16), P(16), P(16), 1, P(16), P(16), P(16), 4, P(16), 7, 2, 128, 10, 16, 0.1, 0, None, None, 16, 64,
             *tail) == B.PA_EINVAL
    # host lengths come in pairs
    cu = np.array([0, 16], np.int32)
    assert f(P(16), P(16), P(16), 1, P(16), P(16), P(16), 4, P(16), 8, 2, 128, 10, 16, 0.1, 0, None, None, 16, 64,
             cu.ctypes.data, None, None, 0, None) == B.PA_EINVAL


def _plan_case(chunks):
    """cu_q_lens / context_lens (host int32) of prefill chunks given as (new tokens, history) pairs."""
    c = np.array([n for n, _ in chunks], np.int32)
    cu = np.concatenate([[0], np.cumsum(c)]).astype(np.int32)
    ctx = np.array([n + h for n, h in chunks], np.int32)
    return cu, ctx


def test_prefill_plan_workspace():
    """The prefill plan splits the key ranges of CTAs that are long next to the launch's work per SM and
    asks for workspace for their partials; a launch of even CTAs needs none; a call that would split
    without enough workspace is refused before anything is launched."""
    ws = B.pa_paged_prefill_workspace_size
    # two long histories in a small launch: the long CTAs are split
    cu, ctx = _plan_case([(512, 8000), (256, 6000)])
    need = ws(cu, ctx, 32, 8, 128, 1024, 16, 512, 8512)
    assert need > 0 and need % (256 * 130 * 4) == 0
    # no host lengths: nothing planned
    assert L_ws_none() == 0
    # many equal CTAs: balanced, nothing to split
    cu2, ctx2 = _plan_case([(2048, 0)] * 40)
    assert ws(cu2, ctx2, 32, 8, 128, 128, 16, 2048, 2048) == 0
    # lengths the kernel would reject (context past max_context_len): no plan
    assert ws(cu, ctx, 32, 8, 128, 1024, 16, 512, 4096) == 0
    P = ctypes.c_void_p
    lib = B.lib()
    st = lib.pa_paged_prefill(P(16), P(16), P(16), 2, P(16), P(16), P(16), 1024, P(16), 32, 8, 128, 10, 16, 0.1, 0,
                              None, None, 512, 8512, cu.ctypes.data, ctx.ctypes.data, None, 0, None)
    assert st == B.PA_EWORKSPACE


def L_ws_none():
    return int(B.lib().pa_paged_prefill_workspace_size(2, None, None, 32, 8, 128, 1024, 16, 512, 8512))


def test_source_digest_ignores_comments_only():
    """Profiles are tied to kernel code by a digest of the sources without their comments: a comment
    edit keeps a committed DRAM measurement valid, any code edit voids it."""
    strip = build._code_only
    a = "int f() {  // returns one\n  return 1; /* the\n value */\n}\n"
    assert strip(a) == strip("int f() {\n  return 1;\n\n}  // changed comment\n")
    assert strip(a) != strip("int f() {\n  return 2;\n}\n")
