"""Thin ctypes binding of ``libpagedattn.so`` (declared in ``include/pagedattn.h``).

Each function has the name of the C entry point it calls and only marshals arguments:
torch CUDA tensors become device pointers, sizes are read off tensor shapes, the stream
defaults to torch's current stream, and a non-zero status raises :class:`PagedAttnError`.
Every step of the computation runs in the library's CUDA kernels; there is no fallback.
If the library is missing this module raises on first use.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.environ.get("PAGEDATTN_LIB") or os.path.join(HERE, "libpagedattn.so")

PA_OK = 0
PA_EINVAL = -1
PA_EUNSUPPORTED = -2
PA_ECUDA = -3
PA_EDEVICE_OOB = -4
PA_EWORKSPACE = -5
PA_BLOCK_SIZE = 16
PA_KV_BF16 = 0
PA_KV_FP8_E4M3 = 1
PA_KV_INT8 = 2

# every entry point include/pagedattn.h declares
EXPORTED = (
    "pa_kv_append", "pa_copy_blocks", "pa_paged_attention_workspace_size",
    "pa_paged_attention_auto_split", "pa_paged_attention_uses_tensor_cores", "pa_paged_attention",
    "pa_paged_prefill", "pa_paged_prefill_workspace_size",
    "pa_get_device_error", "pa_status_string", "pa_kv_cache_bytes", "pa_version",
    "pa_paged_attention_noalloc", "pa_swap_blocks",
    "pa_bm_create", "pa_bm_destroy", "pa_bm_num_free", "pa_bm_add", "pa_bm_fork", "pa_bm_append", "pa_bm_free",
    "pa_bm_length", "pa_bm_tables", "pa_bm_stats", "pa_selftest_bounded_wait", "pa_bm_add_prompt",
    "pa_bm_prefix_stats", "pa_bm_set_prefix_caching", "pa_bm_commit", "pa_bm_block_size",
)
PA_ENOMEM = -6


class PagedAttnError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {pa_status_string(status)} ({status})")


_lib = None


def lib() -> ctypes.CDLL:
    """Load the CUDA library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libpagedattn.so not built ({LIB_PATH}); run "
                              "`python -m pagedattention_block_table_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, I, I64, F, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
        L.pa_kv_append.restype = I
        L.pa_kv_append.argtypes = [P, P, P, P, P, I64, I, I, I64, I, I, P, P, P]
        L.pa_copy_blocks.restype = I
        L.pa_copy_blocks.argtypes = [P, P, P, I, I, I, I64, I, I, P]
        L.pa_swap_blocks.restype = I
        L.pa_swap_blocks.argtypes = [P, P, I64, P, P, I64, P, I, I, I, I, I, P]
        L.pa_paged_attention_workspace_size.restype = SZ
        L.pa_paged_attention_workspace_size.argtypes = [I, I, I, I, I]
        L.pa_paged_attention_auto_split.restype = I
        L.pa_paged_attention_auto_split.argtypes = [I, I, I, I, I, I]
        L.pa_paged_attention_uses_tensor_cores.restype = I
        L.pa_paged_attention_uses_tensor_cores.argtypes = [I, I, I, I]
        L.pa_paged_attention.restype = I
        L.pa_paged_attention.argtypes = [P, P, P, P, P, I, P, I, I, I, I, I64, I, F, I, P, P, I, I, P, P, SZ, P]
        L.pa_paged_attention_noalloc.restype = I
        L.pa_paged_attention_noalloc.argtypes = [P, P, P, P, P, I, P, I, I, I, I, I64, F, I, P, P, I, I, P]
        L.pa_paged_prefill.restype = I
        L.pa_paged_prefill.argtypes = [P, P, P, I, P, P, P, I, P, I, I, I, I64, I, F, I, P, P, I, I, P, P, P, SZ, P]
        L.pa_paged_prefill_workspace_size.restype = SZ
        L.pa_paged_prefill_workspace_size.argtypes = [I, P, P, I, I, I, I, I, I, I]
        L.pa_get_device_error.restype = I
        L.pa_get_device_error.argtypes = [P]
        L.pa_selftest_bounded_wait.restype = I
        L.pa_selftest_bounded_wait.argtypes = [P]
        L.pa_status_string.restype = ctypes.c_char_p
        L.pa_status_string.argtypes = [I]
        L.pa_kv_cache_bytes.restype = I64
        L.pa_kv_cache_bytes.argtypes = [I64] * 6
        L.pa_version.restype = ctypes.c_char_p
        L.pa_version.argtypes = []
        U64 = ctypes.c_uint64
        L.pa_bm_create.restype = P
        L.pa_bm_create.argtypes = [I64, I, U64]
        L.pa_bm_block_size.restype = I
        L.pa_bm_block_size.argtypes = [P]
        L.pa_bm_commit.restype = I
        L.pa_bm_commit.argtypes = [P, I64, I64]
        L.pa_bm_destroy.restype = None
        L.pa_bm_destroy.argtypes = [P]
        L.pa_bm_num_free.restype = I64
        L.pa_bm_num_free.argtypes = [P]
        L.pa_bm_add.restype = I
        L.pa_bm_add.argtypes = [P, I64]
        L.pa_bm_fork.restype = I
        L.pa_bm_fork.argtypes = [P, I64, I64]
        L.pa_bm_append.restype = I
        L.pa_bm_append.argtypes = [P, I64, ctypes.c_int32, P, P, P]
        L.pa_bm_free.restype = I
        L.pa_bm_free.argtypes = [P, I64]
        L.pa_bm_length.restype = I64
        L.pa_bm_length.argtypes = [P, I64]
        L.pa_bm_tables.restype = I
        L.pa_bm_tables.argtypes = [P, P, ctypes.c_int32, P, ctypes.c_int32, P]
        L.pa_bm_stats.restype = I
        L.pa_bm_stats.argtypes = [P, P, P, P, P]
        L.pa_bm_add_prompt.restype = I
        L.pa_bm_add_prompt.argtypes = [P, I64, P, I64, P, P]
        L.pa_bm_prefix_stats.restype = I
        L.pa_bm_prefix_stats.argtypes = [P, P, P]
        L.pa_bm_set_prefix_caching.restype = I
        L.pa_bm_set_prefix_caching.argtypes = [P, I]
        _lib = L
    return _lib


# ------------------------------------------------------------------------------ helpers

def _ptr(t: Optional[torch.Tensor], name: str, dtypes=None, cuda=True):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if cuda and not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtypes is not None and t.dtype not in dtypes:
        raise TypeError(f"{name} has dtype {t.dtype}, expected one of {dtypes}")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _check(status: int, what: str):
    if status != PA_OK:
        raise PagedAttnError(status, what)


_CACHE_DTYPES = {PA_KV_BF16: (torch.bfloat16,), PA_KV_FP8_E4M3: (torch.uint8, torch.float8_e4m3fn),
                 PA_KV_INT8: (torch.int8,)}


def _cache_geometry(k_cache: torch.Tensor):
    """(num_blocks, num_kv_heads, head_dim, block_size) of a [num_blocks][Hkv][16 or 32][D] cache."""
    if k_cache.dim() != 4 or k_cache.shape[2] not in (16, 32):
        raise ValueError("cache must be [num_blocks][num_kv_heads][block_size 16 or 32][head_dim]")
    nb, hkv, bs, d = k_cache.shape
    return int(nb), int(hkv), int(d), int(bs)


# ------------------------------------------------------------------------------ entry points

def pa_version() -> str:
    return lib().pa_version().decode()


def pa_status_string(status: int) -> str:
    return lib().pa_status_string(int(status)).decode()


def pa_kv_cache_bytes(layers, kv_heads, head_dim, seq_len, batch, elem_bytes) -> int:
    return int(lib().pa_kv_cache_bytes(layers, kv_heads, head_dim, seq_len, batch, elem_bytes))


def pa_kv_append(k_cache, v_cache, k, v, slot_mapping, kv_dtype=PA_KV_BF16, k_scale=None, v_scale=None,
                 stream=None):
    nb, hkv, d, bs = _cache_geometry(k_cache)
    cd = _CACHE_DTYPES[kv_dtype]
    if k.shape != (slot_mapping.shape[0], hkv, d) or v.shape != k.shape:
        raise ValueError("k/v must be [num_tokens][num_kv_heads][head_dim]")
    st = lib().pa_kv_append(
        _ptr(k_cache, "k_cache", cd), _ptr(v_cache, "v_cache", cd), _ptr(k, "k", (torch.bfloat16,)),
        _ptr(v, "v", (torch.bfloat16,)), _ptr(slot_mapping, "slot_mapping", (torch.int64,)),
        int(slot_mapping.shape[0]), hkv, d, nb, bs, int(kv_dtype),
        _ptr(k_scale, "k_scale", (torch.float32,)), _ptr(v_scale, "v_scale", (torch.float32,)), _stream(stream))
    _check(st, "pa_kv_append")


def pa_copy_blocks(k_cache, v_cache, src_dst_pairs, kv_dtype=PA_KV_BF16, stream=None):
    nb, hkv, d, bs = _cache_geometry(k_cache)
    cd = _CACHE_DTYPES[kv_dtype]
    pairs = src_dst_pairs
    n = int(pairs.numel() // 2)
    st = lib().pa_copy_blocks(_ptr(k_cache, "k_cache", cd), _ptr(v_cache, "v_cache", cd),
                              _ptr(pairs, "src_dst_pairs", (torch.int32,)), n, hkv, d, nb, bs, int(kv_dtype),
                              _stream(stream))
    _check(st, "pa_copy_blocks")


def pa_swap_blocks(dst_k, dst_v, src_k, src_v, src_dst_pairs, kv_dtype=PA_KV_BF16, stream=None):
    """Copy whole blocks between two pools (device cache <-> pinned host pool).  Host tensors must be
    pinned (``pin_memory()``); the pairs tensor may be on the device or pinned."""
    nbd, hkv, d, bs = _cache_geometry(dst_k)
    nbs, hkv2, d2, bs2 = _cache_geometry(src_k)
    if (hkv, d, bs) != (hkv2, d2, bs2) or src_k.dtype != dst_k.dtype:
        raise ValueError("source and destination pools differ in geometry or dtype")
    for t, n in ((dst_k, "dst_k"), (dst_v, "dst_v"), (src_k, "src_k"), (src_v, "src_v"), (src_dst_pairs, "pairs")):
        if not t.is_cuda and not t.is_pinned():
            raise ValueError(f"{n} must be a CUDA tensor or pinned host memory")
    cd = _CACHE_DTYPES[kv_dtype]
    st = lib().pa_swap_blocks(
        _ptr(dst_k, "dst_k", cd, cuda=False), _ptr(dst_v, "dst_v", cd, cuda=False), nbd,
        _ptr(src_k, "src_k", cd, cuda=False), _ptr(src_v, "src_v", cd, cuda=False), nbs,
        _ptr(src_dst_pairs, "src_dst_pairs", (torch.int32,), cuda=False), int(src_dst_pairs.numel() // 2), hkv, d,
        bs, int(kv_dtype), _stream(stream))
    _check(st, "pa_swap_blocks")


def pa_paged_attention_workspace_size(num_seqs, num_q_heads, head_dim, max_context_len, split_tokens) -> int:
    return int(lib().pa_paged_attention_workspace_size(num_seqs, num_q_heads, head_dim, max_context_len,
                                                       split_tokens))


def pa_paged_attention_auto_split(num_seqs, num_q_heads, num_kv_heads, head_dim, max_context_len,
                                  kv_dtype=PA_KV_BF16) -> int:
    return int(lib().pa_paged_attention_auto_split(num_seqs, num_q_heads, num_kv_heads, head_dim,
                                                   max_context_len, kv_dtype))


def pa_paged_attention_uses_tensor_cores(num_q_heads, num_kv_heads, head_dim=128, kv_dtype=PA_KV_BF16) -> int:
    return int(lib().pa_paged_attention_uses_tensor_cores(num_q_heads, num_kv_heads, head_dim, kv_dtype))


def _host_i32(a, n, name="host_context_lens"):
    """Host pointer of an int32 array of n elements (numpy or CPU tensor), or None."""
    if a is None:
        return None
    if isinstance(a, torch.Tensor):
        if a.device.type != "cpu" or a.dtype != torch.int32 or not a.is_contiguous() or a.numel() != n:
            raise ValueError(f"{name} must be a contiguous int32 CPU tensor of {n} elements")
        return a.data_ptr()
    import numpy as np
    if not isinstance(a, np.ndarray) or a.dtype != np.int32 or not a.flags["C_CONTIGUOUS"] or a.size != n:
        raise ValueError(f"{name} must be a contiguous int32 array of {n} elements")
    return a.ctypes.data


def pa_paged_attention(out, q, k_cache, v_cache, block_tables, context_lens, scale, max_context_len,
                       kv_dtype=PA_KV_BF16, k_scale=None, v_scale=None, split_tokens=0, workspace=None,
                       stream=None, host_context_lens=None):
    """host_context_lens: optional host copy of context_lens (int32 numpy array or CPU tensor); it only
    orders the launch's work items longest first."""
    nb, hkv, d, bs = _cache_geometry(k_cache)
    cd = _CACHE_DTYPES[kv_dtype]
    b, hq, dq = q.shape
    if dq != d or out.shape != q.shape:
        raise ValueError("q/out must be [num_seqs][num_q_heads][head_dim]")
    if block_tables.dim() != 2 or block_tables.shape[0] != b or context_lens.shape != (b,):
        raise ValueError("block_tables [num_seqs][max_blocks] / context_lens [num_seqs] mismatch")
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib().pa_paged_attention(
        _ptr(out, "out", (torch.bfloat16,)), _ptr(q, "q", (torch.bfloat16,)), _ptr(k_cache, "k_cache", cd),
        _ptr(v_cache, "v_cache", cd), _ptr(block_tables, "block_tables", (torch.int32,)),
        int(block_tables.shape[1]), _ptr(context_lens, "context_lens", (torch.int32,)), b, hq, hkv, d, nb, bs,
        float(scale), int(kv_dtype), _ptr(k_scale, "k_scale", (torch.float32,)),
        _ptr(v_scale, "v_scale", (torch.float32,)), int(max_context_len), int(split_tokens),
        _host_i32(host_context_lens, b), _ptr(workspace, "workspace"), ws_bytes, _stream(stream))
    _check(st, "pa_paged_attention")


def pa_paged_attention_noalloc(out, q, k_cache, v_cache, block_tables, context_lens, scale, max_context_len,
                               kv_dtype=PA_KV_BF16, k_scale=None, v_scale=None, split_tokens=0, stream=None):
    """pa_paged_attention without a workspace argument, for callers that cannot allocate device memory:
    the split partials go to the library's static per-device scratch (shared by every call)."""
    nb, hkv, d, bs = _cache_geometry(k_cache)
    if bs != PA_BLOCK_SIZE:
        raise ValueError("pa_paged_attention_noalloc takes 16-token blocks")
    cd = _CACHE_DTYPES[kv_dtype]
    b, hq, dq = q.shape
    if dq != d or out.shape != q.shape:
        raise ValueError("q/out must be [num_seqs][num_q_heads][head_dim]")
    if block_tables.dim() != 2 or block_tables.shape[0] != b or context_lens.shape != (b,):
        raise ValueError("block_tables [num_seqs][max_blocks] / context_lens [num_seqs] mismatch")
    st = lib().pa_paged_attention_noalloc(
        _ptr(out, "out", (torch.bfloat16,)), _ptr(q, "q", (torch.bfloat16,)), _ptr(k_cache, "k_cache", cd),
        _ptr(v_cache, "v_cache", cd), _ptr(block_tables, "block_tables", (torch.int32,)),
        int(block_tables.shape[1]), _ptr(context_lens, "context_lens", (torch.int32,)), b, hq, hkv, d, nb,
        float(scale), int(kv_dtype), _ptr(k_scale, "k_scale", (torch.float32,)),
        _ptr(v_scale, "v_scale", (torch.float32,)), int(max_context_len), int(split_tokens), _stream(stream))
    _check(st, "pa_paged_attention_noalloc")


def pa_paged_prefill_workspace_size(host_cu_q_lens, host_context_lens, num_q_heads, num_kv_heads, head_dim,
                                    max_blocks_per_seq, block_size, max_q_len, max_context_len) -> int:
    """Workspace bytes pa_paged_prefill needs with these host lengths (int32 numpy arrays or CPU tensors)."""
    n = len(host_context_lens)
    return int(lib().pa_paged_prefill_workspace_size(
        n, _host_i32(host_cu_q_lens, n + 1, "host_cu_q_lens"), _host_i32(host_context_lens, n), int(num_q_heads),
        int(num_kv_heads), int(head_dim), int(max_blocks_per_seq), int(block_size), int(max_q_len),
        int(max_context_len)))


def pa_paged_prefill(out, q, cu_q_lens, k_cache, v_cache, block_tables, context_lens, scale, max_q_len,
                     max_context_len, kv_dtype=PA_KV_BF16, k_scale=None, v_scale=None, stream=None,
                     host_cu_q_lens=None, host_context_lens=None, workspace=None):
    """host_cu_q_lens / host_context_lens: optional host copies of the length arrays (int32 numpy arrays or CPU
    tensors, the same values); with them the launch is planned, and `workspace` (a CUDA tensor of at least
    pa_paged_prefill_workspace_size bytes) holds the partials of split key ranges."""
    nb, hkv, d, bs = _cache_geometry(k_cache)
    cd = _CACHE_DTYPES[kv_dtype]
    tq, hq, dq = q.shape
    n = int(cu_q_lens.shape[0]) - 1
    if dq != d or out.shape != q.shape:
        raise ValueError("q/out must be [total_q][num_q_heads][head_dim]")
    if block_tables.dim() != 2 or block_tables.shape[0] != n or context_lens.shape != (n,):
        raise ValueError("block_tables [num_chunks][max_blocks] / context_lens [num_chunks] mismatch")
    st = lib().pa_paged_prefill(
        _ptr(out, "out", (torch.bfloat16,)), _ptr(q, "q", (torch.bfloat16,)),
        _ptr(cu_q_lens, "cu_q_lens", (torch.int32,)), n, _ptr(k_cache, "k_cache", cd),
        _ptr(v_cache, "v_cache", cd), _ptr(block_tables, "block_tables", (torch.int32,)),
        int(block_tables.shape[1]), _ptr(context_lens, "context_lens", (torch.int32,)), hq, hkv, d, nb, bs,
        float(scale), int(kv_dtype), _ptr(k_scale, "k_scale", (torch.float32,)),
        _ptr(v_scale, "v_scale", (torch.float32,)), int(max_q_len), int(max_context_len),
        _host_i32(host_cu_q_lens, n + 1, "host_cu_q_lens"), _host_i32(host_context_lens, n),
        _ptr(workspace, "workspace"), 0 if workspace is None else workspace.numel() * workspace.element_size(),
        _stream(stream))
    _check(st, "pa_paged_prefill")


def pa_selftest_bounded_wait(stream=None):
    """Launch the library's never-completing bounded wait (it gives up after 0.2 s and sets the error word)."""
    _check(lib().pa_selftest_bounded_wait(_stream(stream)), "pa_selftest_bounded_wait")


def pa_get_device_error(stream=None) -> int:
    """Synchronise the stream; return PA_EDEVICE_OOB (and clear it) if a kernel flagged a bad index."""
    return int(lib().pa_get_device_error(_stream(stream)))


# ------------------------------------------------------------------------------ host block manager
# Same names as the C entry points; `bm` is the opaque handle pa_bm_create returns.

def pa_bm_create(num_blocks: int, block_size: int = PA_BLOCK_SIZE, shuffle_seed: int = 0):
    h = lib().pa_bm_create(int(num_blocks), int(block_size), int(shuffle_seed))
    if not h:
        raise PagedAttnError(PA_EINVAL, "pa_bm_create")
    return h


def pa_bm_block_size(bm) -> int:
    return int(lib().pa_bm_block_size(bm))


def pa_bm_commit(bm, seq_id: int, tokens_written: int):
    """Report the K/V of the first tokens_written tokens of seq_id written: its full prompt blocks within
    them join the prefix tree."""
    _check(lib().pa_bm_commit(bm, int(seq_id), int(tokens_written)), "pa_bm_commit")


def pa_bm_destroy(bm):
    lib().pa_bm_destroy(bm)


def pa_bm_num_free(bm) -> int:
    return int(lib().pa_bm_num_free(bm))


def pa_bm_add(bm, seq_id: int):
    _check(lib().pa_bm_add(bm, int(seq_id)), "pa_bm_add")


def pa_bm_add_prompt(bm, seq_id: int, tokens):
    """Register a sequence with a prompt of token ids, sharing the blocks of earlier prompts that start
    alike.  Returns (slots int64 array of the tokens not shared, number of shared tokens)."""
    import numpy as np
    toks = np.ascontiguousarray(tokens, np.int32)
    slots = np.zeros(max(1, toks.shape[0]), np.int64)
    reused = ctypes.c_int64(0)
    st = lib().pa_bm_add_prompt(bm, int(seq_id), toks.ctypes.data_as(ctypes.c_void_p), int(toks.shape[0]),
                                slots.ctypes.data_as(ctypes.c_void_p), ctypes.byref(reused))
    _check(st, "pa_bm_add_prompt")
    return slots[:toks.shape[0] - reused.value], int(reused.value)


def pa_bm_set_prefix_caching(bm, keep_freed: bool):
    _check(lib().pa_bm_set_prefix_caching(bm, 1 if keep_freed else 0), "pa_bm_set_prefix_caching")


def pa_bm_prefix_stats(bm) -> dict:
    v = [ctypes.c_int64(0) for _ in range(2)]
    _check(lib().pa_bm_prefix_stats(bm, *[ctypes.byref(x) for x in v]), "pa_bm_prefix_stats")
    return dict(cached_blocks=v[0].value, tokens_reused=v[1].value)


def pa_bm_fork(bm, parent: int, child: int):
    _check(lib().pa_bm_fork(bm, int(parent), int(child)), "pa_bm_fork")


def pa_bm_append(bm, seq_id: int, n_tokens: int):
    """Reserve slots for n_tokens new tokens.  Returns (slots int64 array, cow pair or None)."""
    import numpy as np
    slots = np.zeros(max(1, n_tokens), np.int64)
    pair = np.zeros(2, np.int32)
    ncow = ctypes.c_int32(0)
    st = lib().pa_bm_append(bm, int(seq_id), int(n_tokens), slots.ctypes.data_as(ctypes.c_void_p),
                            pair.ctypes.data_as(ctypes.c_void_p), ctypes.byref(ncow))
    _check(st, "pa_bm_append")
    return slots[:n_tokens], (pair.copy() if ncow.value else None)


def pa_bm_free(bm, seq_id: int):
    _check(lib().pa_bm_free(bm, int(seq_id)), "pa_bm_free")


def pa_bm_length(bm, seq_id: int) -> int:
    return int(lib().pa_bm_length(bm, int(seq_id)))


def pa_bm_tables(bm, seq_ids, max_blocks_per_seq: int):
    """Block tables int32 [n][max_blocks_per_seq] (-1 padded) and lengths int32 [n] of seq_ids."""
    import numpy as np
    ids = np.ascontiguousarray(seq_ids, np.int64)
    tables = np.empty((ids.shape[0], max_blocks_per_seq), np.int32)
    lens = np.empty(ids.shape[0], np.int32)
    st = lib().pa_bm_tables(bm, ids.ctypes.data_as(ctypes.c_void_p), ids.shape[0],
                            tables.ctypes.data_as(ctypes.c_void_p), int(max_blocks_per_seq),
                            lens.ctypes.data_as(ctypes.c_void_p))
    _check(st, "pa_bm_tables")
    return tables, lens


def pa_bm_stats(bm) -> dict:
    v = [ctypes.c_int64(0) for _ in range(4)]
    _check(lib().pa_bm_stats(bm, *[ctypes.byref(x) for x in v]), "pa_bm_stats")
    return dict(tokens_stored=v[0].value, blocks_used=v[1].value, blocks_shared=v[2].value, cow_copies=v[3].value)
