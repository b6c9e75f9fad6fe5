"""Python face of the CPU oracle (``oracle.c``), fp64, for tests and baselines only.

TEST INFRASTRUCTURE: only the test-suite, the smoke check and the benchmark's
CPU-baseline leg may import this module.  The product path (the CUDA library and
its binding) never does, and fails loudly if its own extension is missing.

Every function takes NumPy arrays laid out as the CUDA library's are (bf16 values
as ``uint16`` bit patterns, E4M3 values as ``uint8`` codes, cache
``[num_blocks][num_kv_heads][16][head_dim]``) and returns NumPy arrays.  The
arithmetic lives in ``oracle.c``; this file only marshals arguments.  Where each
step comes from on the pages is stated beside the C functions.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build  # noqa: F401  (relative import when used as a package)

_lib = None


def configure(lib):
    """Declare the C signatures on a loaded oracle library."""
    P = ctypes.c_void_p
    I = ctypes.c_int
    L = ctypes.c_int64
    D = ctypes.c_double
    lib.oracle_e4m3_decode.restype = D
    lib.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
    lib.oracle_e4m3_encode.restype = ctypes.c_uint8
    lib.oracle_e4m3_encode.argtypes = [ctypes.c_float]
    lib.oracle_int8_encode.restype = ctypes.c_int8
    lib.oracle_int8_encode.argtypes = [ctypes.c_float]
    lib.oracle_kv_cache_bytes.restype = L
    lib.oracle_kv_cache_bytes.argtypes = [L, L, L, L, L, L]
    lib.oracle_kv_append.restype = I
    lib.oracle_kv_append.argtypes = [P, P, P, P, P, L, I, I, L, I, I, P, P]
    lib.oracle_copy_blocks.restype = I
    lib.oracle_copy_blocks.argtypes = [P, P, P, L, I, I, L, I, I]
    lib.oracle_swap_blocks.restype = I
    lib.oracle_swap_blocks.argtypes = [P, P, L, P, P, L, P, L, I, I, I, I]
    lib.oracle_paged_decode.restype = I
    lib.oracle_paged_decode.argtypes = [P, P, P, P, P, I, P, I, I, I, I, L, I, D, I, P, P]
    lib.oracle_paged_prefill.restype = I
    lib.oracle_paged_prefill.argtypes = [P, P, P, I, P, P, P, I, P, I, I, I, L, I, D, I, P, P]
    lib.oracle_num_threads.restype = I
    lib.oracle_num_threads.argtypes = []
    lib.oracle_set_num_threads.restype = None
    lib.oracle_set_num_threads.argtypes = [I]
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = configure(ctypes.CDLL(_build.build()))
    return _lib


class OracleError(RuntimeError):
    pass


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _check(rc, what):
    if rc != 0:
        raise OracleError(f"{what}: oracle status {rc}")


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def set_num_threads(n: int) -> None:
    """Run later oracle calls on n OpenMP threads."""
    _load().oracle_set_num_threads(int(n))


def kv_cache_bytes(layers, kv_heads, head_dim, seq_len, batch, elem_bytes) -> int:
    """KV size formula of the KV-Cache-to-vLLM page, section 2.1."""
    return int(_load().oracle_kv_cache_bytes(layers, kv_heads, head_dim, seq_len, batch, elem_bytes))


def e4m3_decode(codes) -> np.ndarray:
    """E4M3 byte codes -> float64 values (OCP FP8 definition)."""
    lib = _load()
    c = np.asarray(codes, dtype=np.uint8)
    return np.array([lib.oracle_e4m3_decode(int(x)) for x in c.ravel()], dtype=np.float64).reshape(c.shape)


def e4m3_encode(x) -> np.ndarray:
    """float32 values -> E4M3 codes, round to nearest even, saturating at +-448."""
    lib = _load()
    a = np.asarray(x, dtype=np.float32)
    return np.array([lib.oracle_e4m3_encode(float(v)) for v in a.ravel()], dtype=np.uint8).reshape(a.shape)


def int8_encode(x) -> np.ndarray:
    """float32 values -> int8 codes: round to nearest (ties to even), clamp to [-127, 127]."""
    lib = _load()
    a = np.asarray(x, dtype=np.float32)
    return np.array([lib.oracle_int8_encode(float(v)) for v in a.ravel()], dtype=np.int8).reshape(a.shape)


def kv_append(k_cache, v_cache, k, v, slot_mapping, kv_dtype=0, k_scale=None, v_scale=None):
    """Scatter token K/V rows into the paged cache in place (see ``oracle_kv_append``).
    kv_dtype 0: uint16 bf16 cache; 1: uint8 E4M3 codes; 2: int8 codes."""
    lib = _load()
    assert k_cache.flags.c_contiguous and v_cache.flags.c_contiguous
    nb, hkv, bs, d = k_cache.shape
    k = _c(k, np.uint16)
    v = _c(v, np.uint16)
    sm = _c(slot_mapping, np.int64)
    ks = None if k_scale is None else _c(k_scale, np.float32)
    vs = None if v_scale is None else _c(v_scale, np.float32)
    rc = lib.oracle_kv_append(_p(k_cache), _p(v_cache), _p(k), _p(v), _p(sm), sm.shape[0], hkv, d,
                              nb, bs, kv_dtype, _p(ks), _p(vs))
    _check(rc, "kv_append")


def copy_blocks(k_cache, v_cache, pairs):
    """Copy whole blocks src -> dst for each pair, in place (see ``oracle_copy_blocks``)."""
    lib = _load()
    nb, hkv, bs, d = k_cache.shape
    pr = _c(pairs, np.int32).reshape(-1, 2)
    rc = lib.oracle_copy_blocks(_p(k_cache), _p(v_cache), _p(pr), pr.shape[0], hkv, d, nb, bs,
                                k_cache.dtype.itemsize)
    _check(rc, "copy_blocks")


def swap_blocks(dst_k, dst_v, src_k, src_v, pairs):
    """Copy whole blocks src (of the source pool) -> dst (of the destination pool), in place."""
    lib = _load()
    nbd, hkv, bs, d = dst_k.shape
    nbs = src_k.shape[0]
    assert src_k.shape[1:] == dst_k.shape[1:] and src_k.dtype == dst_k.dtype
    pr = _c(pairs, np.int32).reshape(-1, 2)
    rc = lib.oracle_swap_blocks(_p(dst_k), _p(dst_v), nbd, _p(np.ascontiguousarray(src_k)),
                                _p(np.ascontiguousarray(src_v)), nbs, _p(pr), pr.shape[0], hkv, d, bs,
                                dst_k.dtype.itemsize)
    _check(rc, "swap_blocks")


def paged_decode(q, k_cache, v_cache, block_tables, context_lens, scale, kv_dtype=0,
                 k_scale=None, v_scale=None) -> np.ndarray:
    """Decode attention, fp64 output [B][Hq][D] (see ``oracle_paged_decode``)."""
    lib = _load()
    q = _c(q, np.uint16)
    b, hq, d = q.shape
    nb, hkv, bs, d2 = k_cache.shape
    assert d == d2
    bt = _c(block_tables, np.int32)
    cl = _c(context_lens, np.int32)
    out = np.zeros((b, hq, d), dtype=np.float64)
    ks = None if k_scale is None else _c(k_scale, np.float32)
    vs = None if v_scale is None else _c(v_scale, np.float32)
    rc = lib.oracle_paged_decode(_p(out), _p(q), _p(k_cache), _p(v_cache), _p(bt), bt.shape[1],
                                 _p(cl), b, hq, hkv, d, nb, bs, float(scale), kv_dtype, _p(ks), _p(vs))
    _check(rc, "paged_decode")
    return out


def paged_prefill(q, cu_q_lens, k_cache, v_cache, block_tables, context_lens, scale, kv_dtype=0,
                  k_scale=None, v_scale=None) -> np.ndarray:
    """Causal chunk attention over paged history, fp64 output [sum C][Hq][D]."""
    lib = _load()
    q = _c(q, np.uint16)
    tq, hq, d = q.shape
    nb, hkv, bs, _ = k_cache.shape
    cu = _c(cu_q_lens, np.int32)
    bt = _c(block_tables, np.int32)
    cl = _c(context_lens, np.int32)
    assert cu[-1] == tq
    out = np.zeros((tq, hq, d), dtype=np.float64)
    ks = None if k_scale is None else _c(k_scale, np.float32)
    vs = None if v_scale is None else _c(v_scale, np.float32)
    rc = lib.oracle_paged_prefill(_p(out), _p(q), _p(cu), cu.shape[0] - 1, _p(k_cache), _p(v_cache),
                                  _p(bt), bt.shape[1], _p(cl), hq, hkv, d, nb, bs, float(scale), kv_dtype,
                                  _p(ks), _p(vs))
    _check(rc, "paged_prefill")
    return out
