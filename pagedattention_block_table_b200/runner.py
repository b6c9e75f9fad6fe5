"""One serving step over a paged KV cache, on the device, through the C ABI.

A step is what the pages describe for one iteration of a continuously batched engine
(vLLM overview page, "Continuous Batching"; Core Concepts page §3.2): forks of shared
pages are copied (copy-on-write), every request's new tokens are appended at the end of
its current block, decoding requests attend over their whole context and prefill chunks
attend causally over their history plus themselves.  This module only places tensors on
the device and calls the binding; all arithmetic runs in libpagedattn's kernels.
"""
from __future__ import annotations

from typing import Optional

import numpy as np
import torch

from . import binding as B
from .inputs import PagedBatch


class DeviceStep:
    """Device-resident state (cache, tables, inputs) of one :class:`PagedBatch` step."""

    def __init__(self, batch: PagedBatch, device="cuda", split_tokens: Optional[int] = None,
                 zero_cache: bool = True, overlap: bool = True, plan_prefill: bool = True):
        self.batch = batch
        self.device = torch.device(device)
        self.overlap = overlap
        self._side = None
        self._ev = None
        dev = self.device
        nb, hkv, d = batch.num_blocks, batch.num_kv_heads, batch.head_dim
        self.kv_dtype = batch.kv_dtype
        cdt = {0: torch.bfloat16, 1: torch.uint8, 2: torch.int8}[batch.kv_dtype]
        alloc = torch.zeros if zero_cache else torch.empty
        bs = batch.block_size
        self.k_cache = alloc((nb, hkv, bs, d), dtype=cdt, device=dev)
        self.v_cache = alloc((nb, hkv, bs, d), dtype=cdt, device=dev)
        self.k_scale = None if batch.k_scale is None else batch.k_scale.to(dev, torch.float32).contiguous()
        self.v_scale = None if batch.v_scale is None else batch.v_scale.to(dev, torch.float32).contiguous()

        nd = batch.num_decode
        ctx = batch.context_lens
        self.dec_tables = torch.from_numpy(batch.decode_tables).to(dev)
        self.dec_lens_host = np.ascontiguousarray(ctx[:nd], dtype=np.int32)   # orders the decode launch
        self.dec_lens = torch.from_numpy(self.dec_lens_host).to(dev)
        self.dec_max_len = int(ctx[:nd].max()) if nd else 0
        self.pre_tables = torch.from_numpy(batch.prefill_tables).to(dev)
        self.pre_lens_host = np.ascontiguousarray(ctx[nd:], dtype=np.int32)   # plan the prefill launch
        self.pre_cu_host = np.ascontiguousarray(batch.cu_q_lens, dtype=np.int32)
        self.pre_lens = torch.from_numpy(self.pre_lens_host.copy()).to(dev)
        self.pre_max_len = int(ctx[nd:].max()) if ctx.shape[0] > nd else 0
        self.cu_q = torch.from_numpy(batch.cu_q_lens).to(dev)
        self.max_q = int(batch.new_lens[nd:].max()) if ctx.shape[0] > nd else 0
        self.q_dec = batch.q_decode.to(dev).contiguous()
        self.q_pre = batch.q_prefill.to(dev).contiguous()
        self.out_dec = torch.empty_like(self.q_dec)
        self.out_pre = torch.empty_like(self.q_pre)
        self.cow = torch.from_numpy(np.ascontiguousarray(batch.cow_pairs)).to(dev)
        rows = torch.from_numpy(batch.step_rows()).to(batch.tok_k.device)
        self.k_new = batch.tok_k.index_select(0, rows).to(dev).contiguous()
        self.v_new = batch.tok_v.index_select(0, rows).to(dev).contiguous()
        self.step_slots = torch.from_numpy(batch.step_slots).to(dev)

        hq = batch.num_q_heads
        if split_tokens is None:
            split_tokens = batch.split_tokens or 0
        if split_tokens == 0 and nd:
            split_tokens = B.pa_paged_attention_auto_split(nd, hq, hkv, d, self.dec_max_len, self.kv_dtype)
        self.split_tokens = split_tokens
        ws = B.pa_paged_attention_workspace_size(nd, hq, d, self.dec_max_len, split_tokens) if nd else 0
        self.workspace = torch.empty(max(ws, 16) // 4 + 4, dtype=torch.float32, device=dev) if ws else None
        self.plan_prefill = plan_prefill and self.max_q > 0
        pws = 0
        if self.plan_prefill:
            pws = B.pa_paged_prefill_workspace_size(self.pre_cu_host, self.pre_lens_host, hq, hkv, d,
                                                    batch.prefill_tables.shape[1], bs, self.max_q, self.pre_max_len)
        self.pre_workspace = torch.empty(pws // 4 + 4, dtype=torch.float32, device=dev) if pws else None

    # ------------------------------------------------------------------ set-up (not part of a step)
    def fill_history(self, chunk_tokens: int = 1 << 16):
        """Write every sequence's history into the cache (the earlier prefills and decodes)."""
        b = self.batch
        slots = torch.from_numpy(b.setup_slots)
        n = slots.shape[0]
        for lo in range(0, n, chunk_tokens):
            hi = min(n, lo + chunk_tokens)
            k = b.tok_k[lo:hi].to(self.device).contiguous()
            v = b.tok_v[lo:hi].to(self.device).contiguous()
            B.pa_kv_append(self.k_cache, self.v_cache, k, v, slots[lo:hi].to(self.device).contiguous(),
                           self.kv_dtype, self.k_scale, self.v_scale)

    # ------------------------------------------------------------------ the step
    def fork(self, stream=None):
        if self.cow.shape[0]:
            B.pa_copy_blocks(self.k_cache, self.v_cache, self.cow, self.kv_dtype, stream)

    def append(self, stream=None):
        B.pa_kv_append(self.k_cache, self.v_cache, self.k_new, self.v_new, self.step_slots, self.kv_dtype,
                       self.k_scale, self.v_scale, stream)

    def decode(self, stream=None, split_tokens: Optional[int] = None):
        if self.batch.num_decode == 0:
            return
        B.pa_paged_attention(self.out_dec, self.q_dec, self.k_cache, self.v_cache, self.dec_tables, self.dec_lens,
                             self.batch.scale, self.dec_max_len, self.kv_dtype, self.k_scale, self.v_scale,
                             self.split_tokens if split_tokens is None else split_tokens, self.workspace, stream,
                             host_context_lens=self.dec_lens_host)

    def prefill(self, stream=None):
        if self.max_q == 0:
            return
        plan = self.plan_prefill
        B.pa_paged_prefill(self.out_pre, self.q_pre, self.cu_q, self.k_cache, self.v_cache, self.pre_tables,
                           self.pre_lens, self.batch.scale, self.max_q, self.pre_max_len, self.kv_dtype,
                           k_scale=self.k_scale, v_scale=self.v_scale, stream=stream,
                           host_cu_q_lens=self.pre_cu_host if plan else None,
                           host_context_lens=self.pre_lens_host if plan else None,
                           workspace=self.pre_workspace if plan else None)

    def step(self, stream=None):
        """copy-on-write forks -> append -> decode attention and prefill attention.

        Decode and prefill both read the cache the append has just written and write separate outputs,
        so with ``overlap`` (and both present) the decode runs on a second stream beside the prefill:
        the HBM-bound decode CTAs fill the SMs the tensor-bound prefill leaves idle in its last waves.
        """
        s = stream if stream is not None else torch.cuda.current_stream(self.device)
        self.fork(s)
        self.append(s)
        if self.overlap and self.batch.num_decode and self.max_q:
            if self._side is None:
                self._side = torch.cuda.Stream(device=self.device)
                self._ev = (torch.cuda.Event(), torch.cuda.Event())
            self._ev[0].record(s)
            self._side.wait_event(self._ev[0])
            self.decode(self._side)
            self.prefill(s)
            self._ev[1].record(self._side)
            s.wait_event(self._ev[1])
        else:
            self.decode(s)
            self.prefill(s)



class HostPipeline:
    """Serving steps fed from host memory, double-buffered: while the device computes step i, a copy
    stream brings step i+1's inputs (queries, new K/V, slots, tables, lengths) in from pinned host
    memory and takes step i-1's outputs back out.  Every step still moves all of its own inputs and
    outputs across the host link; the copies only overlap the computation instead of preceding it.

    The inputs of a step travel as one packed buffer (one host-to-device copy) and its outputs as one
    (one device-to-host copy).  Each of the two slots runs its step as a CUDA graph captured once on
    that slot's buffers (``use_graphs``), so the host issues a handful of calls per step instead of a
    launch per kernel; the graphs keep the host-side parameters of the :class:`DeviceStep` (maximum
    length, split, the host copy of the lengths that orders the launch), as the eager launches do.
    """

    IN_KEYS = ("q_dec", "k_new", "v_new", "step_slots", "dec_tables", "dec_lens", "q_pre")
    OUT_KEYS = ("out_dec", "out_pre")
    ALIGN = 256

    @classmethod
    def _layout(cls, st, keys):
        off, lay = 0, []
        for k in keys:
            t = getattr(st, k)
            n = t.numel() * t.element_size()
            lay.append((k, off, n, t.dtype, tuple(t.shape)))
            off += (n + cls.ALIGN - 1) // cls.ALIGN * cls.ALIGN
        return lay, max(off, cls.ALIGN)

    @staticmethod
    def _views(buf, lay):
        return {k: buf[o:o + n].view(dt).view(shape) for k, o, n, dt, shape in lay}

    def __init__(self, st: DeviceStep, use_graphs: bool = True):
        self.st = st
        dev = st.device
        self.lay_in, nin = self._layout(st, self.IN_KEYS)
        self.lay_out, nout = self._layout(st, self.OUT_KEYS)
        self.host_in_buf = torch.empty(nin, dtype=torch.uint8).pin_memory()
        self.host_in = self._views(self.host_in_buf, self.lay_in)
        for k in self.IN_KEYS:
            self.host_in[k].copy_(getattr(st, k).detach().cpu())
        self.dev_in = [torch.empty(nin, dtype=torch.uint8, device=dev) for _ in range(2)]
        self.slots_in = [self._views(b, self.lay_in) for b in self.dev_in]
        self.dev_out = [torch.empty(nout, dtype=torch.uint8, device=dev) for _ in range(2)]
        self.slots_out = [self._views(b, self.lay_out) for b in self.dev_out]
        self.host_out_buf = [torch.empty(nout, dtype=torch.uint8).pin_memory() for _ in range(2)]
        self.host_out = [tuple(self._views(b, self.lay_out)[k] for k in self.OUT_KEYS) for b in self.host_out_buf]
        self.copy = torch.cuda.Stream(device=dev)
        self.comp = torch.cuda.current_stream(dev)
        self.h2d_done = [torch.cuda.Event() for _ in range(2)]
        self.comp_done = [torch.cuda.Event() for _ in range(2)]
        self.d2h_done = [torch.cuda.Event() for _ in range(2)]
        self.graphs = [self._capture(s) for s in range(2)] if use_graphs else [None, None]
        self.i = 0

    @property
    def h2d_bytes(self) -> int:
        """Bytes copied in per step: the packed input buffer, alignment padding included."""
        return self.host_in_buf.numel()

    @property
    def d2h_bytes(self) -> int:
        """Bytes copied out per step: the packed output buffer."""
        return self.host_out_buf[0].numel()

    def _bind(self, slot: int):
        for k, t in self.slots_in[slot].items():
            setattr(self.st, k, t)
        for k, t in self.slots_out[slot].items():
            setattr(self.st, k, t)

    def _capture(self, slot: int):
        """The step on slot's buffers as a CUDA graph (None if capture is refused: eager launches)."""
        dev = self.st.device
        self._bind(slot)
        self.dev_in[slot].copy_(self.host_in_buf)
        try:
            torch.cuda.synchronize(dev)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=torch.cuda.Stream(dev), capture_error_mode="thread_local"):
                self.st.step()
            torch.cuda.synchronize(dev)
            return g
        except RuntimeError:
            torch.cuda.synchronize(dev)
            return None

    def _load(self, slot: int):
        with torch.cuda.stream(self.copy):
            if self.i >= 2:
                self.copy.wait_event(self.comp_done[slot])      # slot's previous step has read its inputs
            self.dev_in[slot].copy_(self.host_in_buf, non_blocking=True)
            self.h2d_done[slot].record(self.copy)

    def step(self):
        """Run one step on the inputs already in flight, and start the next step's input copies."""
        s = self.i % 2
        if self.i == 0:
            self._load(0)
        self.comp.wait_event(self.h2d_done[s])
        if self.i >= 2:
            self.comp.wait_event(self.d2h_done[s])              # output slot free again
        if self.graphs[s] is not None:
            with torch.cuda.stream(self.comp):
                self.graphs[s].replay()
        else:
            self._bind(s)
            self.st.step(self.comp)
        self.comp_done[s].record(self.comp)
        self.i += 1
        self._load(self.i % 2)
        with torch.cuda.stream(self.copy):
            self.copy.wait_event(self.comp_done[s])
            self.host_out_buf[s].copy_(self.dev_out[s], non_blocking=True)
            self.d2h_done[s].record(self.copy)

    def finish(self):
        """Wait for the last outputs to reach the host."""
        torch.cuda.current_stream(self.st.device).wait_stream(self.copy)
