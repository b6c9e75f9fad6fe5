"""Benchmark of one paged-attention serving step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--partition replicas|kv_heads]
                    [--impl ours|reference]

A step is one pass of the hot path over one batch: copy-on-write forks (when the workload has shared
prefixes), kv_append of every new token, paged decode attention (split-K + LSE reduce) and paged prefill
(when the workload has prefill chunks).  The default workload is the Llama-3-8B-shaped decode batch (64
sequences, 32 query / 8 KV heads, head_dim 128, 16-token blocks, contexts uniform in [513, 4097] after the
append, blocks shuffled over a pool 1.25x the need).  Inputs are seeded synthetic data, resident in HBM
before timing; every KV pool is larger than the 126 MB L2, so each step streams the cache from HBM.

metric: KV-read HBM GB/s = algorithmic bytes of the decode attention (every cached K and V element once,
plus q, out, tables and lengths) / step time, summed over ranks.  One JSON line on rank 0.  At one GPU the
line also carries, under "workloads", the other three full-size workloads (the continuous-batching mixed
step, the long-context batch, the MHA batch over an FP8 cache), each timed the same way with its own
fraction of the roofline.

--gpus N launches N ranks itself (one process per GPU) unless it already runs under torchrun.
--partition replicas: every rank runs the whole batch on its own pool (weak scaling, no collective);
kv_heads: rank r holds KV heads [r*Hkv/N, (r+1)*Hkv/N) of every block and the query heads that use them
(tensor parallelism, strong scaling); attention needs no exchange between ranks either way.
--impl reference: the CPU oracle timed on a bounded sample of the same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "paged-attn decode: KV-read HBM GB/s (% of peak), sequence-steps/s"
DEFAULT_WORKLOAD = "llama3_8b_decode"
SUB_WORKLOADS = ("mixed_step", "long_context_decode", "mha_fp8_decode")
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


# ----------------------------------------------------------------------------- helpers

def _peaks_file():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return json.load(f)
    return None


def peaks():
    d = _peaks_file()
    if d and "hbm_gbs" in d:
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def bf16_peak():
    d = _peaks_file()
    if d and "bf16_tflops" in d:
        return float(d["bf16_tflops"]), "measured (burst)"
    return FALLBACK_BF16_TFLOPS, "fallback"


def decode_bytes(batch) -> int:
    """Algorithmic bytes of one decode-attention call: each cached K/V element of every decoding
    sequence once, the queries, the outputs, the block-table entries used and the lengths."""
    nd = batch.num_decode
    ctx = batch.context_lens[:nd].astype(np.int64)
    e = 1 if batch.kv_dtype else 2
    kv = int(ctx.sum()) * 2 * batch.num_kv_heads * batch.head_dim * e
    qo = 2 * nd * batch.num_q_heads * batch.head_dim * 2
    tables = int(((ctx + batch.block_size - 1) // batch.block_size).sum()) * 4 + 4 * nd
    return kv + qo + tables


def prefill_flops(batch) -> int:
    """4 * D * Hq * sum over chunk rows of the keys each row attends (QK^T and PV, causal)."""
    tot = 0
    ctx = batch.context_lens
    for s in range(batch.num_decode, batch.num_seqs):
        C = int(batch.new_lens[s])
        H = int(ctx[s]) - C
        tot += C * H + C * (C + 1) // 2
    return 4 * batch.head_dim * batch.num_q_heads * tot


def kv_unique_bytes(batch) -> int:
    """Bytes of the distinct cache slots the decode reads: a prefix block shared by several sequences
    counts once (it is stored once in HBM; the other readers can be served from L2)."""
    nd = batch.num_decode
    e = 1 if batch.kv_dtype else 2
    slots = []
    for s in range(nd):
        L = int(batch.context_lens[s])
        t = np.arange(L, dtype=np.int64)
        bs = batch.block_size
        slots.append(batch.block_tables[s, t // bs].astype(np.int64) * bs + t % bs)
    n = np.unique(np.concatenate(slots)).shape[0] if slots else 0
    return int(n) * 2 * batch.num_kv_heads * batch.head_dim * e


def kv_bytes(batch) -> int:
    nd = batch.num_decode
    e = 1 if batch.kv_dtype else 2
    return int(batch.context_lens[:nd].astype(np.int64).sum()) * 2 * batch.num_kv_heads * batch.head_dim * e


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


class ClockSampler:
    """Polls SM clock, max clock and throttle reasons through NVML while the timed regions run."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
        0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
        0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
    }

    def __init__(self, index: int, period_s: float = 0.002):
        self.samples, self.reasons, self.max_mhz = [], 0, None
        self.period = period_s
        self._stop = threading.Event()
        self._on = threading.Event()
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # NVML unavailable: report no clocks rather than guess
            self.err = str(e)

    def _run(self):
        while not self._stop.is_set():
            if self._on.is_set():
                try:
                    self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                    self.reasons |= int(self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h))
                except Exception:
                    pass
            time.sleep(self.period)

    def timed(self):
        """Context manager: sample only while a timed region runs."""
        sampler = self

        class _T:
            def __enter__(self):
                sampler._on.set()

            def __exit__(self, *a):
                sampler._on.clear()
        return _T()

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self.ok:
            self.t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz, "reasons": names,
                "samples": len(self.samples)}


def traffic_record(kernel_tag: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on the current sources."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    try:
        with open(p) as f:
            d = json.load(f).get(kernel_tag)
        if not d:
            return None
        from pagedattention_block_table_b200.build import source_digest
        if d.get("source_digest") != source_digest(d.get("sources")):
            return None
        return d
    except Exception:
        return None


def combine_over_ranks(times_ms: dict, work_per_step: float, world: int, device) -> dict:
    """Whole-job figures from every rank's own timings: each time is the MAX over ranks (the job is
    as slow as its slowest rank) and the work is the SUM of the ranks' work per step."""
    keys = sorted(times_ms)
    t = torch.tensor([float(times_ms[k]) for k in keys] + [float(work_per_step)], dtype=torch.float64,
                     device=device)
    if world > 1:
        mx = t[:-1].clone()
        torch.distributed.all_reduce(mx, op=torch.distributed.ReduceOp.MAX)
        tot = t[-1:].clone()
        torch.distributed.all_reduce(tot, op=torch.distributed.ReduceOp.SUM)
        t = torch.cat([mx, tot])
    out = {k: float(v) for k, v in zip(keys, t[:-1].tolist())}
    out["bytes"] = float(t[-1])
    return out


def graph_steps(K: int) -> int:
    """Steps per captured CUDA graph: the largest of 10, 8, 5, 4, 2, 1 that divides K."""
    return next(g for g in (10, 8, 5, 4, 2, 1) if K % g == 0)


def capture(fn, G: int, dev):
    """A CUDA graph of G calls of fn (the library's launches keep their programmatic dependencies), or
    None if capture is refused."""
    try:
        graph = torch.cuda.CUDAGraph()
        # thread_local: the capture rules apply to this thread only, not to NCCL's helper threads
        with torch.cuda.graph(graph, stream=torch.cuda.Stream(dev), capture_error_mode="thread_local"):
            for _ in range(G):
                fn()
        torch.cuda.synchronize(dev)
        for _ in range(2):
            graph.replay()
        torch.cuda.synchronize(dev)
        return graph
    except RuntimeError as e:
        print(f"bench: CUDA graph capture failed ({e}); timing stream launches", file=sys.stderr)
        torch.cuda.synchronize(dev)
        return None


def time_calls(fn, K: int, dev, use_graph: bool, clk) -> tuple:
    """Average ms of one call of fn over K calls run back to back (from CUDA graphs of several calls when
    use_graph), timed with CUDA events on the launching stream, synchronised on both sides."""
    G = graph_steps(K) if use_graph else 0
    graph = capture(fn, G, dev) if G else None
    stream = torch.cuda.current_stream(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    with clk.timed():
        e0.record(stream)
        if graph is not None:
            for _ in range(K // G):
                graph.replay()
        else:
            for _ in range(K):
                fn()
        e1.record(stream)
        torch.cuda.synchronize(dev)
    how = f"CUDA graph of {G} calls, replayed" if graph is not None else "stream launches"
    del graph
    return e0.elapsed_time(e1) / K, how


# ----------------------------------------------------------------------------- our arm

def workload_config(name, batch) -> dict:
    """The workload's identifying sizes (the same keys on both arms)."""
    return {
        "workload": name,
        "num_seqs": batch.num_decode, "num_q_heads": batch.num_q_heads, "num_kv_heads": batch.num_kv_heads,
        "head_dim": batch.head_dim, "block_size": batch.block_size, "num_blocks": batch.num_blocks,
        "context_tokens": int(batch.context_lens[:batch.num_decode].sum()),
        "prefill_chunks": int(batch.num_seqs - batch.num_decode), "cow_pairs": int(batch.cow_pairs.shape[0]),
    }


def rank_batch(full, rank: int, world: int, partition: str):
    """The part of the workload rank `rank` of `world` runs: all of it (replicas), or its KV heads of every
    block and the query heads that use them (kv_heads, tensor parallelism)."""
    if partition == "kv_heads" and world > 1:
        from pagedattention_block_table_b200 import sharding
        return sharding.shard_batch(full, rank, world)
    if partition not in ("replicas", "kv_heads"):
        raise ValueError(partition)
    return full


def launches_per_step(st) -> int:
    """Kernels of this library one step launches: fork, append, decode, LSE reduce, prefill (when present)."""
    b = st.batch
    return ((1 if b.cow_pairs.shape[0] else 0) + 1 + (1 if b.num_decode else 0)
            + (1 if st.workspace is not None else 0) + (1 if st.max_q else 0)
            + (1 if st.max_q and st.pre_workspace is not None else 0))


def decode_kernel_label(batch) -> str:
    """Which decode kernel pa_paged_attention runs for this batch (the library decides)."""
    from pagedattention_block_table_b200 import binding as B
    tc = B.pa_paged_attention_uses_tensor_cores(batch.num_q_heads, batch.num_kv_heads, batch.head_dim,
                                                batch.kv_dtype)
    k = "paged_decode_mma_kernel (mma.sync)" if tc == 1 else "paged_decode_kernel"
    return f"pa_paged_attention ({k} + lse_reduce_kernel)"


def prefill_kernel_label(batch, split=False) -> str:
    """The prefill kernel pa_paged_prefill runs for this batch's cache (and the merge of split key ranges)."""
    k = ("paged_prefill_kernel (tcgen05, f16 products on converted one-byte codes)" if batch.kv_dtype
         else "paged_prefill_kernel (tcgen05)")
    return k + (" + prefill_combine_kernel" if split else "")


def workload_batch(name, device, num_seqs=0):
    """The named workload's synthetic batch; num_seqs > 0 keeps its shapes and length distribution but
    draws that many sequences (a smaller case of the same workload, for profiling)."""
    from pagedattention_block_table_b200.inputs import WORKLOADS, make_batch
    ov = None
    if num_seqs:
        ov = {"num_seqs": num_seqs}
        hist = WORKLOADS[name]["hist"]
        if hist[0] == "fixed":
            ov["hist"] = ("fixed", list(hist[1])[:num_seqs])
    return make_batch(name, device=device, overrides=ov)


def measure(name, dev, K, W, args, rank, world, clk, e2e=False):
    """Time one workload on this rank: the whole step, the decode call alone and the prefill call alone
    (each from CUDA graphs of back-to-back calls), and optionally the end-to-end host-fed step."""
    from pagedattention_block_table_b200 import binding as B
    from pagedattention_block_table_b200.runner import DeviceStep, HostPipeline

    full = workload_batch(name, dev, args.num_seqs if name == args.workload else 0)
    batch = rank_batch(full, rank, world, args.partition)
    st = DeviceStep(batch, device=dev, split_tokens=args.split or None, overlap=not args.no_overlap)
    st.fill_history()
    torch.cuda.synchronize(dev)
    for _ in range(max(3, W)):
        st.step()
    torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    use_graph = not args.no_graph
    step_ms, launch = time_calls(st.step, K, dev, use_graph, clk)
    dec_ms = time_calls(st.decode, K, dev, use_graph, clk)[0] if batch.num_decode else 0.0
    pre_ms = time_calls(st.prefill, K, dev, use_graph, clk)[0] if st.max_q else 0.0
    if world > 1:
        torch.distributed.barrier()
    if B.pa_get_device_error() != B.PA_OK:
        raise RuntimeError(f"device error flagged while timing {name}")
    res = dict(batch=batch, full=full, st=st, step_ms=step_ms, dec_ms=dec_ms, pre_ms=pre_ms, launch=launch)
    if e2e:
        # end to end through the public API: every step copies its inputs in from pinned host memory and
        # its outputs back out; a copy stream overlaps those copies with the neighbouring steps' compute
        pipe = HostPipeline(st)
        for _ in range(max(3, W)):
            pipe.step()
        pipe.finish()
        torch.cuda.synchronize(dev)
        if world > 1:
            torch.distributed.barrier()
        K2 = max(1, min(K, 500))
        stream = torch.cuda.current_stream(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with clk.timed():
            e0.record(stream)
            for _ in range(K2):
                pipe.step()
            pipe.finish()
            e1.record(stream)
            torch.cuda.synchronize(dev)
        res.update(e2e_ms=e0.elapsed_time(e1) / K2, h2d=pipe.h2d_bytes, d2h=pipe.d2h_bytes)
        if B.pa_get_device_error() != B.PA_OK:
            raise RuntimeError(f"device error flagged in the end-to-end leg of {name}")
    return res


def sub_record(name, dev, args, clk):
    """The workloads sub-record of one more full-size workload at one GPU: decode GB/s (logical and unique
    bytes) and prefill TFLOP/s, each against its measured peak."""
    K = max(10, min(args.steps, args.sub_steps))
    m = measure(name, dev, K, args.warmup, args, 0, 1, clk)
    batch, st = m["batch"], m["st"]
    peak, peak_kind = peaks()
    rec = {"config": {**workload_config(name, batch), "split_tokens": st.split_tokens}, "steps": K,
           "ms_per_step": round(m["step_ms"], 5), "launch": m["launch"]}
    if batch.num_decode:
        db, kvb, kvu = decode_bytes(batch), kv_bytes(batch), kv_unique_bytes(batch)
        ach = db / (m["dec_ms"] * 1e-3) / 1e9
        rec["decode"] = {
            "kernel": decode_kernel_label(batch), "bound": "hbm",
            "unit": "GB/s", "achieved": round(ach, 2), "peak": peak, "peak_kind": peak_kind,
            "frac": round(ach / peak, 4), "avg_launch_ms": round(m["dec_ms"], 5), "algorithmic_bytes": db,
            "dtype": {0: "bf16", 1: "fp8_e4m3", 2: "int8"}[batch.kv_dtype],
        }
        if kvu != kvb:
            au = (db - kvb + kvu) / (m["dec_ms"] * 1e-3) / 1e9
            rec["decode"].update(achieved_unique=round(au, 2), frac_unique=round(au / peak, 4),
                                 unique_bytes=db - kvb + kvu)
    if st.max_q:
        pf = prefill_flops(batch)
        tp, tk = bf16_peak()
        ach = pf / (m["pre_ms"] * 1e-3) / 1e12
        rec["prefill"] = {"kernel": prefill_kernel_label(batch, st.pre_workspace is not None), "bound": "tensor",
                          "unit": "TFLOP/s",
                          "achieved": round(ach, 2), "peak": tp, "peak_kind": tk, "frac": round(ach / tp, 4),
                          "flops": pf, "avg_launch_ms": round(m["pre_ms"], 5)}
    del m, st, batch
    torch.cuda.synchronize(dev)
    torch.cuda.empty_cache()
    return rec


def run_ours(args, rank, world, local_rank):
    from pagedattention_block_table_b200 import binding as B

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    B.lib()
    K = args.steps
    with ClockSampler(local_rank) as clk:
        m = measure(args.workload, dev, K, args.warmup, args, rank, world, clk, e2e=True)
        batch, st = m["batch"], m["st"]
        dbytes = decode_bytes(batch)
        kvb = kv_bytes(batch)
        agg = combine_over_ranks({"step_ms": m["step_ms"], "dec_ms": m["dec_ms"], "e2e_ms": m["e2e_ms"],
                                  "pre_ms": m["pre_ms"]}, dbytes, world, dev)
        subs = {}
        if world == 1 and not args.no_workloads and args.workload == DEFAULT_WORKLOAD:
            for name in SUB_WORKLOADS:
                subs[name] = sub_record(name, dev, args, clk)
    step_ms, dec_ms, e2e_ms = agg["step_ms"], agg["dec_ms"], agg["e2e_ms"]
    peak, peak_kind = peaks()
    value = agg["bytes"] / (step_ms * 1e-3) / 1e9
    achieved = dbytes / (dec_ms * 1e-3) / 1e9
    tr = traffic_record(f"decode/{args.workload}")
    kvu = kv_unique_bytes(batch)
    scaling = "strong" if args.partition == "kv_heads" and world > 1 else "weak"
    line = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": round(step_ms, 5),
        "higher_is_better": True,
        "scaling": scaling,
        "vs_baseline": None,
        "dtype": {0: "bf16", 1: "fp8_e4m3 KV, bf16 q/out, fp32 accumulate",
                  2: "int8 KV, bf16 q/out, fp32 accumulate"}[batch.kv_dtype],
        "data": "synthetic",
        "config": {
            **workload_config(args.workload, m["full"]),
            "split_tokens": st.split_tokens,
            "launch": m["launch"],
            "l2": "inputs larger than L2: KV pool %.2f GB vs 126 MB" % (2 * st.k_cache.numel() * st.k_cache.element_size() / 1e9),
            "parallelism": (f"kv_heads x{world} (tensor parallel: {batch.num_kv_heads} of "
                            f"{m['full'].num_kv_heads} KV heads per rank)") if scaling == "strong"
            else f"replicas x{world}",
        },
        "pct_of_peak": round(100 * value / world / peak, 2),
        "pct_of_spec_8000_gbs": round(100 * value / world / 8000.0, 2),   # B200 HBM3e datasheet figure
        "seq_steps_per_s": round((world if scaling == "weak" else 1) * batch.num_decode / (step_ms * 1e-3), 1),
        "decode_kv_bytes_per_step": kvb,
        "decode_kv_unique_bytes_per_step": kvu,
        "roofline": {
            "kernel": decode_kernel_label(batch),
            "bound": "hbm", "achieved": round(achieved, 2), "peak": peak, "unit": "GB/s",
            "frac": round(achieved / peak, 4), "peak_kind": peak_kind,
            "traffic": None if tr is None else tr.get("bytes_per_launch"),
            "algorithmic_bytes": dbytes, "avg_launch_ms": round(dec_ms, 5),
            "timing": "decode calls alone, " + m["launch"],
            "achieved_unique": round((dbytes - kvb + kvu) / (dec_ms * 1e-3) / 1e9, 2),
        },
        "e2e": {"value": round(agg["bytes"] / (e2e_ms * 1e-3) / 1e9, 2), "unit": "GB/s",
                "ms_per_step": round(e2e_ms, 5), "h2d_bytes_per_step": int(m["h2d"]),
                "d2h_bytes_per_step": int(m["d2h"])},
        "gpu_launches": launches_per_step(st) * K,
        "clocks": clk.summary(),
    }
    if st.max_q:
        pf = prefill_flops(batch)
        tp, tk = bf16_peak()
        pre_ms = agg["pre_ms"]
        line["prefill"] = {"kernel": prefill_kernel_label(batch, st.pre_workspace is not None), "bound": "tensor",
                           "unit": "TFLOP/s",
                           "achieved": round(pf / (pre_ms * 1e-3) / 1e12, 2), "peak": tp, "peak_kind": tk,
                           "frac": round(pf / (pre_ms * 1e-3) / 1e12 / tp, 4), "flops": pf,
                           "avg_launch_ms": round(pre_ms, 5)}
    if subs:
        line["workloads"] = subs
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(batch, args.cpu_budget_s)
    return line


# ----------------------------------------------------------------------------- oracle legs

def _oracle_sample(batch, nseq, first=0, kv_head=None):
    """Host inputs of the oracle for decoding sequences first .. first+nseq-1 (all KV heads, or only
    `kv_head` and its query-head group), laid out in a fresh contiguous cache."""
    from pagedattention_block_table_b200.inputs import bf16_bits
    ctx = batch.context_lens
    seqs = list(range(first, min(first + nseq, batch.num_decode)))
    G = batch.num_q_heads // batch.num_kv_heads
    hsel = slice(None) if kv_head is None else slice(kv_head, kv_head + 1)
    qsel = slice(None) if kv_head is None else slice(kv_head * G, (kv_head + 1) * G)
    k_rows, v_rows, slots, tables, lens = [], [], [], [], []
    base = 0
    mb = max((int(ctx[s]) + 15) // 16 for s in seqs)
    for s in seqs:
        L = int(ctx[s])
        rows = torch.from_numpy(batch.seq_rows(s)[:L]).to(batch.tok_k.device)
        k_rows.append(bf16_bits(batch.tok_k.index_select(0, rows)[:, hsel]))
        v_rows.append(bf16_bits(batch.tok_v.index_select(0, rows)[:, hsel]))
        nb = (L + 15) // 16
        slots.append(base * 16 + np.arange(L, dtype=np.int64))
        t = np.full(mb, -1, np.int32)
        t[:nb] = base + np.arange(nb)
        tables.append(t)
        lens.append(L)
        base += nb
    q = bf16_bits(batch.q_decode[first:first + len(seqs)][:, qsel])
    hkv = batch.num_kv_heads if kv_head is None else 1
    ks = vs = None
    if batch.kv_dtype:
        ks = batch.k_scale.cpu().numpy()[hsel].copy()
        vs = batch.v_scale.cpu().numpy()[hsel].copy()
    return dict(k=np.concatenate(k_rows), v=np.concatenate(v_rows), slots=np.concatenate(slots),
                tables=np.stack(tables), lens=np.array(lens, np.int32), q=q, nb=base, ks=ks, vs=vs, hkv=hkv,
                kv_bytes=int(sum(lens)) * 2 * hkv * batch.head_dim * (1 if batch.kv_dtype else 2))


def _oracle_run(batch, smp):
    from oracle import oracle as O
    dt = {0: np.uint16, 1: np.uint8, 2: np.int8}[batch.kv_dtype]
    kc = np.zeros((smp["nb"], smp["hkv"], 16, batch.head_dim), dt)
    vc = np.zeros_like(kc)
    t0 = time.perf_counter()
    O.kv_append(kc, vc, smp["k"], smp["v"], smp["slots"], batch.kv_dtype, smp["ks"], smp["vs"])
    O.paged_decode(smp["q"], kc, vc, smp["tables"], smp["lens"], batch.scale, batch.kv_dtype, smp["ks"], smp["vs"])
    return time.perf_counter() - t0


def cpu_baseline(batch, budget_s=4.0):
    """The oracle on the host cores: append + decode of (sequence, KV head) units in order.  The sample is
    the units one all-core pass reaches in about `budget_s` seconds; it is run three times on all cores
    (median reported) and its first 1/cores part once on one core (scaled to the same unit)."""
    from oracle import oracle as O
    cores = O.num_threads()
    units = [(s, g) for s in range(batch.num_decode) for g in range(batch.num_kv_heads)]
    samples = [_oracle_sample(batch, 1, first=s, kv_head=g) for s, g in units[:4096]]
    n, secs, nbytes = 0, 0.0, 0
    for smp in samples:                       # pass 1 sizes the sample
        secs += _oracle_run(batch, smp)
        nbytes += smp["kv_bytes"]
        n += 1
        if secs >= budget_s:
            break
    runs = [secs]
    for _ in range(2):
        runs.append(sum(_oracle_run(batch, smp) for smp in samples[:n]))
    med = statistics.median(runs)
    n1 = max(1, n // max(1, cores))
    O.set_num_threads(1)
    try:
        t1 = sum(_oracle_run(batch, smp) for smp in samples[:n1])
    finally:
        O.set_num_threads(cores)
    b1 = sum(smp["kv_bytes"] for smp in samples[:n1])
    tokens = int(sum(int(smp["lens"].sum()) for smp in samples[:n]))
    return {"value": round(nbytes / med / 1e9, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
            "cpu_model": cpu_model(), "runs": 3, "run_s": [round(r, 3) for r in runs],
            "value_1core": round(b1 / t1 / 1e9, 4),
            "sample": f"append + decode of the first {n} (sequence, KV head) units of {batch.num_decode} x "
                      f"{batch.num_kv_heads} ({tokens} token-heads), fp64, median of 3 all-core runs; "
                      f"1 core: the first {n1} units"}


def run_reference(args, rank, world):
    if rank != 0:
        return None
    from oracle import oracle as O
    batch = workload_batch(args.workload, "cpu", args.num_seqs)
    smp = _oracle_sample(batch, args.ref_sample_seqs)
    for _ in range(max(0, min(args.warmup, 1))):
        _oracle_run(batch, smp)
    # each step is the same bounded sample; stop early once the run has used its time budget
    K = max(1, min(args.steps, args.ref_max_steps))
    times = []
    for _ in range(K):
        times.append(_oracle_run(batch, smp))
        if sum(times) > args.ref_budget_s:
            break
    K = len(times)
    secs = sum(times) / K
    value = smp["kv_bytes"] / secs / 1e9
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": round(secs * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {**workload_config(args.workload, batch), "sample_seqs": len(smp["lens"])},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": O.num_threads(), "kind": "oracle",
                         "cpu_model": cpu_model(),
                         "sample": f"append + decode of {len(smp['lens'])} of {batch.num_decode} sequences per step"},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# ----------------------------------------------------------------------------- swap (KV eviction)

def run_swap(args):
    """Throughput of pa_swap_blocks between the device cache and a pinned host pool, against the
    host link's own copy bandwidth measured in the same run (a plain pinned <-> device memcpy)."""
    from pagedattention_block_table_b200 import binding as B
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    nb_dev, nb_host, hkv, d, n = 8192, 4096, 8, 128, 1024
    g = torch.Generator(device=dev).manual_seed(1)
    dk = torch.randn((nb_dev, hkv, 16, d), device=dev, generator=g).to(torch.bfloat16)
    dv = torch.randn((nb_dev, hkv, 16, d), device=dev, generator=g).to(torch.bfloat16)
    hk = torch.empty((nb_host, hkv, 16, d), dtype=torch.bfloat16).pin_memory()
    hv = torch.empty_like(hk).pin_memory()
    gc = torch.Generator().manual_seed(2)
    out_pairs = torch.stack([torch.randperm(nb_dev, generator=gc)[:n], torch.randperm(nb_host, generator=gc)[:n]],
                            1).int().contiguous().to(dev)
    in_pairs = out_pairs[:, [1, 0]].contiguous()
    nbytes = n * 2 * hkv * 16 * d * 2

    def timed(f, k):
        for _ in range(3):
            f()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(True), torch.cuda.Event(True)
        e0.record()
        for _ in range(k):
            f()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / k

    K = max(3, min(args.steps, 50))
    t_out = timed(lambda: B.pa_swap_blocks(hk, hv, dk, dv, out_pairs), K)
    t_in = timed(lambda: B.pa_swap_blocks(dk, dv, hk, hv, in_pairs), K)
    big_h = torch.empty(nbytes // 2, dtype=torch.bfloat16).pin_memory()
    big_d = torch.empty(nbytes // 2, dtype=torch.bfloat16, device=dev)
    t_d2h = timed(lambda: big_h.copy_(big_d, non_blocking=True), K)
    t_h2d = timed(lambda: big_d.copy_(big_h, non_blocking=True), K)
    assert B.pa_get_device_error() == B.PA_OK
    gbs = lambda t: round(nbytes / (t * 1e-3) / 1e9, 2)
    return {"metric": "swap_blocks device<->pinned host GB/s", "unit": "GB/s", "blocks": n,
            "bytes_per_call": nbytes, "swap_out": gbs(t_out), "swap_in": gbs(t_in),
            "link_memcpy_d2h": gbs(t_d2h), "link_memcpy_h2d": gbs(t_h2d),
            "frac_out": round(t_d2h / t_out, 3), "frac_in": round(t_h2d / t_in, 3), "steps": K}


# ----------------------------------------------------------------------------- launch

def _free_port() -> int:
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def relaunch_command(argv, n: int, port: int) -> list:
    """The torchrun command that runs this script on n local ranks with the same arguments."""
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
            "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.abspath(__file__), *argv]


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--num-seqs", type=int, default=0,
                    help="draw this many sequences of the workload instead of its own count (profiling)")
    ap.add_argument("--partition", choices=["replicas", "kv_heads"], default="replicas",
                    help="N>1: whole batch per rank (weak scaling) or KV heads split over the ranks (strong)")
    ap.add_argument("--split", type=int, default=0, help="split_tokens (0 = library default)")
    ap.add_argument("--no-graph", action="store_true", help="time the steps as stream launches, not graph replays")
    ap.add_argument("--no-overlap", action="store_true",
                    help="run a step's decode and prefill one after the other on one stream")
    ap.add_argument("--no-workloads", action="store_true", help="skip the other full-size workloads at N=1")
    ap.add_argument("--sub-steps", type=int, default=50, help="timed steps of each of the other workloads")
    ap.add_argument("--cpu-budget-s", type=float, default=4.0)
    ap.add_argument("--ref-sample-seqs", type=int, default=4)
    ap.add_argument("--ref-max-steps", type=int, default=20)
    ap.add_argument("--ref-budget-s", type=float, default=60.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--mode", choices=["step", "swap"], default="step",
                    help="step: the hot-path step (default); swap: KV eviction throughput")
    return ap.parse_args(argv)


def main():
    args = parse_args()
    if args.mode == "swap":
        print(json.dumps(run_swap(args)), flush=True)
        return
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if "WORLD_SIZE" not in os.environ and args.gpus > 1:
        # one process per GPU: launch the ranks ourselves
        if args.gpus > torch.cuda.device_count():
            raise SystemExit(f"bench: --gpus {args.gpus} but only {torch.cuda.device_count()} CUDA devices visible")
        cmd = relaunch_command(sys.argv[1:], args.gpus, _free_port())
        raise SystemExit(subprocess.call(["timeout", "-k", "60", "1800", *cmd]))
    if args.gpus != world:
        raise SystemExit(f"bench: --gpus {args.gpus} but WORLD_SIZE={world}")
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        # the oracle runs on rank 0's host cores only; other ranks have nothing to do
        if rank == 0:
            print(json.dumps(run_reference(args, rank, world)), flush=True)
        return
    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        line = run_ours(args, rank, world, local_rank)
        if rank == 0 and line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
