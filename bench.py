"""Benchmark of one paged-attention serving step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one pass of the hot path over one batch: copy-on-write forks (when the workload
has shared prefixes), kv_append of every new token, paged decode attention (split-K + LSE
reduce) and paged prefill (when the workload has prefill chunks).  The default workload is the
Llama-3-8B-shaped decode batch (64 sequences, 32 query / 8 KV heads, head_dim 128, 16-token
blocks, contexts uniform in [513, 4097] after the append, blocks shuffled over a pool 1.25x the
need).  Inputs are seeded synthetic data; every input is resident in HBM before timing and
the KV pool (about 1.2 GB) is larger than L2, so every step streams the cache from HBM.

metric: KV-read HBM GB/s = algorithmic bytes of the decode attention (every cached K and V
element once, plus q, out, tables and lengths) / step time, summed over ranks.
One JSON line on rank 0.  With --impl reference the CPU oracle is timed instead on a bounded
sample of the same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "paged-attn decode: KV-read HBM GB/s (% of peak), sequence-steps/s"
DEFAULT_WORKLOAD = "llama3_8b_decode"
FALLBACK_HBM_GBS = 6650.0


# ----------------------------------------------------------------------------- helpers

def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


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


def bf16_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return float(json.load(f)["bf16_tflops"]), "measured (burst)"
    return 1590.0, "fallback"


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


class ClockSampler:
    """Polls SM clock, max clock and throttle reasons through NVML while the timed region runs."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
        0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
        0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
    }

    def __init__(self, index: int, period_s: float = 0.005):
        self.samples, self.reasons, self.max_mhz = [], 0, None
        self.period = period_s
        self._stop = threading.Event()
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
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                self.reasons |= int(self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h))
            except Exception:
                pass
            time.sleep(self.period)

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
        if d.get("source_digest") != source_digest():
            return None
        return d
    except Exception:
        return None


def combine_over_ranks(times_ms: dict, bytes_per_step: int, world: int, device) -> dict:
    """Whole-job figures from every rank's own timings: each time is the MAX over ranks (the job is
    as slow as its slowest replica) and the work is the SUM of the ranks' bytes per step."""
    keys = sorted(times_ms)
    t = torch.tensor([float(times_ms[k]) for k in keys] + [float(bytes_per_step)], dtype=torch.float64,
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


def run_ours(args, rank, world, local_rank):
    from pagedattention_block_table_b200 import binding as B
    from pagedattention_block_table_b200.inputs import make_batch
    from pagedattention_block_table_b200.runner import DeviceStep

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    B.lib()
    batch = make_batch(args.workload, device=dev)
    st = DeviceStep(batch, device=dev, split_tokens=args.split or None)
    st.fill_history()
    torch.cuda.synchronize(dev)
    stream = torch.cuda.current_stream(dev)

    launches = (1 if batch.cow_pairs.shape[0] else 0) + 1 + (1 if batch.num_decode else 0) \
        + (1 if st.workspace is not None else 0) + (1 if st.max_q else 0)

    for _ in range(max(3, args.warmup)):
        st.step()
    torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()

    K = args.steps
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    d0 = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    d1 = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    p1 = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    # The step value replays the K steps from CUDA graphs of G steps each, so that the Python launch path
    # (ctypes marshalling, the GIL shared with the clock sampler) cannot leave gaps between kernels.  The
    # graph holds the same launches as st.step(), with their programmatic (PDL) dependencies.
    G = next(g for g in (10, 8, 5, 4, 2, 1) if K % g == 0) if not args.no_graph else 0
    graph = None
    if G:
        try:
            graph = torch.cuda.CUDAGraph()
            # thread_local: the capture rules apply to this thread only, not to NCCL's helper threads
            with torch.cuda.graph(graph, stream=torch.cuda.Stream(dev), capture_error_mode="thread_local"):
                for _ in range(G):
                    st.step()
            torch.cuda.synchronize(dev)
            for _ in range(2):
                graph.replay()
            torch.cuda.synchronize(dev)
        except RuntimeError as e:            # capture refused: time stream launches instead, and say so
            print(f"bench: CUDA graph capture failed ({e}); timing stream launches", file=sys.stderr)
            graph, G = None, 0
            torch.cuda.synchronize(dev)
    with ClockSampler(local_rank) as clk:
        # the step value: K steps back to back, no event between the kernels (an event record between
        # two launches ends the programmatic overlap of the second with the first)
        torch.cuda.synchronize(dev)
        ev0.record(stream)
        if graph is not None:
            for _ in range(K // G):
                graph.replay()
        else:
            for i in range(K):
                st.step()
        ev1.record(stream)
        torch.cuda.synchronize(dev)
        # the same K steps again with events around each attention call: the kernels' own durations
        for i in range(K):
            st.fork()
            st.append()
            d0[i].record(stream)
            st.decode()
            d1[i].record(stream)
            st.prefill()
            p1[i].record(stream)
        torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    step_ms = ev0.elapsed_time(ev1) / K
    dec_ms = sum(a.elapsed_time(b) for a, b in zip(d0, d1)) / K
    pre_ms = sum(a.elapsed_time(b) for a, b in zip(d1, p1)) / K
    if B.pa_get_device_error() != B.PA_OK:
        raise RuntimeError("device error flagged during the timed region")

    # end to end through the public API: every step copies its inputs in from pinned host memory and
    # its outputs back out; a copy stream overlaps those copies with the neighbouring steps' compute
    from pagedattention_block_table_b200.runner import HostPipeline
    pipe = HostPipeline(st)
    h2d, d2h = pipe.h2d_bytes, pipe.d2h_bytes
    for _ in range(max(3, args.warmup)):
        pipe.step()
    pipe.finish()
    torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    K2 = max(1, min(K, 500))
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(K2):
        pipe.step()
    pipe.finish()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = e0.elapsed_time(e1) / K2

    dbytes = decode_bytes(batch)
    kvb = kv_bytes(batch)
    agg = combine_over_ranks({"step_ms": step_ms, "dec_ms": dec_ms, "e2e_ms": e2e_ms}, dbytes, world, dev)
    step_ms, dec_ms, e2e_ms = agg["step_ms"], agg["dec_ms"], agg["e2e_ms"]
    peak, peak_kind = peaks()
    value = agg["bytes"] / (step_ms * 1e-3) / 1e9
    achieved = dbytes / (dec_ms * 1e-3) / 1e9
    tr = traffic_record(f"decode/{args.workload}")
    line = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": round(step_ms, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": {0: "bf16", 1: "fp8_e4m3 KV, bf16 q/out, fp32 accumulate",
                  2: "int8 KV, bf16 q/out, fp32 accumulate"}[batch.kv_dtype],
        "data": "synthetic",
        "config": {
            **workload_config(args.workload, batch),
            "split_tokens": st.split_tokens,
            "launch": f"CUDA graph of {G} steps, replayed" if G else "stream launches",
            "l2": "inputs larger than L2: KV pool %.2f GB vs 126 MB" % (2 * st.k_cache.numel() * st.k_cache.element_size() / 1e9),
            "parallelism": f"replicas x{world}",
        },
        "pct_of_peak": round(100 * value / world / peak, 2),
        "pct_of_spec_8000_gbs": round(100 * value / world / 8000.0, 2),   # B200 HBM3e datasheet figure
        "seq_steps_per_s": round(world * batch.num_decode / (step_ms * 1e-3), 1),
        "decode_kv_bytes_per_step": kvb,
        "decode_kv_unique_bytes_per_step": kv_unique_bytes(batch),
        "roofline": {
            "kernel": "pa_paged_attention (paged_decode_kernel + lse_reduce_kernel)",
            "bound": "hbm", "achieved": round(achieved, 2), "peak": peak, "unit": "GB/s",
            "frac": round(achieved / peak, 4), "peak_kind": peak_kind,
            "traffic": None if tr is None else tr.get("bytes_per_launch"),
            "algorithmic_bytes": dbytes, "avg_launch_ms": round(dec_ms, 5),
            "achieved_unique": round((dbytes - kvb + kv_unique_bytes(batch)) / (dec_ms * 1e-3) / 1e9, 2),
        },
        "e2e": {"value": round(agg["bytes"] / (e2e_ms * 1e-3) / 1e9, 2), "unit": "GB/s",
                "ms_per_step": round(e2e_ms, 5), "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h)},
        "gpu_launches": launches * K,
        "clocks": clk.summary(),
    }
    if st.max_q:
        pf = prefill_flops(batch)
        tf_peak = bf16_peak()
        line["prefill"] = {"kernel": "paged_prefill_kernel (tcgen05)", "bound": "tensor", "unit": "TFLOP/s",
                           "achieved": round(pf / (pre_ms * 1e-3) / 1e12, 2), "peak": tf_peak[0],
                           "peak_kind": tf_peak[1], "frac": round(pf / (pre_ms * 1e-3) / 1e12 / tf_peak[0], 4),
                           "flops": pf, "avg_launch_ms": round(pre_ms, 5)}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(batch, args.cpu_sample_seqs)
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


def cpu_baseline(batch, nseq, budget_s=15.0):
    """The oracle on the host cores: append + decode, one (sequence, KV head) unit at a time in order,
    until `nseq` sequences are done or about `budget_s` seconds of oracle work have been spent."""
    from oracle import oracle as O
    done_bytes, secs, units, tokens = 0, 0.0, 0, 0
    for s in range(min(nseq, batch.num_decode)):
        for g in range(batch.num_kv_heads):
            smp = _oracle_sample(batch, 1, first=s, kv_head=g)
            secs += _oracle_run(batch, smp)
            done_bytes += smp["kv_bytes"]
            units += 1
            tokens += int(smp["lens"].sum())
            if secs >= budget_s:
                break
        if secs >= budget_s:
            break
    return {"value": round(done_bytes / secs / 1e9, 4), "unit": "GB/s", "cores": O.num_threads(), "kind": "oracle",
            "sample": f"append + decode of the first {units} (sequence, KV head) units of {batch.num_decode} x "
                      f"{batch.num_kv_heads} ({tokens} token-heads), fp64, {secs:.2f} s of oracle time"}


def run_reference(args, rank, world):
    if rank != 0:
        return None
    from oracle import oracle as O
    from pagedattention_block_table_b200.inputs import make_batch
    batch = make_batch(args.workload, device="cpu")
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


# ----------------------------------------------------------------------------- main

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--split", type=int, default=0, help="split_tokens (0 = library default)")
    ap.add_argument("--no-graph", action="store_true", help="time the steps as stream launches, not graph replays")
    ap.add_argument("--cpu-sample-seqs", type=int, default=16)
    ap.add_argument("--ref-sample-seqs", type=int, default=4)
    ap.add_argument("--ref-max-steps", type=int, default=20)
    ap.add_argument("--ref-budget-s", type=float, default=60.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--mode", choices=["step", "swap"], default="step",
                    help="step: the hot-path step (default); swap: KV eviction throughput")
    args = ap.parse_args()
    if args.mode == "swap":
        print(json.dumps(run_swap(args)), flush=True)
        return

    world = int(os.environ.get("WORLD_SIZE", "1"))
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
