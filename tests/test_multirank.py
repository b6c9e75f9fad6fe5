"""The N>1 path of bench.py on CPU: two gloo ranks combine their own timings into whole-job figures
(max time over ranks, sum of work), as the NCCL ranks do on GPUs."""
import os
import socket

import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        times = {"step_ms": 1.0 + rank, "dec_ms": 0.5 + 0.25 * rank, "e2e_ms": 3.0 - rank}
        out = bench.combine_over_ranks(times, 1000 * (rank + 1), world, torch.device("cpu"))
        q.put((rank, out))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_max_time_and_sum_work():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in range(2):
        assert res[r] == {"step_ms": 2.0, "dec_ms": 0.75, "e2e_ms": 3.0, "bytes": 3000.0}


def test_single_rank_is_identity():
    import bench
    out = bench.combine_over_ranks({"step_ms": 1.5}, 42, 1, torch.device("cpu"))
    assert out == {"step_ms": 1.5, "bytes": 42.0}


def _tp_worker(rank, world, port, q):
    """One rank of bench.py's kv_heads partition, with the oracle standing in for the kernels: the rank runs
    the shard bench.rank_batch gives it; gathered over the ranks the outputs are the unsharded ones."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        import numpy as np
        from oracle import oracle as O
        from pagedattention_block_table_b200.inputs import make_batch
        from tests.common import oracle_step
        full = make_batch("mixed_step", seed=62, overrides=dict(
            num_seqs=5, hist=("uniform", 1, 70), share_group=0, share_prefix=0, num_q_heads=8, num_kv_heads=4,
            head_dim=64, prefill_chunks=2, chunk_len=(3, 30), chunk_hist=(1, 40)))
        part = bench.rank_batch(full, rank, world, "kv_heads")
        assert part.num_kv_heads == 4 // world and part.num_q_heads == 8 // world
        assert bench.rank_batch(full, rank, world, "replicas") is full
        res = oracle_step(part, O)
        outs = []
        for key in ("decode", "prefill"):
            t = torch.from_numpy(res[key])
            g = [torch.empty_like(t) for _ in range(world)]
            dist.all_gather(g, t)
            outs.append(torch.cat(g, dim=1).numpy())
        agg = bench.combine_over_ranks({"step_ms": 1.0 + rank}, bench.decode_bytes(part), world, torch.device("cpu"))
        if rank == 0:
            ref = oracle_step(full, O)
            work = sum(bench.decode_bytes(bench.rank_batch(full, r, world, "kv_heads")) for r in range(world))
            q.put(bool(np.array_equal(outs[0], ref["decode"]) and np.array_equal(outs[1], ref["prefill"])
                       and agg["step_ms"] == float(world) and agg["bytes"] == work))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_run_the_kv_head_partition():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_tp_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    ok = q.get(timeout=300)
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert ok


def test_bench_launches_its_own_ranks_or_fails_loudly(monkeypatch):
    import bench
    cmd = bench.relaunch_command(["--gpus", "4", "--steps", "10"], 4, 29511)
    assert cmd[1:4] == ["-m", "torch.distributed.run", "--nnodes=1"] and "--nproc-per-node=4" in cmd
    assert cmd[cmd.index("--master-addr") + 1] == "127.0.0.1" and cmd[-4:] == ["--gpus", "4", "--steps", "10"]
    # more GPUs asked than visible: a clear exit, not a silent one-GPU run
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    monkeypatch.setattr("sys.argv", ["bench.py", "--gpus", "2"])
    monkeypatch.setattr(torch.cuda, "device_count", lambda: 1)
    import pytest
    with pytest.raises(SystemExit) as e:
        bench.main()
    assert "--gpus 2" in str(e.value)
    # under torchrun, --gpus must agree with the world size
    monkeypatch.setenv("WORLD_SIZE", "4")
    with pytest.raises(SystemExit) as e:
        bench.main()
    assert "WORLD_SIZE=4" in str(e.value)
