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
