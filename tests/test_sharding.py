"""KV-head sharding (tensor parallelism) on the CPU: two gloo ranks each run the oracle on their
shard of a batch; gathered over the ranks the outputs equal the unsharded oracle exactly."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from pagedattention_block_table_b200 import sharding


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from oracle import oracle as O
        from pagedattention_block_table_b200.inputs import make_batch
        from tests.common import oracle_step
        batch = make_batch("mixed_step", seed=61, overrides=dict(
            num_seqs=6, hist=("uniform", 1, 90), share_group=3, share_prefix=32, num_q_heads=8, num_kv_heads=4,
            head_dim=64, prefill_chunks=2, chunk_len=(3, 30), chunk_hist=(1, 40)))
        part = sharding.shard_batch(batch, rank, world)
        res = oracle_step(part, O)
        dec = torch.from_numpy(res["decode"])
        pre = torch.from_numpy(res["prefill"])
        gd = [torch.empty_like(dec) for _ in range(world)]
        gp = [torch.empty_like(pre) for _ in range(world)]
        dist.all_gather(gd, dec)
        dist.all_gather(gp, pre)
        if rank == 0:
            full = oracle_step(batch, O)
            ok = (np.array_equal(torch.cat(gd, dim=1).numpy(), full["decode"])
                  and np.array_equal(torch.cat(gp, dim=1).numpy(), full["prefill"]))
            q.put(ok)
    finally:
        dist.destroy_process_group()


def test_two_rank_kv_head_shards_reassemble_the_unsharded_result():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    ok = q.get(timeout=300)
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert ok


def test_head_ranges():
    assert sharding.kv_head_range(1, 4, 8) == (2, 4)
    assert sharding.q_head_range(1, 4, 32, 8) == (8, 16)
    with pytest.raises(ValueError):
        sharding.kv_head_range(0, 3, 8)
