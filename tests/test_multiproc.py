"""The N > 1 path of bench.py on CPU: two gloo ranks.

Each rank serves its own disjoint block of requests with its own allocator
(no collective on the data path); the only collectives are the barrier and
the max / sum over ranks used for timing and the whole-job byte count.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import datetime

    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    import paged_kv_cache_358_b200 as pkv

    ids = list(bench.shard_requests(32, world, rank))
    # each rank admits its own requests into its own pool and appends one token
    a = pkv.BlockAllocator(4096, 16, free_order=list(range(4095, -1, -1)))
    for i in ids:
        assert a.add_seq(i, 100 + i) == 0
    rc, per, copies = a.append(ids)
    assert rc == 0 and copies == [] and a.check()
    my_time = 1.0 + rank          # a fake per-rank step time
    t_max = bench.max_over_ranks(my_time, dist, device="cpu")
    b_sum = bench.sum_over_ranks(float(len(ids)), dist, device="cpu")
    gathered = [None] * world
    dist.all_gather_object(gathered, ids)
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, t_max, b_sum, gathered))


def test_two_rank_sharding_and_timing():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, t_max, b_sum, gathered in res:
        assert t_max == 2.0                      # max over ranks, not the local value
        assert b_sum == 64.0                     # whole-job count
        flat = sorted(i for part in gathered for i in part)
        assert flat == list(range(64))           # disjoint shards that cover every request
