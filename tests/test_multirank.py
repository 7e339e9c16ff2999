"""The N>1 path on CPU: two gloo ranks run the benchmark's rank-level logic
(independent problems per rank, max-over-ranks timing, summed work)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import bench
    step = 10.0 + rank           # rank 1 is the slower one
    att = 8.0 + 2 * rank
    e2e = 20.0 - rank
    flops = 1e12 * (rank + 1)
    out = bench.reduce_over_ranks(step, att, e2e, flops, world, torch.device("cpu"))
    q.put((rank, out, bench.rank_seed(rank)))
    dist.barrier()
    dist.destroy_process_group()


def test_two_ranks_reduce_and_seed():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(2)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    for rank, (step, att, e2e, fl), seed in res:
        assert step == 11.0 and att == 10.0 and e2e == 20.0 and fl == 3e12
    assert res[0][2] != res[1][2]      # independent problems per rank
