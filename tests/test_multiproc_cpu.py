"""Multi-rank host logic of bench.py on CPU with the gloo backend (world size 2):
per-rank sequence seeds, max-over-ranks timing and whole-job throughput."""
import os
import socket

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
    local_ms = 10.0 + 5.0 * rank          # rank 1 is the slow one
    ms = bench.max_over_ranks(local_ms, dist, "cpu")
    seeds = [None] * world
    dist.all_gather_object(seeds, bench.rank_seed(rank))
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, ms, seeds, bench.job_tokens_per_s(world, 50, ms)))


def test_two_ranks_gloo():
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
    for rank, ms, seeds, tps in res:
        assert ms == 15.0                      # every rank sees the slowest rank's time
        assert len(set(seeds)) == 2            # the ranks decode different sequences
        assert abs(tps - 2 * 8 * 50 / 0.015) < 1e-6
