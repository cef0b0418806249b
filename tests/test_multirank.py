"""The N > 1 path of bench.py on CPU: two gloo ranks check that the tile
shards are disjoint (no data-path exchange is needed) and that timing is the
maximum over ranks."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    import datetime

    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import bench
    ids = bench.rank_layer_ids(rank, 3)
    gathered = [None] * world
    dist.all_gather_object(gathered, ids)
    t = bench.max_over_ranks(10.0 + rank)
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, gathered, t))


def test_two_rank_shards_and_max_timing():
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
    for rank, gathered, t in res:
        flat = [i for ids in gathered for i in ids]
        assert len(flat) == len(set(flat)) == 6      # disjoint shards
        assert t == 11.0                             # max over ranks


def test_single_process_identity():
    import bench
    assert bench.max_over_ranks(3.5) == 3.5
    assert bench.rank_layer_ids(0, 2) == [0, 1]
