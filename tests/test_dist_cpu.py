"""Multi-rank plumbing on CPU (gloo, world size 2): batch sharding, barrier and
max-over-ranks timing as bench.py uses them on several GPUs."""
import os
import socket

import pytest

from mamba_ssd_scan_chunked_b200 import dist


def test_shard_covers_batch_once():
    for gb in (0, 1, 7, 8, 512):
        for world in (1, 2, 3, 8):
            parts = [dist.shard(gb, r, world) for r in range(world)]
            flat = [i for p in parts for i in p]
            assert flat == list(range(gb))
            assert max(map(len, parts)) - min(map(len, parts)) <= 1
    with pytest.raises(ValueError):
        dist.shard(4, 2, 2)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    pg = dist.init(world, rank, rank, backend="gloo", timeout_s=30)
    dist.barrier(pg)
    m = dist.max_over_ranks(pg, 10.0 + rank)       # e.g. ms per step measured on this rank
    mine = dist.shard(8, rank, world)
    dist.barrier(pg)
    dist.finish(pg)
    out.put((rank, m, mine))


def test_gloo_two_ranks_max_and_shards():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [11.0, 11.0]          # both ranks see the slowest rank's time
    assert res[0][2] == [0, 1, 2, 3] and res[1][2] == [4, 5, 6, 7]
