"""Multi-process (world size 2, gloo, CPU) checks of the replica plumbing: sequence
sharding, the max-over-ranks job time, and a rank that dies being detected by the
others through a short process-group timeout instead of a hang."""
import os
import socket
import time

import pytest
import torch.multiprocessing as mp

from bit_compressed_decode_b200 import replicas


def _port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _env(rank, world, port):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))


def _worker_ok(rank, world, port, q):
    _env(rank, world, port)
    replicas.init("gloo", timeout_s=30)
    r, w, _ = replicas.env_ranks()
    start, count = replicas.shard(1000, w, r)
    t = replicas.max_over_ranks(1.5 + r)            # rank 1 is the slow one
    q.put((r, start, count, t))
    import torch.distributed as dist
    dist.barrier()
    dist.destroy_process_group()


def _worker_dies(rank, world, port, q):
    _env(rank, world, port)
    replicas.init("gloo", timeout_s=3)
    import torch.distributed as dist
    if rank == 1:
        q.put((rank, "left"))
        q.close()
        q.join_thread()                             # flush the report before leaving
        os._exit(0)                                 # leaves between steps, nothing in flight
    t0 = time.time()
    try:
        dist.barrier()
        q.put((rank, "no error"))
    except Exception as e:                          # the timeout surfaces as an error on the host
        q.put((rank, "error", type(e).__name__, time.time() - t0))


def test_shard_covers_all_sequences():
    for total in (0, 1, 7, 512, 1000):
        for world in (1, 2, 3, 8):
            parts = [replicas.shard(total, world, r) for r in range(world)]
            assert sum(c for _, c in parts) == total
            pos = 0
            for s, c in parts:
                assert s == pos
                pos += c
            assert max(c for _, c in parts) - min(c for _, c in parts) <= 1


def test_two_ranks_shard_and_max_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _port()
    ps = [ctx.Process(target=_worker_ok, args=(r, 2, port, q)) for r in range(2)]
    for p in ps:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(2))
    for p in ps:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res[0][1:3] == (0, 500) and res[1][1:3] == (500, 500)
    assert res[0][3] == res[1][3] == 2.5


def test_dead_rank_is_reported_not_hung():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _port()
    ps = [ctx.Process(target=_worker_dies, args=(r, 2, port, q)) for r in range(2)]
    for p in ps:
        p.start()
    res = {}
    for _ in range(2):
        item = q.get(timeout=120)
        res[item[0]] = item[1:]
    for p in ps:
        p.join(timeout=60)
    assert res[1] == ("left",)
    assert res[0][0] == "error" and res[0][2] < 60
