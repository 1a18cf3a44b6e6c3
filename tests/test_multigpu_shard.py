"""Multi-process (gloo, world size 2, CPU) checks of the request-sharding bookkeeping:
ranks own disjoint request ranges that cover the batch, timing reduces to the max over
ranks, and a rank that fails raises instead of hanging the others."""
import os
import socket

import pytest
import torch.multiprocessing as mp

from sparse_attention_decode_ls_b200 import shard


def test_request_range_partitions():
    for total in [0, 1, 7, 8, 36, 257]:
        for world in [1, 2, 3, 8]:
            ranges = [shard.request_range(total, world, r) for r in range(world)]
            assert ranges[0][0] == 0 and ranges[-1][1] == total
            for (a0, a1), (b0, b1) in zip(ranges, ranges[1:]):
                assert a1 == b0
            sizes = [b - a for a, b in ranges]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        shard.request_range(8, 2, 2)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import torch.distributed as dist
    try:
        shard.init("gloo", timeout_s=30)
        lo, hi = shard.request_range(16, world, rank)
        got = [None] * world
        dist.all_gather_object(got, (lo, hi))
        t = shard.reduce_max(10.0 + rank)
        shard.barrier()
        q.put((rank, got, t))
    finally:
        if dist.is_initialized():
            dist.destroy_process_group()


def test_gloo_two_ranks_shard_and_max():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, got, t in res:
        assert got == [(0, 8), (8, 16)]
        assert t == 11.0


def _failing_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import torch.distributed as dist
    shard.init("gloo", timeout_s=10)
    if rank == 1:
        os._exit(3)  # leaves between steps, before the next collective
    try:
        shard.reduce_max(1.0)
        q.put("no error")
    except Exception as e:  # noqa: BLE001
        q.put(type(e).__name__)
    finally:
        try:
            dist.destroy_process_group()
        except Exception:  # noqa: BLE001
            pass


def test_gloo_rank_failure_is_an_error_not_a_hang():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_failing_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    assert procs[1].exitcode == 3
    assert q.get(timeout=10) != "no error"
