"""Host side of the context-parallel split (CPU): page-aligned shards that cover every
request, and the candidate / partial exchange layout over two gloo ranks."""
import os
import socket

import torch
import torch.multiprocessing as mp

from sparse_attention_decode_ls_b200 import cp


def test_shard_ranges_cover_page_aligned_and_balanced():
    for lens in ([1], [64], [65], [64 * 900 + 13, 64 * 700, 3000], [1048576] * 4):
        for world in (1, 2, 3, 8):
            rows = cp.shard_ranges(lens, world)
            for L, row in zip(lens, rows):
                assert row[0][0] == 0 and row[-1][1] == L
                for (a0, a1), (b0, b1) in zip(row, row[1:]):
                    assert a1 == b0
                for a, b in row:
                    assert a <= b and (a % 64 == 0 or a == b == L)  # an empty shard sits at the end
                pages = [-(-(b - a) // 64) for a, b in row]
                assert max(pages) - min(pages) <= 1


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import torch.distributed as dist
    try:
        dist.init_process_group("gloo", rank=rank, world_size=world)
        # each rank's [B, k] candidates carry its rank in the positions: the gathered
        # [world, B, k] tensor must come back in rank (shard) order
        local = torch.full((2, 5), rank, dtype=torch.int32) * 1000 + torch.arange(5, dtype=torch.int32)
        got = cp.all_gather(local, world)
        q.put((rank, got.tolist()))
    finally:
        if dist.is_initialized():
            dist.destroy_process_group()


def test_gloo_two_ranks_gather_in_shard_order():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = dict(q.get(timeout=10) for _ in range(2))
    for rank in (0, 1):
        got = torch.tensor(res[rank])
        assert got.shape == (2, 2, 5)
        for r in range(2):
            assert (got[r] // 1000 == r).all()
    assert cp.all_gather(torch.ones(3), 1).shape == (1, 3)
