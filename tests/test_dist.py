"""Replica plumbing on CPU: batch shards and the max-over-ranks timing (gloo, 2 ranks)."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

from kv_cache_offload_nosa_b200 import dist as D


def test_shards_cover_the_batch_exactly():
    for batch in (1, 7, 16, 64):
        for world in (1, 2, 3, 8):
            spans = [D.shard_batch(batch, world, r) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == batch
            for (a, b), (c, _) in zip(spans, spans[1:]):
                assert b == c
            sizes = [b - a for a, b in spans]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        D.shard_batch(4, 2, 2)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    D.init("gloo", timeout_s=60)
    D.barrier()
    got = D.max_over_ranks([float(rank) * 10 + 1, 5.0 - rank])
    q.put((rank, got, D.shard_batch(16, world, rank)))
    import torch.distributed as dist
    dist.destroy_process_group()


def test_gloo_two_ranks_max_and_shards():
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
    for rank, got, span in res:
        assert got == [11.0, 5.0]
    assert [s for _, _, s in res] == [(0, 8), (8, 16)]
