"""Multi-GPU plumbing for the decode step: replicas over the batch, no data exchange.

Every GQA group is independent through append, scoring, selection, gather and
attention, so N GPUs run N independent shards of the batch (one process per
GPU). The only collectives are a barrier and the max over ranks of a timed
region; nothing on the data path crosses NVLink.
"""
from __future__ import annotations

import datetime
import os
from typing import Tuple


def rank_info() -> Tuple[int, int, int]:
    """(rank, world_size, local_rank) from the launcher's environment (1 process if unset)."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def shard_batch(batch: int, world: int, rank: int) -> Tuple[int, int]:
    """Contiguous [start, stop) slice of a global batch for `rank`; sizes differ by at most 1."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"bad rank {rank} of {world}")
    base, extra = divmod(batch, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def init(backend: str = "nccl", timeout_s: int = 300):
    """Initialises the default process group when WORLD_SIZE > 1 (short timeout so that ranks
    waiting on a dead peer end with an error)."""
    import torch.distributed as dist
    _, world, _ = rank_info()
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s))
    return world


def max_over_ranks(values, device=None):
    """Element-wise max over ranks of a list of floats (identity with one process)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def barrier():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.barrier()
