"""Host-side multi-GPU plumbing for the indexer path.

Decode requests and prefill query rows are independent problems, so the path
shards them across ranks with no collective on the data path: each rank
scores and selects its own rows.  The only cross-rank traffic is timing
(a max over ranks) and barriers, over torch.distributed (NCCL on GPUs, gloo
on CPU in the tests).
"""
from __future__ import annotations

import datetime
import os
from typing import List, Tuple


def env_rank() -> Tuple[int, int, int]:
    """(rank, world_size, local_rank) from the torchrun environment (defaults: one process)."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def shard_rows(total: int, world: int, rank: int) -> Tuple[int, int]:
    """Contiguous [start, end) slice of `total` independent rows for `rank`;
    slices differ in size by at most one and cover every row exactly once."""
    if world < 1 or not (0 <= rank < world) or total < 0:
        raise ValueError("bad shard request")
    base, extra = divmod(total, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def init(backend: str, device=None, timeout_s: int = 120):
    """Initialise the default process group with a short timeout (ranks that wait
    on a missing peer end with an error instead of hanging)."""
    import torch.distributed as dist
    kw = {"timeout": datetime.timedelta(seconds=timeout_s)}
    if device is not None and backend == "nccl":
        kw["device_id"] = device
    dist.init_process_group(backend, **kw)
    return dist


def max_over_ranks(values: List[float], device=None) -> List[float]:
    """Element-wise max of per-rank values (identity when not distributed)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return list(values)
    t = torch.tensor(values, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()
