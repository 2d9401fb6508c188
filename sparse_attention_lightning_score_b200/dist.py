"""Host-side multi-GPU plumbing for the indexer path.

Decode requests and prefill query rows are independent problems, so the path
shards them across ranks with no collective on the data path: each rank
scores and selects its own rows.  The only cross-rank traffic is timing
(a max over ranks) and barriers, over torch.distributed (NCCL on GPUs, gloo
on CPU in the tests).

One long context can instead be split along L: rank p holds cache positions
p * shard_len .. (p + 1) * shard_len - 1 of every request, selects its own k
best (li_decode_select with values), the ranks all-gather those (score,
position) lists, and li_merge_shards takes the global top-k from them.  That
exchange is the only collective, 8 bytes per candidate.
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


def shard_lens(lens, rank: int, shard_len: int):
    """Visible positions of each request inside rank `rank`'s slice of the cache:
    clamp(len - rank * shard_len, 0, shard_len).  Works on int tensors or ints."""
    if shard_len <= 0 or rank < 0:
        raise ValueError("bad shard")
    import torch
    if isinstance(lens, torch.Tensor):
        return torch.clamp(lens - rank * shard_len, min=0, max=shard_len).to(lens.dtype)
    return max(0, min(int(lens) - rank * shard_len, shard_len))


def gather_selections(vals, idx, group=None):
    """All-gather every rank's (values [rows, k], positions [rows, k]) into
    [world, rows, k] tensors in rank order, the layout li_merge_shards reads."""
    import torch
    import torch.distributed as dist
    world = dist.get_world_size(group)
    if dist.get_backend(group) == "nccl":
        gv = torch.empty((world,) + tuple(vals.shape), dtype=vals.dtype, device=vals.device)
        gi = torch.empty((world,) + tuple(idx.shape), dtype=idx.dtype, device=idx.device)
        dist.all_gather_into_tensor(gv, vals.contiguous(), group=group)
        dist.all_gather_into_tensor(gi, idx.contiguous(), group=group)
        return gv, gi
    lv = [torch.empty_like(vals) for _ in range(world)]
    li = [torch.empty_like(idx) for _ in range(world)]
    dist.all_gather(lv, vals.contiguous(), group=group)
    dist.all_gather(li, idx.contiguous(), group=group)
    return torch.stack(lv), torch.stack(li)


def lshard_decode_select(q, w, k8_slice, ks_slice, k: int, lens, shard_len: int, group=None):
    """Decode step for contexts split along L across the ranks of `group`:
    q [B,64,128] bf16 and w [B,64] on every rank, this rank's cache slice
    k8_slice [B, shard_len, 128] / ks_slice [B, shard_len], lens [B] over the whole
    context.  Returns the global top-k positions [B, k] (and values) on every rank."""
    import torch.distributed as dist
    from . import api
    rank = dist.get_rank(group)
    local = shard_lens(lens, rank, shard_len)
    _, idx, vals = api.li_decode_select(q, w, k8_slice, ks_slice, k, lens=local, with_values=True)
    gv, gi = gather_selections(vals, idx, group)
    return api.li_merge_shards(gv, gi, shard_len, k, with_values=True)
