"""Token data parallelism for the block across ranks (one process per GPU).

Every token's output depends only on that token (the block has no
cross-token term: the router, the experts and the restore all act per
token), so a batch shards across ranks by rows with no exchange on the data
path; each rank holds all weights.  Collectives appear only around the data
path: reassembling a sharded batch (``gather_rows``) and taking the slowest
rank's time (``max_over_ranks``).  Works with the ``nccl`` and ``gloo``
backends.
"""

from __future__ import annotations

from typing import Callable, Optional, Tuple

import torch
import torch.distributed as dist


def shard_rows(T: int, rank: int, world: int) -> Tuple[int, int]:
    """Contiguous, balanced row range [lo, hi) of ``rank``; shards differ by at most one row."""
    if world <= 0 or not 0 <= rank < world or T < 0:
        raise ValueError("bad shard request")
    base, extra = divmod(T, world)
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)


def rank_token_seed(seed: int, rank: int) -> int:
    """Seed of rank ``rank``'s own token batch in a weak-scaling run."""
    return seed + 1000 * rank


def _world(group) -> Tuple[int, int]:
    if not dist.is_available() or not dist.is_initialized():
        return 0, 1
    return dist.get_rank(group), dist.get_world_size(group)


def _coll_device(group) -> torch.device:
    backend = dist.get_backend(group)
    return torch.device("cuda", torch.cuda.current_device()) if backend == "nccl" \
        else torch.device("cpu")


def max_over_ranks(value: float, group=None) -> float:
    rank, world = _world(group)
    if world == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=_coll_device(group))
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())


def gather_rows(local: torch.Tensor, T: int, group=None) -> torch.Tensor:
    """Reassembles row shards produced under ``shard_rows`` into the [T, ...] tensor on every rank."""
    rank, world = _world(group)
    if world == 1:
        return local
    dev = local.device if dist.get_backend(group) == "nccl" else torch.device("cpu")
    sizes = [shard_rows(T, r, world) for r in range(world)]
    width = max(hi - lo for lo, hi in sizes)
    pad = torch.zeros((width,) + tuple(local.shape[1:]), dtype=local.dtype, device=dev)
    pad[: local.shape[0]] = local.to(dev)
    parts = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(parts, pad, group=group)
    return torch.cat([p[: hi - lo] for p, (lo, hi) in zip(parts, sizes)]).to(local.device)


def data_parallel_forward(x: torch.Tensor, fn: Callable[[torch.Tensor], torch.Tensor],
                          group=None, gather: bool = True) -> torch.Tensor:
    """Runs ``fn`` on this rank's rows of ``x``; returns the full output (or only the shard)."""
    rank, world = _world(group)
    lo, hi = shard_rows(x.shape[0], rank, world)
    y = fn(x[lo:hi].contiguous())
    return gather_rows(y, x.shape[0], group) if gather else y
