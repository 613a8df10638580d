"""Token data parallelism and expert parallelism for the block across ranks
(one process per GPU).

Every token's output depends only on that token (the block has no
cross-token term: the router, the experts and the restore all act per
token), so a batch shards across ranks by rows with no exchange on the data
path; each rank holds all weights.  Collectives appear only around the data
path: reassembling a sharded batch (``gather_rows``) and taking the slowest
rank's time (``max_over_ranks``).  Works with the ``nccl`` and ``gloo``
backends.

Expert parallelism (``ep_forward``) splits the experts instead: rank r holds
experts [r*E/N, (r+1)*E/N) and its own tokens.  Each rank routes and permutes
its tokens (the rows for every rank's experts are then contiguous), an
all-to-all sends the rows with their expert ids and router weights to the
experts' ranks, which sort them by expert and run their experts; a second
all-to-all returns the weighted rows, and each rank restores its tokens (plus
the shared expert on its own tokens).  Every row and the restore use the
block's own arithmetic and order, so the output equals the single-GPU block's
bit for bit.  The pages claim no expert parallelism; this form is the
library's own.
"""

from __future__ import annotations

import dataclasses
from typing import Callable, List, Optional, Sequence, Tuple

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


# ---------------------------------------------------------------------------
# expert parallelism
# ---------------------------------------------------------------------------
class CudaBackend:
    """The compute steps of ``ep_forward``: the library's kernels (C ABI)."""

    weight_dtype = torch.float32  # router weights of the rows

    def route(self, x, Wr, bias, cfg):
        from . import ops
        return ops.route(x, Wr, bias, cfg)

    def permute(self, ids, w, x, cfg):
        from . import ops
        return ops.permute(ids, cfg, topk_w=w, x=x)

    def rows_expert_ids(self, offsets, E):
        from . import ops
        return ops.rows_expert_ids(offsets, E)

    def expert_rows(self, xr, offsets, w13, w2, row_dest, row_w, y_rows):
        from . import ops
        return ops.expert_rows(xr, offsets, w13, w2, row_dest, row_w=row_w, y_rows=y_rows)

    def dense_ffn(self, x, w13, w2):
        from . import ops
        return ops.dense_ffn(x, w13, w2)

    def combine_rows(self, y, row_of, top_k, shared, residual):
        from . import ops
        return ops.combine_rows(y, row_of, top_k, shared=shared, residual=residual)

    def to_host(self, t) -> List[int]:
        return [int(v) for v in t.cpu().tolist()]


def ep_split(E: int, world: int, rank: int) -> Tuple[int, int]:
    """Expert range [base, base + E/world) held by ``rank``."""
    if world <= 0 or not 0 <= rank < world or E % world != 0:
        raise ValueError("the experts must split evenly across the ranks")
    el = E // world
    return rank * el, el


def ep_send_counts(offsets: Sequence[int], E: int, world: int) -> List[int]:
    """Rows this rank sends to each rank: the expert-sorted rows of rank q's
    experts are the contiguous range [offsets[q*E/N], offsets[(q+1)*E/N])."""
    el = E // world
    return [int(offsets[(q + 1) * el] - offsets[q * el]) for q in range(world)]


def _all_to_all(t: torch.Tensor, send: Sequence[int], recv: Sequence[int], group):
    """Rows of ``t`` split by ``send`` go to the ranks in order; returns the rows
    received, ``recv[q]`` from rank q, in rank order."""
    out = torch.empty((int(sum(recv)),) + tuple(t.shape[1:]), dtype=t.dtype, device=t.device)
    dist.all_to_all_single(out, t.contiguous(), output_split_sizes=list(recv),
                           input_split_sizes=list(send), group=group)
    return out


def ep_forward(x: torch.Tensor, Wr: torch.Tensor, bias: torch.Tensor, w13_local: torch.Tensor,
               w2_local: torch.Tensor, ws13: Optional[torch.Tensor],
               ws2: Optional[torch.Tensor], cfg, group=None,
               residual: Optional[torch.Tensor] = None, backend=None) -> torch.Tensor:
    """The block on this rank's tokens ``x`` [T,H] with the experts split
    across the ranks of ``group``: ``w13_local`` / ``w2_local`` hold this rank's
    E/N experts (``ep_split``); router and shared-expert weights are whole on
    every rank.  Returns this rank's output [T,H]; every rank must call it (the
    exchanges are collectives), with any T, including 0."""
    be = backend if backend is not None else CudaBackend()
    rank, world = _world(group)
    E, k = cfg.E, cfg.top_k
    base, el = ep_split(E, world, rank)
    T = x.shape[0]
    cfg_t = dataclasses.replace(cfg, T=T)
    # 1. route and sort this rank's (token, slot) rows by expert
    if T > 0:
        ids, w = be.route(x, Wr, bias, cfg_t)
        p = be.permute(ids, w, x, cfg_t)
        offs = be.to_host(p["expert_offsets"])
        row_ids = be.rows_expert_ids(p["expert_offsets"], E)
    else:  # nothing to route; this rank still takes part in the exchanges
        p = dict(xp=x.new_empty((0, x.shape[1])),
                 row_of=torch.empty(0, dtype=torch.int32, device=x.device),
                 w_of=torch.empty(0, dtype=be.weight_dtype, device=x.device))
        offs = [0] * (E + 1)
        row_ids = torch.empty(0, dtype=torch.int32, device=x.device)
    send = ep_send_counts(offs, E, world)
    # 2. dispatch: rows, their expert ids and router weights to the experts' ranks
    if world > 1:
        dev = x.device if dist.get_backend(group) == "nccl" else torch.device("cpu")
        cnt = torch.tensor(send, dtype=torch.int64, device=dev)
        got = torch.empty_like(cnt)
        dist.all_to_all_single(got, cnt, group=group)
        recv = [int(v) for v in got.cpu().tolist()]
        xr = _all_to_all(p["xp"], send, recv, group)
        ir = _all_to_all(row_ids, send, recv, group)
        wr = _all_to_all(p["w_of"], send, recv, group)
    else:
        recv = send
        xr, ir, wr = p["xp"], row_ids, p["w_of"]
    R_in = int(sum(recv))
    # 3. this rank's experts on the received rows, results in received order
    if R_in > 0:
        cfg1 = dataclasses.replace(cfg, T=R_in, top_k=1)
        q = be.permute(ir.reshape(R_in, 1), wr.reshape(R_in, 1), xr, cfg1)
        local_offsets = q["expert_offsets"][base:base + el + 1]  # this rank's experts
        yr = be.expert_rows(q["xp"], local_offsets, w13_local, w2_local, q["tok_of"],
                            q["w_of"], R_in)
    else:
        yr = xr.new_empty((0, x.shape[1]))
    # 4. combine: the weighted rows back to their tokens' ranks, in the order sent
    yb = _all_to_all(yr, recv, send, group) if world > 1 else yr
    if T == 0:
        return x.new_empty((0, x.shape[1]))
    sh = be.dense_ffn(x, ws13, ws2) if ws13 is not None else None
    return be.combine_rows(yb, p["row_of"], k, sh, residual)
