"""Splitting decode work across GPUs (one process per GPU).

Decode attention over a packed cache is independent per (batch row, KV head): no unit
reads another unit's cache, so N GPUs each take their own units and no data crosses
between them while the kernels run. The only communication is host-side bookkeeping:
agreeing on the timing window (a barrier) and reducing the measured totals (sum of
keys, max of time), done with torch.distributed over whichever backend the caller
initialised (NCCL on GPUs, gloo in CPU tests).
"""
from __future__ import annotations

from dataclasses import dataclass


@dataclass(frozen=True)
class Shard:
    """The units one rank owns: batch rows [b0, b1) and KV heads [h0, h1)."""

    b0: int
    b1: int
    h0: int
    h1: int

    @property
    def units(self) -> int:
        return max(0, self.b1 - self.b0) * max(0, self.h1 - self.h0)


def _split(n: int, parts: int, i: int) -> tuple[int, int]:
    base, extra = divmod(n, parts)
    start = i * base + min(i, extra)
    return start, start + base + (1 if i < extra else 0)


def shard_units(batch: int, h_kv: int, rank: int, world: int) -> Shard:
    """Contiguous batch rows per rank when there are at least as many rows as ranks;
    otherwise each batch row's KV heads are split among the ranks that share it."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("bad rank/world")
    if batch >= world:
        b0, b1 = _split(batch, world, rank)
        return Shard(b0, b1, 0, h_kv)
    # fewer rows than ranks: ranks r*batch//world.. share a row, splitting its heads
    row = rank * batch // world
    first = -(-row * world // batch)           # first rank assigned to this row
    last = -(-(row + 1) * world // batch)      # one past the last
    h0, h1 = _split(h_kv, last - first, rank - first)
    return Shard(row, row + 1, h0, h1)


def aggregate(local_keys: float, local_ms: float, dist=None) -> tuple[float, float]:
    """(total keys over ranks, max time over ranks in ms). With dist None: single rank."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(local_keys), float(local_ms)
    import torch
    backend = dist.get_backend()
    dev = torch.device("cuda", torch.cuda.current_device()) if backend == "nccl" else torch.device("cpu")
    k = torch.tensor([float(local_keys)], dtype=torch.float64, device=dev)
    t = torch.tensor([float(local_ms)], dtype=torch.float64, device=dev)
    dist.all_reduce(k, op=dist.ReduceOp.SUM)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(k.item()), float(t.item())


# ------------------------------------------------------------------ one sequence over GPUs
def token_range(length: int, rank: int, world: int, tile: int = 64) -> tuple[int, int]:
    """Tokens [t0, t1) of a sequence of `length` tokens that rank `rank` of `world` holds
    when one long sequence is split over GPUs: whole 64-token tiles, as even as possible,
    in rank order (the last rank holds the newest tokens)."""
    if world < 1 or not 0 <= rank < world or length < 0:
        raise ValueError("bad rank/world/length")
    tiles = -(-length // tile)
    a, b = _split(tiles, world, rank)
    return min(length, a * tile), min(length, b * tile)


def split_sequence_decode(partial_fn, merge_fn, dist=None):
    """Decode attention of one query step over a sequence split across ranks: each rank
    computes the partial records (m, l, o') of its own token range (partial_fn() -> tensor
    [B, h_q, 130]), all ranks exchange them (one all-gather: the only data-path
    collective), and each rank merges them in rank order (merge_fn(stacked [world, B, h_q,
    130]) -> output). With dist None or a single rank, the local records are merged alone.
    The records are a few hundred bytes per query head, whatever the context length."""
    import torch
    rec = partial_fn()
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return merge_fn(rec[None])
    world = dist.get_world_size()
    parts = [torch.empty_like(rec) for _ in range(world)]
    dist.all_gather(parts, rec.contiguous())
    return merge_fn(torch.stack(parts))
