"""Multi-GPU layout of the BASA forward path: shards of (batch, head) units.

Pooling, routing and attention are computed per (batch, head) with no term
across heads, so a layer spread over N GPUs is N independent problems: rank r
owns a contiguous range of the B * heads units and runs the three kernels on
it with no collective on the data path. The only cross-rank step is the
timing reduction of a benchmark (the max over ranks of the device time).
"""
from __future__ import annotations


def unit_shard(B: int, heads: int, world: int, rank: int) -> tuple:
    """Half-open range [start, stop) of flattened (b, head) units owned by `rank`.

    Units are split as evenly as possible; the first (B*heads) % world ranks get
    one extra unit. Every unit belongs to exactly one rank.
    """
    if world < 1 or not 0 <= rank < world:
        raise ValueError("need 0 <= rank < world")
    n = B * heads
    base, extra = divmod(n, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def shard_view(x, start: int, stop: int):
    """The units [start, stop) of a [B, heads, rows, d] tensor as a [1, stop - start,
    rows, d] view of the same memory (no copy): with B and heads flattened, a range of
    units is one contiguous block, so a layer built for B = 1 and stop - start heads
    runs on it unchanged and writes its outputs in place."""
    flat = x.reshape(1, -1, *x.shape[2:])
    if flat.data_ptr() != x.data_ptr():
        raise ValueError("shard_view needs a contiguous tensor")
    return flat[:, start:stop]


def max_over_ranks(value: float, group=None) -> float:
    """Max of a per-rank scalar over the process group (identity without one)."""
    import torch
    import torch.distributed as dist

    if not dist.is_available() or not dist.is_initialized() or dist.get_world_size(group) == 1:
        return value
    backend = dist.get_backend(group)
    dev = "cuda" if backend == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())
