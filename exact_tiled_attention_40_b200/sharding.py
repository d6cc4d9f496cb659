"""Host-side partitioning of attention work across ranks (one process per GPU).

Exact attention is independent per (batch, KV-head group): the query heads of
one KV head (GQA, devhandbook.co.kr "Flash Attention 2 ... PyTorch native",
example 5) never read another group's keys.  So the work shards over batch
entries or KV-head groups with no exchange step and no collective: each rank
calls the library on its own slice and writes a disjoint part of the output.
"""
from __future__ import annotations


def even_range(n: int, world: int, rank: int) -> tuple[int, int]:
    """[start, stop) of rank's share of n items; shares differ by at most one."""
    if world <= 0 or not 0 <= rank < world:
        raise ValueError("bad world/rank")
    base, extra = divmod(n, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def batch_shard(B: int, world: int, rank: int) -> tuple[int, int]:
    """Batch entries handled by `rank`."""
    return even_range(B, world, rank)


def head_shard(Hq: int, Hkv: int, world: int, rank: int):
    """(query-head range, KV-head range) handled by `rank`: whole GQA groups, so
    a rank's query heads only need its own KV heads."""
    if Hkv <= 0 or Hq % Hkv:
        raise ValueError("Hq must be a positive multiple of Hkv")
    g0, g1 = even_range(Hkv, world, rank)
    group = Hq // Hkv
    return (g0 * group, g1 * group), (g0, g1)
