"""Host-side partitioning of attention work across ranks (one process per GPU).

Exact attention is independent per (batch, KV-head group): the query heads of
one KV head (GQA, devhandbook.co.kr "Flash Attention 2 ... PyTorch native",
example 5) never read another group's keys.  So the work shards over batch
entries or KV-head groups with no exchange step and no collective: each rank
calls the library on its own slice and writes a disjoint part of the output.
Ragged (packed) batches shard over whole sequences the same way, in contiguous
runs so that every rank's packed rows form one slice.
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


def ragged_shard(cu_seqlens_q, cu_seqlens_k, world: int, rank: int):
    """Sequences of a ragged batch handled by `rank`: a contiguous run of whole
    sequences, cut where the running work (Nq_b * Nk_b summed, the score count)
    crosses rank / world of the total, so ranks get similar work and each one's
    packed rows are one slice.

    cu_seqlens_q/k: [B + 1] offsets (any integer sequence type).  Returns
    (b0, b1, (q_lo, q_hi), (k_lo, k_hi), cu_q_local, cu_k_local): the sequence
    range, the packed row slices, and the offsets rebased to those slices.
    """
    if world <= 0 or not 0 <= rank < world:
        raise ValueError("bad world/rank")
    cq = [int(x) for x in cu_seqlens_q]
    ck = [int(x) for x in cu_seqlens_k]
    if len(cq) != len(ck) or not cq:
        raise ValueError("cu_seqlens must be [B + 1] offsets of equal length")
    B = len(cq) - 1
    work = [(cq[b + 1] - cq[b]) * max(1, ck[b + 1] - ck[b]) for b in range(B)]
    total = sum(work)
    # sequence b goes to the rank whose share holds the midpoint of its work
    owner, run = [], 0
    for w in work:
        mid2 = 2 * run + w                 # twice the midpoint, kept integral
        owner.append(min(world - 1, (mid2 * world) // (2 * total)) if total else 0)
        run += w
    mine = [b for b in range(B) if owner[b] == rank]
    if mine:
        b0, b1 = mine[0], mine[-1] + 1
    else:                                  # an empty run, placed after the ranks before it
        earlier = [b for b in range(B) if owner[b] < rank]
        b0 = b1 = (earlier[-1] + 1) if earlier else 0
    q_lo, q_hi = cq[b0], cq[b1]
    k_lo, k_hi = ck[b0], ck[b1]
    cu_q_local = [x - q_lo for x in cq[b0:b1 + 1]]
    cu_k_local = [x - k_lo for x in ck[b0:b1 + 1]]
    return b0, b1, (q_lo, q_hi), (k_lo, k_hi), cu_q_local, cu_k_local
