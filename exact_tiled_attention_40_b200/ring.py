"""Sequence-sharded exact attention over ranks (one process per GPU).

Long contexts (devhandbook.co.kr, "Flash Attention 2 ... PyTorch native",
section 1 and the comparison table of section 2: 32K to 128K+ tokens) can be
split along the sequence.  The sequence is cut into 2W equal chunks and rank r
holds chunks r and 2W-1-r of Q, K and V ("zigzag"), so that under the causal
mask every rank has the same work.  The K/V chunks travel around a ring of
ranks: at step s rank r holds rank (r - s) mod W's two chunks and computes its
own query chunks against them with the library's forward -- a key chunk before
the query chunk needs no mask, the same chunk the causal one, a later chunk
nothing -- and folds each result into an fp32 accumulator by the LSE merge of
unite.ai, "Flash Attention: Revolutionizing Transformer Efficiency", section
"The Mathematics of Flash Attention" (fa_merge_partials).  The chunks of the
next step are sent to rank r + 1 and received from rank r - 1 while the current
ones are computed; W steps in all, W - 1 of them with an exchange, taken in the
same order on every rank.  The pages do not describe this exchange; it is the
plainest sharding of the sequence that keeps the result exact.

The per-chunk forward and the merge are parameters so that the exchange and the
schedule can be tested on CPU ranks (gloo) with reference implementations; by
default they are the library's fa.attention and fa.merge_partials.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

FULL, CAUSAL, SKIP = "full", "causal", "skip"


def zigzag_chunks(rank: int, world: int) -> tuple[int, int]:
    """The two sequence chunks (of 2 * world) that `rank` holds."""
    if world <= 0 or not 0 <= rank < world:
        raise ValueError("bad world/rank")
    return rank, 2 * world - 1 - rank


def chunk_pair_mode(q_chunk: int, k_chunk: int, causal: bool) -> str:
    """How query chunk q_chunk meets key chunk k_chunk (equal chunk lengths)."""
    if not causal:
        return FULL
    if k_chunk < q_chunk:
        return FULL
    return CAUSAL if k_chunk == q_chunk else SKIP


def zigzag_shard(x: torch.Tensor, rank: int, world: int, dim: int = -2) -> torch.Tensor:
    """Rank's two chunks of x along the sequence dimension `dim`, stacked in a new
    leading dimension: [2, ...] (each chunk contiguous).  x's length along `dim`
    must be a multiple of 2 * world."""
    n = x.shape[dim]
    if n % (2 * world):
        raise ValueError(f"sequence length {n} is not a multiple of 2 * world = {2 * world}")
    c = n // (2 * world)
    a, b = zigzag_chunks(rank, world)
    return torch.stack([x.narrow(dim, a * c, c), x.narrow(dim, b * c, c)]).contiguous()


def zigzag_unshard(parts, dim: int = -2) -> torch.Tensor:
    """Inverse of zigzag_shard: parts[r] is rank r's [2, ...] tensor."""
    world = len(parts)
    chunks = [None] * (2 * world)
    for r, p in enumerate(parts):
        a, b = zigzag_chunks(r, world)
        chunks[a], chunks[b] = p[0], p[1]
    return torch.cat(chunks, dim=dim)


@dataclass(frozen=True)
class RingWork:
    step: int        # ring step (the K/V chunks come from rank (rank - step) mod world)
    q_index: int     # 0 or 1: which of the rank's query chunks
    k_index: int     # 0 or 1: which of the visiting ranks' K/V chunks
    causal: bool     # the diagonal pair (causal mask) or a full pair
    last: bool       # the last work item of this query chunk


def ring_schedule(rank: int, world: int, causal: bool) -> list[RingWork]:
    """Work items of `rank` in execution order (no item for skipped pairs)."""
    items = []
    for s in range(world):
        src = (rank - s) % world
        for qi, qc in enumerate(zigzag_chunks(rank, world)):
            for ki, kc in enumerate(zigzag_chunks(src, world)):
                mode = chunk_pair_mode(qc, kc, causal)
                if mode != SKIP:
                    items.append([s, qi, ki, mode == CAUSAL])
    out = []
    for i, (s, qi, ki, c) in enumerate(items):
        last = all(it[1] != qi for it in items[i + 1:])
        out.append(RingWork(s, qi, ki, c, last))
    return out


def _default_attend(q, k, v, causal, scale):
    from . import fa
    return fa.attention(q, k, v, scale, causal, return_lse=True)


def _default_merge(o_acc, lse_acc, o, lse, first, o_out):
    from . import fa
    fa.merge_partials(o_acc, lse_acc, o, lse, first=first, o_out=o_out)


def ring_attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool,
                   scale: float | None = None, group=None, attend=None, merge=None,
                   fetch=None, rank: int | None = None, world: int | None = None):
    """Exact attention of a zigzag-sharded sequence.

    q [2, B, Hq, C, D], k, v [2, B, Hkv, C, D]: this rank's two chunks
    (zigzag_shard of the full tensors).  Returns (O [2, B, Hq, C, D] in q's
    dtype, LSE [2, B, Hq, C] fp32), this rank's rows of the full result.
    `group` is the torch.distributed process group (None: the default one,
    or a single process when torch.distributed is not initialised).

    With `fetch` (and `rank`, `world`) nothing is exchanged: fetch(s) returns
    the K/V chunks of step s, i.e. those of rank (rank - s) mod world; this runs
    one rank's share of the computation on its own, e.g. every rank in turn on
    one device.
    """
    import torch.distributed as dist
    if q.dim() != 5 or k.dim() != 5 or q.shape[0] != 2 or k.shape != v.shape or \
            k.shape[0] != 2 or k.shape[1] != q.shape[1] or k.shape[3:] != q.shape[3:]:
        raise ValueError("q [2, B, Hq, C, D] and k, v [2, B, Hkv, C, D] expected "
                         "(zigzag_shard of [B, H, N, D] tensors)")
    attend = attend or _default_attend
    merge = merge or _default_merge
    D = q.shape[-1]
    if scale is None:
        scale = D ** -0.5
    if fetch is not None:
        if rank is None or world is None:
            raise ValueError("fetch needs rank and world")
    elif dist.is_available() and dist.is_initialized():
        world = dist.get_world_size(group)
        rank = dist.get_rank(group)
    else:
        world, rank = 1, 0
    o_acc = torch.empty(q.shape, dtype=torch.float32, device=q.device)
    lse_acc = torch.empty(q.shape[:-1], dtype=torch.float32, device=q.device)
    out = torch.empty_like(q)
    started = [False, False]
    schedule = ring_schedule(rank, world, causal)

    def run_step(s, k_cur, v_cur):
        for w in schedule:
            if w.step != s:
                continue
            o, lse = attend(q[w.q_index], k_cur[w.k_index], v_cur[w.k_index], w.causal, scale)
            merge(o_acc[w.q_index], lse_acc[w.q_index], o, lse, not started[w.q_index],
                  out[w.q_index] if w.last else None)
            started[w.q_index] = True

    if fetch is not None:
        for s in range(world):
            k_s, v_s = fetch(s)
            run_step(s, k_s, v_s)
        return out, lse_acc

    def peer(r):   # global rank of group rank r
        return dist.get_global_rank(group, r) if group is not None else r
    nxt = peer((rank + 1) % world)
    prv = peer((rank - 1) % world)
    k_cur, v_cur = k.contiguous(), v.contiguous()
    for s in range(world):
        reqs = []
        if s + 1 < world:
            k_next, v_next = torch.empty_like(k_cur), torch.empty_like(v_cur)
            ops = [dist.P2POp(dist.isend, k_cur, nxt, group),
                   dist.P2POp(dist.isend, v_cur, nxt, group),
                   dist.P2POp(dist.irecv, k_next, prv, group),
                   dist.P2POp(dist.irecv, v_next, prv, group)]
            reqs = dist.batch_isend_irecv(ops)
        run_step(s, k_cur, v_cur)
        for r in reqs:
            r.wait()
        if s + 1 < world:
            k_cur, v_cur = k_next, v_next
    return out, lse_acc
