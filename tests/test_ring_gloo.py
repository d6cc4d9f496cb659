"""Sequence-sharded (ring) attention, host logic on CPU ranks.

The zigzag sharding, the ring schedule and the K/V exchange of
exact_tiled_attention_40_b200.ring run on gloo ranks (world sizes 2 and 3) with
the fp64 oracle standing in for the per-chunk forward and the oracle's LSE merge
for fa_merge_partials; the reassembled result must equal the oracle on the
whole sequence.  (The library's own per-chunk forward and merge are covered on
the GPU by tests/test_ring_gpu.py.)
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from exact_tiled_attention_40_b200 import ring


def test_zigzag_shard_round_trip_and_chunk_assignment():
    x = torch.arange(2 * 3 * 24 * 4, dtype=torch.float32).reshape(2, 3, 24, 4)
    for world in (1, 2, 3, 4):
        parts = [ring.zigzag_shard(x, r, world) for r in range(world)]
        assert all(p.shape == (2, 2, 3, 24 // (2 * world), 4) for p in parts)
        assert torch.equal(ring.zigzag_unshard(parts), x)
    assert ring.zigzag_chunks(0, 4) == (0, 7) and ring.zigzag_chunks(3, 4) == (3, 4)
    with pytest.raises(ValueError):
        ring.zigzag_shard(x, 0, 5)             # 24 is not a multiple of 10


@pytest.mark.parametrize("world", [1, 2, 3, 4, 7])
@pytest.mark.parametrize("causal", [False, True])
def test_schedule_meets_every_visible_chunk_pair_once(world, causal):
    seen = {}
    work = []
    for r in range(world):
        items = ring.ring_schedule(r, world, causal)
        steps = [w.step for w in items]
        assert steps == sorted(steps)
        cost = 0.0
        for w in items:
            src = (r - w.step) % world
            qc = ring.zigzag_chunks(r, world)[w.q_index]
            kc = ring.zigzag_chunks(src, world)[w.k_index]
            assert (qc, kc) not in seen
            seen[(qc, kc)] = w.causal
            assert w.causal == (causal and qc == kc)
            cost += 0.5 if w.causal else 1.0
        work.append(cost)
        # exactly one last item per query chunk, and nothing of that chunk after it
        for qi in (0, 1):
            mine = [i for i, w in enumerate(items) if w.q_index == qi]
            assert [items[i].last for i in mine] == [False] * (len(mine) - 1) + [True]
    n = 2 * world
    want = {(a, b) for a in range(n) for b in range(n) if not causal or b <= a}
    assert set(seen) == want
    assert max(work) == min(work)              # zigzag: every rank has the same work


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _oracle_attend(q, k, v, causal, scale):
    O, L = oracle.attention(q.double().numpy(), k.double().numpy(), v.double().numpy(), scale,
                            causal)
    return torch.from_numpy(O), torch.from_numpy(L)


def _oracle_merge(o_acc, lse_acc, o, lse, first, o_out):
    if first:
        o_acc.copy_(o)
        lse_acc.copy_(lse)
    else:
        O, L = oracle.merge_partials([o_acc.double().numpy(), o.double().numpy()],
                                     [lse_acc.double().numpy(), lse.double().numpy()])
        o_acc.copy_(torch.from_numpy(O))
        lse_acc.copy_(torch.from_numpy(L))
    if o_out is not None:
        o_out.copy_(o_acc)


def _ring_worker(rank, world, port, q, k, v, causal, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        qs = ring.zigzag_shard(q, rank, world)
        ks = ring.zigzag_shard(k, rank, world)
        vs = ring.zigzag_shard(v, rank, world)
        o, lse = ring.ring_attention(qs, ks, vs, causal, 0.3, attend=_oracle_attend,
                                     merge=_oracle_merge)
        parts = [None] * world
        dist.all_gather_object(parts, (o, lse))
        if rank == 0:
            out.put(parts)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,causal", [(2, True), (2, False), (3, True)])
def test_ring_ranks_reassemble_the_oracle_result(world, causal):
    g = torch.Generator().manual_seed(70 + world)
    N = 12 * world
    q = torch.randn((2, 4, N, 8), generator=g, dtype=torch.float32)
    k = torch.randn((2, 2, N, 8), generator=g, dtype=torch.float32)
    v = torch.randn((2, 2, N, 8), generator=g, dtype=torch.float32)
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_ring_worker, args=(r, world, port, q, k, v, causal, out))
             for r in range(world)]
    for p in procs:
        p.start()
    parts = out.get(timeout=180)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    O = ring.zigzag_unshard([p[0] for p in parts]).double().numpy()
    L = ring.zigzag_unshard([p[1] for p in parts], dim=-1).double().numpy()
    O_ref, L_ref = oracle.attention(q.double().numpy(), k.double().numpy(), v.double().numpy(),
                                    0.3, causal)
    # the accumulators are fp32
    np.testing.assert_allclose(O, O_ref, atol=2e-6)
    np.testing.assert_allclose(L, L_ref, atol=2e-6)


def test_single_process_runs_without_a_process_group():
    g = torch.Generator().manual_seed(75)
    q = torch.randn((1, 2, 16, 8), generator=g)
    k = torch.randn((1, 1, 16, 8), generator=g)
    v = torch.randn((1, 1, 16, 8), generator=g)
    o, lse = ring.ring_attention(ring.zigzag_shard(q, 0, 1), ring.zigzag_shard(k, 0, 1),
                                 ring.zigzag_shard(v, 0, 1), True, 0.5,
                                 attend=_oracle_attend, merge=_oracle_merge)
    O_ref, L_ref = oracle.attention(q.double().numpy(), k.double().numpy(), v.double().numpy(),
                                    0.5, True)
    np.testing.assert_allclose(ring.zigzag_unshard([o]).double().numpy(), O_ref, atol=2e-6)
    np.testing.assert_allclose(ring.zigzag_unshard([lse], dim=-1).double().numpy(), L_ref,
                               atol=2e-6)


def test_one_rank_at_a_time_with_fetched_chunks_equals_the_oracle():
    """The exchange-free form (each rank's share run on its own, K/V chunks handed
    in per step) reassembles the full result too."""
    world = 4
    g = torch.Generator().manual_seed(76)
    q = torch.randn((1, 2, 32, 8), generator=g)
    k = torch.randn((1, 1, 32, 8), generator=g)
    v = torch.randn((1, 1, 32, 8), generator=g)
    ks = [ring.zigzag_shard(k, r, world) for r in range(world)]
    vs = [ring.zigzag_shard(v, r, world) for r in range(world)]
    outs, lses = [], []
    for r in range(world):
        o, lse = ring.ring_attention(
            ring.zigzag_shard(q, r, world), ks[r], vs[r], True, 0.4, attend=_oracle_attend,
            merge=_oracle_merge, rank=r, world=world,
            fetch=lambda s, r=r: (ks[(r - s) % world], vs[(r - s) % world]))
        outs.append(o)
        lses.append(lse)
    O_ref, L_ref = oracle.attention(q.double().numpy(), k.double().numpy(), v.double().numpy(),
                                    0.4, True)
    np.testing.assert_allclose(ring.zigzag_unshard(outs).double().numpy(), O_ref, atol=2e-6)
    np.testing.assert_allclose(ring.zigzag_unshard(lses, dim=-1).double().numpy(), L_ref,
                               atol=2e-6)


def test_ring_rejects_tensors_that_are_not_zigzag_shards():
    q = torch.zeros((2, 1, 2, 8, 4))
    k = torch.zeros((2, 1, 1, 8, 4))
    with pytest.raises(ValueError):
        ring.ring_attention(q[0], k, k, True, attend=_oracle_attend, merge=_oracle_merge)
    with pytest.raises(ValueError):
        ring.ring_attention(q, k[:, :, :, :4], k[:, :, :, :4], True, attend=_oracle_attend,
                            merge=_oracle_merge)
