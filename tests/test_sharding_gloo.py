"""Multi-rank host logic on CPU: two gloo ranks each run the fp64 oracle on their
own shard (batch entries, or whole GQA head groups) and the union of the shards
equals the unsharded result; the max-over-ranks timing reduction is checked too.
The path needs no data collective; gloo is used here only to bring the shards
back to rank 0 for the comparison."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from exact_tiled_attention_40_b200.sharding import batch_shard, even_range, head_shard


def test_even_range_partitions_exactly():
    for n in range(0, 23):
        for world in range(1, 6):
            covered = []
            for r in range(world):
                a, b = even_range(n, world, r)
                covered.extend(range(a, b))
            assert covered == list(range(n))


def test_head_shard_keeps_gqa_groups_whole():
    for r in range(3):
        (h0, h1), (g0, g1) = head_shard(32, 8, 3, r)
        assert h0 == g0 * 4 and h1 == g1 * 4


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q, k, v, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        B, Hq = q.shape[0], q.shape[1]
        Hkv = k.shape[1]
        b0, b1 = batch_shard(B, world, rank)
        Ob, Lb = oracle.attention(q[b0:b1], k[b0:b1], v[b0:b1], 0.3, True)
        (h0, h1), (g0, g1) = head_shard(Hq, Hkv, world, rank)
        Oh, Lh = oracle.attention(q[:, h0:h1], k[:, g0:g1], v[:, g0:g1], 0.3, True)
        parts_b = [None] * world
        parts_h = [None] * world
        dist.all_gather_object(parts_b, (b0, b1, Ob, Lb))
        dist.all_gather_object(parts_h, (h0, h1, Oh, Lh))
        t = torch.tensor([1.5 + rank], dtype=torch.float64)     # per-rank times
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        if rank == 0:
            out.put((parts_b, parts_h, float(t)))
    finally:
        dist.destroy_process_group()


def test_two_rank_shards_reassemble_the_full_result():
    rng = np.random.default_rng(60)
    q = rng.standard_normal((3, 8, 20, 16))
    k = rng.standard_normal((3, 2, 20, 16))
    v = rng.standard_normal((3, 2, 20, 16))
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q, k, v, out)) for r in range(2)]
    for p in procs:
        p.start()
    parts_b, parts_h, tmax = out.get(timeout=120)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    O, L = oracle.attention(q, k, v, 0.3, True)
    Ob = np.concatenate([p[2] for p in sorted(parts_b, key=lambda x: x[0])], axis=0)
    Oh = np.concatenate([p[2] for p in sorted(parts_h, key=lambda x: x[0])], axis=1)
    Lh = np.concatenate([p[3] for p in sorted(parts_h, key=lambda x: x[0])], axis=1)
    np.testing.assert_allclose(Ob, O, atol=1e-12)
    np.testing.assert_allclose(Oh, O, atol=1e-12)
    np.testing.assert_allclose(Lh, L, atol=1e-12)
    assert tmax == 2.5


def test_ragged_shard_partitions_whole_sequences_by_work():
    from exact_tiled_attention_40_b200.sharding import ragged_shard
    nq = [5, 300, 0, 17, 900, 40, 40, 1]
    cq = np.concatenate([[0], np.cumsum(nq)])
    ck = np.concatenate([[0], np.cumsum([x + 3 for x in nq])])
    for world in (1, 2, 3, 5):
        seqs, rows = [], []
        for r in range(world):
            b0, b1, (q0, q1), (k0, k1), cql, ckl = ragged_shard(cq, ck, world, r)
            seqs.extend(range(b0, b1))
            rows.append((q0, q1))
            assert cql[0] == 0 and cql[-1] == q1 - q0 and len(cql) == b1 - b0 + 1
            assert ckl[0] == 0 and ckl[-1] == k1 - k0
        assert seqs == list(range(len(nq)))
        assert all(rows[i][1] == rows[i + 1][0] for i in range(world - 1))


def _ragged_worker(rank, world, port, q, k, v, cq, ck, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from exact_tiled_attention_40_b200.sharding import ragged_shard
        b0, b1, (q0, q1), (k0, k1), cql, ckl = ragged_shard(cq, ck, world, rank)
        O, L = oracle.varlen_attention(q[q0:q1], k[k0:k1], v[k0:k1], np.array(cql),
                                       np.array(ckl), 0.3, True)
        parts = [None] * world
        dist.all_gather_object(parts, (q0, q1, O, L))
        if rank == 0:
            out.put(parts)
    finally:
        dist.destroy_process_group()


def test_two_rank_ragged_shards_reassemble_the_full_result():
    rng = np.random.default_rng(61)
    nq = [7, 30, 1, 12, 25]
    nk = [9, 30, 4, 12, 40]
    cq = np.concatenate([[0], np.cumsum(nq)])
    ck = np.concatenate([[0], np.cumsum(nk)])
    q = rng.standard_normal((cq[-1], 4, 8))
    k = rng.standard_normal((ck[-1], 2, 8))
    v = rng.standard_normal((ck[-1], 2, 8))
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_ragged_worker, args=(r, 2, port, q, k, v, cq, ck, out))
             for r in range(2)]
    for p in procs:
        p.start()
    parts = out.get(timeout=120)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    O, L = oracle.varlen_attention(q, k, v, cq, ck, 0.3, True)
    parts.sort(key=lambda x: x[0])
    np.testing.assert_allclose(np.concatenate([p[2] for p in parts], axis=0), O, atol=1e-12)
    np.testing.assert_allclose(np.concatenate([p[3] for p in parts], axis=1), L, atol=1e-12)
