"""Host-side checks of the seeded input generator (no GPU)."""
import torch

from exact_tiled_attention_40_b200.inputs import (DecodeCase, PrefillCase, make_decode,
                                                   make_prefill, sample_rows)


def test_prefill_is_deterministic_and_shaped():
    c = PrefillCase("t", 2, 4, 2, 33, 47, 64, "bf16", seed=5, causal=True, amp=0.5)
    q1, k1, v1, _ = make_prefill(c)
    q2, k2, v2, _ = make_prefill(c)
    assert q1.shape == (2, 4, 33, 64) and k1.shape == (2, 2, 47, 64) and v1.dtype == torch.bfloat16
    assert torch.equal(q1, q2) and torch.equal(k1, k2) and torch.equal(v1, v2)
    assert not torch.equal(k1, v1)
    assert 0.35 < float(q1.float().std()) < 0.65          # amplitude 0.5


def test_sampled_rows_cover_every_head_and_the_ends():
    c = PrefillCase("t", 1, 4, 1, 100, 100, 64, seed=3)
    _, _, _, gen = make_prefill(c)
    rows = sample_rows(c, gen, 5)
    assert len(rows) == 20
    assert rows[0] == (0, 0, 0) and rows[1] == (0, 0, 99)
    assert {h for _, h, _ in rows} == {0, 1, 2, 3}
    assert all(0 <= i < 100 for _, _, i in rows)


def test_decode_block_table_is_valid_and_pages_distinct():
    c = DecodeCase("d", 6, 8, 2, 64, 16, 20, 100, 64, seed=4)
    q, kc, vc, table, lens = make_decode(c)
    assert q.shape == (6, 8, 64) and kc.shape == (64, 16, 2, 64) and table.shape == (6, 7)
    used = []
    for b in range(6):
        n = -(-int(lens[b]) // 16)
        assert 20 <= int(lens[b]) <= 100
        used.extend(table[b, :n].tolist())
        assert torch.all(table[b, n:] == 0)
    assert len(set(used)) == len(used) and all(0 <= p < 64 for p in used)
    q2, kc2, _, table2, lens2 = make_decode(c)
    assert torch.equal(kc, kc2) and torch.equal(table, table2) and torch.equal(lens, lens2)
