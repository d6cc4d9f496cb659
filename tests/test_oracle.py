"""Pins of the fp64 oracle against facts fixed by the pages and by mathematics.

None of these retypes the oracle's formula: each check is a closed form, a
hand-derived value, an invariant, an independent library routine, or the
pages' own blockwise algorithm agreeing with the definition.  The last group
plants known mistakes in the oracle (on the CPU) and shows that the pins catch
them.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import attention_fp64 as oracle_mod

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_derived_cases.json")
TIGHT = 1e-12


def rand(shape, seed, amp=1.0):
    return amp * np.random.default_rng(seed).standard_normal(shape)


def sdpa_f64(q, k, v, scale, causal):
    """torch's float64 CPU scaled_dot_product_attention (an independent library
    routine) with K/V heads expanded for GQA and the bottom-right causal mask
    passed explicitly; LSE from torch.logsumexp."""
    q, k, v = (torch.from_numpy(np.ascontiguousarray(x)).double() for x in (q, k, v))
    rep = q.shape[1] // k.shape[1]
    k = k.repeat_interleave(rep, dim=1)
    v = v.repeat_interleave(rep, dim=1)
    Nq, Nk = q.shape[2], k.shape[2]
    mask = None
    if causal:
        mask = torch.ones(Nq, Nk, dtype=torch.bool).tril(diagonal=Nk - Nq)
    o = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=mask, scale=scale)
    s = scale * (q @ k.transpose(-1, -2))
    if mask is not None:
        s = s.masked_fill(~mask, float("-inf"))
    return o.numpy(), torch.logsumexp(s, dim=-1).numpy()


# ---------------------------------------------------------------- golden cases
def load_golden():
    with open(GOLDEN) as f:
        return json.load(f)


@pytest.mark.parametrize("case", load_golden()["cases"], ids=lambda c: c["name"])
def test_hand_derived_prefill_cases(case):
    q, k, v = (np.array(case[n], dtype=np.float64) for n in ("q", "k", "v"))
    O, LSE = oracle.attention(q, k, v, case["scale"], case["causal"])
    np.testing.assert_allclose(O, np.array(case["O"]), rtol=0, atol=1e-13)
    np.testing.assert_allclose(LSE, np.array(case["LSE"]), rtol=0, atol=1e-13)


@pytest.mark.parametrize("case", load_golden()["decode_cases"], ids=lambda c: c["name"])
def test_hand_derived_decode_cases(case):
    O, LSE = oracle.decode_paged(np.array(case["q"]), np.array(case["kcache"]),
                                 np.array(case["vcache"]), np.array(case["block_table"]),
                                 np.array(case["seq_lens"]), case["scale"], case["page_size"])
    np.testing.assert_allclose(O, np.array(case["O"]), rtol=0, atol=1e-13)
    np.testing.assert_allclose(LSE, np.array(case["LSE"]), rtol=0, atol=1e-13)


# ---------------------------------------------------------------- closed forms
@pytest.mark.parametrize("causal", [False, True])
def test_zero_query_gives_mean_of_visible_values(causal):
    B, Hq, Hkv, Nq, Nk, D = 2, 4, 2, 5, 9, 6
    q = np.zeros((B, Hq, Nq, D))
    k, v = rand((B, Hkv, Nk, D), 1), rand((B, Hkv, Nk, D), 2)
    O, LSE = oracle.attention(q, k, v, 0.3, causal)
    for b in range(B):
        for h in range(Hq):
            g = h // (Hq // Hkv)
            for i in range(Nq):
                n = i + (Nk - Nq) + 1 if causal else Nk
                np.testing.assert_allclose(O[b, h, i], v[b, g, :n].mean(axis=0), atol=TIGHT)
                assert abs(LSE[b, h, i] - math.log(n)) < TIGHT


def test_single_dominant_key_selects_its_value():
    Nk, D = 16, 8
    q = rand((1, 1, 1, D), 3)
    k = rand((1, 1, Nk, D), 4) * 0.01
    j = 11
    k[0, 0, j] = 60.0 * q[0, 0, 0] / np.dot(q[0, 0, 0], q[0, 0, 0])   # score 60 vs ~0
    v = rand((1, 1, Nk, D), 5)
    O, LSE = oracle.attention(q, k, v, 1.0, False)
    bound = Nk * math.exp(-59.0) * np.abs(v).max() + 1e-12     # weight off key j <= Nk e^-59
    np.testing.assert_allclose(O[0, 0, 0], v[0, 0, j], atol=bound)
    assert abs(LSE[0, 0, 0] - 60.0) < 1e-12 + Nk * math.exp(-59)


def test_causal_first_row_is_first_value():
    q, k, v = rand((1, 3, 7, 5), 6), rand((1, 3, 7, 5), 7), rand((1, 3, 7, 5), 8)
    O, LSE = oracle.attention(q, k, v, 0.7, True)
    np.testing.assert_allclose(O[0, :, 0], v[0, :, 0], atol=TIGHT)
    np.testing.assert_allclose(LSE[0, :, 0], 0.7 * np.einsum("hd,hd->h", q[0, :, 0], k[0, :, 0]),
                               atol=TIGHT)


def test_single_key_and_constant_values():
    q, k = rand((2, 2, 4, 3), 9), rand((2, 2, 1, 3), 10)
    v = rand((2, 2, 1, 3), 11)
    O, _ = oracle.attention(q, k, v, 1.3, False)
    np.testing.assert_allclose(O, np.broadcast_to(v, O.shape), atol=TIGHT)
    c = np.array([0.5, -2.0, 3.25])
    k2 = rand((2, 2, 6, 3), 12)
    v2 = np.broadcast_to(c, (2, 2, 6, 3)).copy()
    O2, _ = oracle.attention(rand((2, 2, 4, 3), 13), k2, v2, 0.9, True)
    np.testing.assert_allclose(O2, np.broadcast_to(c, O2.shape), atol=TIGHT)


def test_fully_masked_row_is_zero_with_minus_inf_lse():
    s = np.array([[1.0, 2.0], [3.0, 4.0]])
    p, m, l = oracle.softmax_rows(s, np.array([[True, True], [False, False]]))
    assert np.all(p[1] == 0) and m[1] == -np.inf and l[1] == 0


# ---------------------------------------------------------------- invariants
def test_softmax_rows_sum_to_one_and_shift_invariance():
    s = rand((6, 33), 14, amp=20.0)
    p, m, l = oracle.softmax_rows(s)
    np.testing.assert_allclose(p.sum(axis=-1), 1.0, atol=TIGHT)
    delta = rand((6, 1), 15, amp=50.0)
    p2, m2, l2 = oracle.softmax_rows(s + delta)
    np.testing.assert_allclose(p2, p, atol=TIGHT)
    np.testing.assert_allclose(m2, m + delta[:, 0], atol=1e-10)
    np.testing.assert_allclose(l2, l, rtol=1e-12)


def test_joint_key_value_permutation_invariance():
    q, k, v = rand((1, 2, 5, 4), 16), rand((1, 2, 12, 4), 17), rand((1, 2, 12, 4), 18)
    perm = np.random.default_rng(19).permutation(12)
    O1, L1 = oracle.attention(q, k, v, 0.5, False)
    O2, L2 = oracle.attention(q, k[:, :, perm], v[:, :, perm], 0.5, False)
    np.testing.assert_allclose(O1, O2, atol=TIGHT)
    np.testing.assert_allclose(L1, L2, atol=TIGHT)


# ---------------------------------------------------------------- library routine
@pytest.mark.parametrize("Hq,Hkv,Nq,Nk,causal", [(2, 2, 7, 7, False), (4, 1, 9, 9, True),
                                                  (8, 2, 5, 13, True), (4, 2, 16, 3, False)])
def test_matches_float64_library_attention(Hq, Hkv, Nq, Nk, causal):
    q, k, v = rand((2, Hq, Nq, 8), 20), rand((2, Hkv, Nk, 8), 21), rand((2, Hkv, Nk, 8), 22)
    O, LSE = oracle.attention(q, k, v, 0.35, causal)
    O_ref, LSE_ref = sdpa_f64(q, k, v, 0.35, causal)
    np.testing.assert_allclose(O, O_ref, atol=TIGHT)
    np.testing.assert_allclose(LSE, LSE_ref, atol=TIGHT)


def test_rows_variant_matches_library():
    q, k, v = rand((1, 4, 20, 8), 23), rand((1, 2, 20, 8), 24), rand((1, 2, 20, 8), 25)
    rows = [(0, 0, 0), (0, 1, 19), (0, 3, 7), (0, 2, 13)]
    O, LSE = oracle.attention_rows(q, k, v, 0.4, True, rows)
    O_ref, LSE_ref = sdpa_f64(q, k, v, 0.4, True)
    for r, (b, h, i) in enumerate(rows):
        np.testing.assert_allclose(O[r], O_ref[b, h, i], atol=TIGHT)
        assert abs(LSE[r] - LSE_ref[b, h, i]) < TIGHT


# ---------------------------------------------------------------- blockwise = full
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("Nq,Nk", [(12, 12), (7, 12)])
def test_blockwise_equals_definition_for_every_block_size(causal, Nq, Nk):
    q, k, v = rand((1, 2, Nq, 4), 26), rand((1, 1, Nk, 4), 27), rand((1, 1, Nk, 4), 28)
    O_ref, L_ref = oracle.attention(q, k, v, 0.8, causal)
    for Br in range(1, Nq + 1):
        for Bc in range(1, Nk + 1):
            O, L = oracle.blockwise_attention(q, k, v, 0.8, causal, Br, Bc)
            np.testing.assert_allclose(O, O_ref, atol=TIGHT)
            np.testing.assert_allclose(L, L_ref, atol=TIGHT)


# ---------------------------------------------------------------- merge / split-KV
def test_merge_of_key_chunks_equals_unsplit():
    q, k, v = rand((1, 4, 3, 8), 29), rand((1, 2, 40, 8), 30), rand((1, 2, 40, 8), 31)
    O_ref, L_ref = oracle.attention(q, k, v, 0.5, False)
    cuts = [0, 1, 9, 10, 27, 40]
    parts = [oracle.attention(q, k[:, :, a:b], v[:, :, a:b], 0.5, False)
             for a, b in zip(cuts[:-1], cuts[1:])]
    O, L = oracle.merge_partials([p[0] for p in parts], [p[1] for p in parts])
    np.testing.assert_allclose(O, O_ref, atol=TIGHT)
    np.testing.assert_allclose(L, L_ref, atol=TIGHT)


def test_merge_closed_forms():
    o1, o2 = np.array([1.0, 2.0]), np.array([3.0, -2.0])
    O, L = oracle.merge_partials([o1, o2], [0.7, 0.7])          # equal mass: average
    np.testing.assert_allclose(O, [2.0, 0.0], atol=TIGHT)
    assert abs(L - (0.7 + math.log(2))) < TIGHT
    O, L = oracle.merge_partials([o1, o2], [math.log(3.0), -np.inf])   # empty part: no weight
    np.testing.assert_allclose(O, o1, atol=TIGHT)
    assert abs(L - math.log(3.0)) < TIGHT


# ---------------------------------------------------------------- paged decode
def test_decode_matches_definition_on_gathered_cache():
    rng = np.random.default_rng(32)
    B, Hq, Hkv, D, ps, pool = 3, 8, 2, 8, 4, 20
    lens = np.array([1, 9, 13])
    perm = rng.permutation(pool)
    table = np.zeros((B, 4), dtype=np.int32)
    cur = 0
    for b in range(B):
        n = -(-lens[b] // ps)
        table[b, :n] = perm[cur:cur + n]
        cur += n
    kc, vc = rand((pool, ps, Hkv, D), 33), rand((pool, ps, Hkv, D), 34)
    q = rand((B, Hq, D), 35)
    O, L = oracle.decode_paged(q, kc, vc, table, lens, 0.3, ps)
    for b in range(B):
        pages = table[b, :-(-lens[b] // ps)]
        kk = np.concatenate([kc[p] for p in pages])[:lens[b]]      # [n, Hkv, D]
        vv = np.concatenate([vc[p] for p in pages])[:lens[b]]
        o_ref, l_ref = sdpa_f64(q[b][None, :, None, :], kk.transpose(1, 0, 2)[None],
                                vv.transpose(1, 0, 2)[None], 0.3, False)
        np.testing.assert_allclose(O[b], o_ref[0, :, 0], atol=TIGHT)
        np.testing.assert_allclose(L[b], l_ref[0, :, 0], atol=TIGHT)


# ---------------------------------------------------------------- planted mistakes
def test_pins_catch_the_printed_blockwise_update():
    """The page's update omits L_old; with more than one key block it is wrong."""
    q, k, v = rand((1, 1, 6, 4), 36), rand((1, 1, 6, 4), 37), rand((1, 1, 6, 4), 38)
    O_ref, _ = oracle.attention(q, k, v, 1.0, False)
    O_bug, _ = oracle.blockwise_attention(q, k, v, 1.0, False, 3, 2, keep_page_bug=True)
    assert np.max(np.abs(O_bug - O_ref)) > 1e-3
    O_one, _ = oracle.blockwise_attention(q, k, v, 1.0, False, 3, 6, keep_page_bug=True)
    np.testing.assert_allclose(O_one, O_ref, atol=TIGHT)   # one block: no merge, no bug


def test_pins_catch_wrong_gqa_mapping(monkeypatch):
    q, k, v = rand((1, 4, 5, 4), 39), rand((1, 2, 5, 4), 40), rand((1, 2, 5, 4), 41)
    monkeypatch.setattr(oracle_mod, "kv_head_of", lambda h, Hq, Hkv: h % Hkv)
    O_bad, _ = oracle_mod.attention(q, k, v, 0.5, False)
    O_ref, _ = sdpa_f64(q, k, v, 0.5, False)
    assert np.max(np.abs(O_bad - O_ref)) > 1e-3


def test_pins_catch_top_left_causal_alignment(monkeypatch):
    q, k, v = rand((1, 1, 4, 4), 42), rand((1, 1, 9, 4), 43), rand((1, 1, 9, 4), 44)
    monkeypatch.setattr(oracle_mod, "causal_allowed",
                        lambda Nq, Nk: np.arange(Nk)[None, :] <= np.arange(Nq)[:, None])
    O_bad, _ = oracle_mod.attention(q, k, v, 0.5, True)
    O_ref, _ = sdpa_f64(q, k, v, 0.5, True)
    assert np.max(np.abs(O_bad - O_ref)) > 1e-3


def test_pins_catch_missing_normalisation(monkeypatch):
    """Dropping the division by the row sum changes the golden case's output."""
    case = load_golden()["cases"][0]
    q, k, v = (np.array(case[n], dtype=np.float64) for n in ("q", "k", "v"))
    real = oracle_mod.softmax_rows

    def unnormalised(s, allowed=None):
        p, m, l = real(s, allowed)
        return p * l[..., None], m, np.ones_like(l)
    monkeypatch.setattr(oracle_mod, "softmax_rows", unnormalised)
    O_bad, _ = oracle_mod.attention(q, k, v, case["scale"], case["causal"])
    assert np.max(np.abs(O_bad - np.array(case["O"]))) > 1e-3


# ---------------------------------------------------------------- ragged batches
def _packed_case(Nq, Nk, Hq, Hkv, D, seed):
    cu_q = np.concatenate([[0], np.cumsum(Nq)]).astype(np.int64)
    cu_k = np.concatenate([[0], np.cumsum(Nk)]).astype(np.int64)
    q = rand((int(cu_q[-1]), Hq, D), seed)
    k = rand((int(cu_k[-1]), Hkv, D), seed + 1)
    v = rand((int(cu_k[-1]), Hkv, D), seed + 2)
    return q, k, v, cu_q, cu_k


def _padded_library(q, k, v, cu_q, cu_k, scale, causal):
    """The padded-batch formulation of a ragged batch, through torch's float64
    scaled_dot_product_attention with an explicit per-sequence boolean mask:
    key j of sequence b is visible to its query i iff j < Nk_b (and, causal,
    j <= i + Nk_b - Nq_b).  Returns O and LSE in the packed layouts; rows with no
    visible key are NaN."""
    B = len(cu_q) - 1
    Nq = np.diff(cu_q)
    Nk = np.diff(cu_k)
    Mq, Mk = max(1, int(Nq.max())), max(1, int(Nk.max()))
    Hq, D = q.shape[1], q.shape[2]
    Hkv = k.shape[1]
    qp = np.zeros((B, Hq, Mq, D))
    kp = np.zeros((B, Hkv, Mk, D))
    vp = np.zeros((B, Hkv, Mk, D))
    mask = np.zeros((B, 1, Mq, Mk), dtype=bool)
    for b in range(B):
        qp[b, :, :Nq[b]] = np.transpose(q[cu_q[b]:cu_q[b + 1]], (1, 0, 2))
        kp[b, :, :Nk[b]] = np.transpose(k[cu_k[b]:cu_k[b + 1]], (1, 0, 2))
        vp[b, :, :Nk[b]] = np.transpose(v[cu_k[b]:cu_k[b + 1]], (1, 0, 2))
        i = np.arange(Mq)[:, None]
        j = np.arange(Mk)[None, :]
        ok = j < Nk[b]
        if causal:
            ok = ok & (j <= i + Nk[b] - Nq[b])
        mask[b, 0] = ok
    tq, tk, tv = (torch.from_numpy(x) for x in (qp, kp, vp))
    rep = Hq // Hkv
    tk = tk.repeat_interleave(rep, dim=1)
    tv = tv.repeat_interleave(rep, dim=1)
    tm = torch.from_numpy(mask)
    o = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=tm, scale=scale)
    s = (scale * (tq @ tk.transpose(-1, -2))).masked_fill(~tm, float("-inf"))
    lse = torch.logsumexp(s, dim=-1)
    O = np.zeros(q.shape)
    L = np.zeros((Hq, q.shape[0]))
    for b in range(B):
        O[cu_q[b]:cu_q[b + 1]] = np.transpose(o[b, :, :Nq[b]].numpy(), (1, 0, 2))
        L[:, cu_q[b]:cu_q[b + 1]] = lse[b, :, :Nq[b]].numpy()
    return O, L


@pytest.mark.parametrize("causal", [False, True])
def test_varlen_matches_padded_library_attention(causal):
    Nq = np.array([5, 0, 9, 1, 3])
    Nk = np.array([7, 3, 9, 4, 3])
    q, k, v, cu_q, cu_k = _packed_case(Nq, Nk, 4, 2, 8, 60)
    O, L = oracle.varlen_attention(q, k, v, cu_q, cu_k, 0.4, causal)
    O_ref, L_ref = _padded_library(q, k, v, cu_q, cu_k, 0.4, causal)
    np.testing.assert_allclose(O, O_ref, atol=TIGHT)
    np.testing.assert_allclose(L, L_ref, atol=TIGHT)


def test_varlen_sequences_without_keys_and_independence():
    Nq = np.array([4, 3, 5])
    Nk = np.array([6, 0, 5])
    q, k, v, cu_q, cu_k = _packed_case(Nq, Nk, 2, 1, 4, 70)
    O, L = oracle.varlen_attention(q, k, v, cu_q, cu_k, 0.5, False)
    assert np.all(O[4:7] == 0) and np.all(L[:, 4:7] == -np.inf)       # sequence 1: no keys
    # changing sequence 2's keys and values leaves sequence 0 untouched
    k2, v2 = k.copy(), v.copy()
    k2[6:] += 1.0
    v2[6:] -= 2.0
    O2, L2 = oracle.varlen_attention(q, k2, v2, cu_q, cu_k, 0.5, False)
    assert np.array_equal(O2[:4], O[:4]) and np.array_equal(L2[:, :4], L[:, :4])
    assert np.max(np.abs(O2[7:] - O[7:])) > 1e-3


def test_pins_catch_a_varlen_offset_mixup():
    """Using the query offsets for the keys (a plausible slip) fails the padded check."""
    Nq = np.array([3, 6, 2])
    Nk = np.array([8, 6, 5])
    q, k, v, cu_q, cu_k = _packed_case(Nq, Nk, 2, 2, 4, 80)
    O_ref, _ = _padded_library(q, k, v, cu_q, cu_k, 0.5, True)
    cu_bad = cu_k.copy()
    cu_bad[1:-1] = cu_q[1:-1]                 # keys split at the query boundaries
    O_bad, _ = oracle.varlen_attention(q, k, v, cu_q, cu_bad, 0.5, False)
    assert np.max(np.abs(O_bad - O_ref)) > 1e-3


def test_paged_prefill_equals_contiguous_ragged_attention():
    """Keys and values scattered into random pages of a pool (by the test, with
    plain indexing) and read back through the block table give the same result
    as the contiguous ragged batch."""
    rng = np.random.default_rng(100)
    page, Hq, Hkv, D = 4, 4, 2, 8
    Nk = np.array([9, 4, 13])
    Nq = np.array([3, 4, 5])                      # the last Nq_b tokens are the queries
    q, k, v, cu_q, cu_k = _packed_case(Nq, Nk, Hq, Hkv, D, 101)
    npages = [int(math.ceil(n / page)) for n in Nk]
    pool = 20
    perm = rng.permutation(pool)
    table = np.zeros((3, max(npages)), dtype=np.int64)
    kc = rng.standard_normal((pool, page, Hkv, D))      # other pages hold unrelated values
    vc = rng.standard_normal((pool, page, Hkv, D))
    used = 0
    for b in range(3):
        table[b, :npages[b]] = perm[used:used + npages[b]]
        used += npages[b]
        for t in range(Nk[b]):
            kc[table[b, t // page], t % page] = k[cu_k[b] + t]
            vc[table[b, t // page], t % page] = v[cu_k[b] + t]
    for causal in (False, True):
        O, L = oracle.paged_prefill(q, kc, vc, table, cu_q, Nk, 0.5, causal, page)
        O_ref, L_ref = _padded_library(q, k, v, cu_q, cu_k, 0.5, causal)
        np.testing.assert_allclose(O, O_ref, atol=TIGHT)
        np.testing.assert_allclose(L, L_ref, atol=TIGHT)


# ---------------------------------------------------------------- backward (recomputation)
@pytest.mark.parametrize("Hq,Hkv,Nq,Nk,causal", [(2, 2, 7, 7, False), (4, 2, 5, 9, True),
                                                   (4, 1, 6, 6, True)])
def test_backward_matches_float64_library_autograd(Hq, Hkv, Nq, Nk, causal):
    """dQ, dK, dV against torch autograd through float64 library attention
    (explicit bottom-right mask, K/V heads repeated for GQA)."""
    q, k, v = rand((2, Hq, Nq, 8), 130), rand((2, Hkv, Nk, 8), 131), rand((2, Hkv, Nk, 8), 132)
    do = rand((2, Hq, Nq, 8), 133)
    O, L = oracle.attention(q, k, v, 0.4, causal)
    dq, dk, dv = oracle.attention_backward(q, k, v, O, L, do, 0.4, causal)
    tq, tk, tv = (torch.from_numpy(x).requires_grad_(True) for x in (q, k, v))
    rep = Hq // Hkv
    mask = torch.ones(Nq, Nk, dtype=torch.bool).tril(diagonal=Nk - Nq) if causal else None
    o = torch.nn.functional.scaled_dot_product_attention(
        tq, tk.repeat_interleave(rep, dim=1), tv.repeat_interleave(rep, dim=1), attn_mask=mask,
        scale=0.4)
    o.backward(torch.from_numpy(do))
    np.testing.assert_allclose(dq, tq.grad.numpy(), atol=1e-10)
    np.testing.assert_allclose(dk, tk.grad.numpy(), atol=1e-10)
    np.testing.assert_allclose(dv, tv.grad.numpy(), atol=1e-10)


def test_backward_matches_finite_differences():
    """Central differences of <dO, O(Q, K, V)> on a tiny causal GQA case."""
    q, k, v = rand((1, 2, 3, 4), 134), rand((1, 1, 4, 4), 135), rand((1, 1, 4, 4), 136)
    do = rand((1, 2, 3, 4), 137)
    O, L = oracle.attention(q, k, v, 0.7, True)
    grads = oracle.attention_backward(q, k, v, O, L, do, 0.7, True)
    eps = 1e-6
    for which, g in zip(range(3), grads):
        base = [q, k, v]
        x = base[which]
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            args_p = list(base)
            args_m = list(base)
            args_p[which] = xp
            args_m[which] = xm
            fp = np.sum(do * oracle.attention(*args_p, 0.7, True)[0])
            fm = np.sum(do * oracle.attention(*args_m, 0.7, True)[0])
            num[idx] = (fp - fm) / (2 * eps)
        np.testing.assert_allclose(g, num, atol=1e-7)


def test_pins_catch_a_missing_delta_term():
    """Dropping the rowsum(dO * O) term (a plausible slip) fails the library check."""
    q, k, v = rand((1, 1, 5, 4), 138), rand((1, 1, 5, 4), 139), rand((1, 1, 5, 4), 140)
    do = rand((1, 1, 5, 4), 141)
    O, L = oracle.attention(q, k, v, 0.5, False)
    dq_bad, _, _ = oracle.attention_backward(q, k, v, np.zeros_like(O), L, do, 0.5, False)
    tq = torch.from_numpy(q).requires_grad_(True)
    o = torch.nn.functional.scaled_dot_product_attention(tq, torch.from_numpy(k),
                                                         torch.from_numpy(v), scale=0.5)
    o.backward(torch.from_numpy(do))
    assert np.max(np.abs(dq_bad - tq.grad.numpy())) > 1e-3


def test_backward_closed_forms():
    """One key: P = 1, so dV sums dO over the group's query heads and rows, and dS =
    dO.v - dO.o = 0 gives dQ = dK = 0.  Zero queries (uniform weights 1/Nk, no
    mask): dV_j = sum_i dO_i / Nk for every key j."""
    q, k, v = rand((1, 4, 3, 8), 150), rand((1, 2, 1, 8), 151), rand((1, 2, 1, 8), 152)
    do = rand((1, 4, 3, 8), 153)
    O, L = oracle.attention(q, k, v, 0.3, False)
    dq, dk, dv = oracle.attention_backward(q, k, v, O, L, do, 0.3, False)
    np.testing.assert_allclose(dq, 0, atol=1e-12)
    np.testing.assert_allclose(dk, 0, atol=1e-12)
    want = do.reshape(1, 2, 2, 3, 8).sum(axis=(2, 3))[:, :, None, :]
    np.testing.assert_allclose(dv, want, atol=1e-12)
    qz = np.zeros((1, 2, 5, 8))
    k2, v2 = rand((1, 2, 6, 8), 154), rand((1, 2, 6, 8), 155)
    do2 = rand((1, 2, 5, 8), 156)
    O2, L2 = oracle.attention(qz, k2, v2, 0.3, False)
    _, _, dv2 = oracle.attention_backward(qz, k2, v2, O2, L2, do2, 0.3, False)
    np.testing.assert_allclose(dv2, np.repeat(do2.sum(axis=2, keepdims=True) / 6, 6, axis=2),
                               atol=1e-12)
