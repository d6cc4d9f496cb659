"""fp64 CPU oracle for exact scaled-dot-product attention.

TEST INFRASTRUCTURE ONLY.  Nothing in the library imports this module; only the
tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` use it.
It shares no code with the CUDA path: its only inputs are the seeded arrays that
the input generator produces, converted exactly to float64.

Every function is the plain definition written out in float64 numpy, with
library matrix products as the only primitive.  Sources (the pages are cited by
site, title and section):

* [unite]  unite.ai, "Flash Attention: Revolutionizing Transformer Efficiency"
  (Korean edition).  Opening listing ``standard_attention``: scores
  ``Q K^T / sqrt(d_k)``, a row softmax, then a product with V.  Section "The
  Mathematics of Flash Attention": formula 1 (softmax decomposition with the
  row maximum subtracted) and formula 2 (merge of two blocks' softmax results).
  Section "Implementation Details": the blockwise algorithm with running
  statistics M (row max) and L (row sum).
* [devh]   devhandbook.co.kr, "Flash Attention 2 ... PyTorch native", examples
  3 (``is_causal=True``) and 5 (GQA: 32 query heads broadcast over 8 KV heads).
* [cabseo] cabseo.com, "Advanced techniques for enhancing LLM throughput",
  sections "Memory requirements" (the KV cache), "Autoregressive and
  memory-bound operations" (one new query token per step) and "Paged
  attention" (the cache split into fixed pages).

Readings where the pages are silent or garbled (each also stated where used):

* causal mask: query i of Nq sees key j of Nk iff j <= i + (Nk - Nq)
  (bottom-right alignment; at Nq == Nk this is "query i sees keys 0..i");
* GQA: query head h uses KV head h // (Hq // Hkv) (contiguous groups);
* LSE: natural log of the row sum of exp(scale * q.k) over the unmasked keys,
  i.e. ``M + ln L`` in the page's running-statistics notation;
* a row with no unmasked key has O = 0 and LSE = -inf.

Parity status: every function here is pinned by tests/test_oracle.py (closed
forms, invariants, a hand-derived golden case, float64 library attention, and
the blockwise algorithm against the definition).
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "softmax_rows",
    "causal_allowed",
    "attention",
    "attention_rows",
    "blockwise_attention",
    "merge_partials",
    "gather_paged_kv",
    "decode_paged",
    "kv_head_of",
]


def kv_head_of(h: int, Hq: int, Hkv: int) -> int:
    """GQA head broadcast ([devh] example 5): contiguous groups of Hq/Hkv query
    heads share one KV head."""
    if Hq % Hkv != 0:
        raise ValueError("Hq must be a multiple of Hkv")
    return h // (Hq // Hkv)


def causal_allowed(Nq: int, Nk: int) -> np.ndarray:
    """Boolean [Nq, Nk] mask of allowed (query, key) pairs under the causal rule
    of [devh] example 3, bottom-right aligned: key j is visible to query i iff
    j <= i + (Nk - Nq)."""
    i = np.arange(Nq)[:, None]
    j = np.arange(Nk)[None, :]
    return j <= i + (Nk - Nq)


def softmax_rows(s: np.ndarray, allowed: np.ndarray | None = None):
    """Row softmax by the decomposition of [unite] formula 1:
    softmax(x) = exp(x - m) / sum(exp(x - m)) with m the row maximum.

    ``s`` is [..., n] float64; ``allowed`` (same shape, optional) removes keys.
    Returns (p, m, l): probabilities, row max m and row sum l of exp(x - m).
    A row with no allowed entry gets p = 0, m = -inf, l = 0.
    """
    s = np.asarray(s, dtype=np.float64)
    if allowed is not None:
        s = np.where(allowed, s, -np.inf)
    m = np.max(s, axis=-1, keepdims=True)
    finite = np.isfinite(m)
    m_safe = np.where(finite, m, 0.0)
    e = np.exp(s - m_safe)
    e = np.where(np.isfinite(s), e, 0.0)
    l = np.sum(e, axis=-1, keepdims=True)
    p = np.where(l > 0, e / np.where(l > 0, l, 1.0), 0.0)
    return p, m[..., 0], l[..., 0]


def _check_shapes(q, k, v):
    if q.ndim != 4 or k.ndim != 4 or v.ndim != 4:
        raise ValueError("q, k, v must be [B, H, N, D]")
    B, Hq, Nq, D = q.shape
    Bk, Hkv, Nk, Dk = k.shape
    if k.shape != v.shape or Bk != B or Dk != D:
        raise ValueError("k and v must be [B, Hkv, Nk, D] matching q")
    if Hq % Hkv != 0:
        raise ValueError("Hq must be a multiple of Hkv")
    return B, Hq, Hkv, Nq, Nk, D


def attention(q, k, v, scale: float, causal: bool):
    """O = softmax(scale * Q K^T [+ causal mask]) V and the row LSE.

    [unite] opening listing ``standard_attention``, with the maximum subtracted
    as in formula 1.  q is [B, Hq, Nq, D]; k, v are [B, Hkv, Nk, D]; any real
    dtype (converted exactly to float64).  Returns O [B, Hq, Nq, D] float64 and
    LSE [B, Hq, Nq] float64 (natural log).
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, Hq, Hkv, Nq, Nk, D = _check_shapes(q, k, v)
    if causal and Nq > Nk:
        raise ValueError("causal attention needs Nq <= Nk")
    O = np.zeros((B, Hq, Nq, D), dtype=np.float64)
    LSE = np.full((B, Hq, Nq), -np.inf, dtype=np.float64)
    if Nq == 0 or Nk == 0:
        return O, LSE
    allowed = causal_allowed(Nq, Nk) if causal else None
    for b in range(B):
        for h in range(Hq):
            g = kv_head_of(h, Hq, Hkv)
            s = scale * (q[b, h] @ k[b, g].T)          # materialised [Nq, Nk] scores
            p, m, l = softmax_rows(s, allowed)
            O[b, h] = p @ v[b, g]
            with np.errstate(divide="ignore"):
                LSE[b, h] = np.where(l > 0, m + np.log(np.where(l > 0, l, 1.0)), -np.inf)
    return O, LSE


def attention_rows(q, k, v, scale: float, causal: bool, rows):
    """The same definition evaluated for selected rows only.

    ``rows`` is an iterable of (b, h, i).  Each row is computed on its own from
    the full key range it may see (its causal prefix when ``causal``), so very
    long sequences can be checked row by row.  Returns O [n, D] and LSE [n].
    """
    B, Hq, Hkv, Nq, Nk, D = _check_shapes(q, k, v)
    rows = list(rows)
    O = np.zeros((len(rows), D), dtype=np.float64)
    LSE = np.full((len(rows),), -np.inf, dtype=np.float64)
    for r, (b, h, i) in enumerate(rows):
        g = kv_head_of(h, Hq, Hkv)
        n = min(Nk, i + (Nk - Nq) + 1) if causal else Nk
        if n <= 0:
            continue
        qi = np.asarray(q[b, h, i], dtype=np.float64)
        kk = np.asarray(k[b, g, :n], dtype=np.float64)
        vv = np.asarray(v[b, g, :n], dtype=np.float64)
        s = scale * (kk @ qi)
        p, m, l = softmax_rows(s[None, :])
        O[r] = p[0] @ vv
        LSE[r] = m[0] + np.log(l[0])
    return O, LSE


def blockwise_attention(q, k, v, scale: float, causal: bool, Br: int, Bc: int,
                        keep_page_bug: bool = False):
    """The blockwise algorithm of [unite] "Implementation Details", fp64.

    Outer loop over query blocks of Br rows, inner loop over key/value blocks of
    Bc keys, with running row max M (init -inf), running row sum L (init 0) and
    a normalised output O (init 0), exactly the page's loop order and state.

    The page's update of O multiplies the old O by exp(M_old - M_new) only; since
    its O is stored normalised (divided by L_old), the old term also needs the
    factor L_old.  This function applies that correction:
        O_new = (L_old * exp(M_old - M_new) * O_old + exp(S - M_new) V) / L_new.
    ``keep_page_bug=True`` reproduces the printed update verbatim; the tests use
    it to show that the pins catch that mistake.

    Returns O [B, Hq, Nq, D] and LSE = M + ln L [B, Hq, Nq].
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, Hq, Hkv, Nq, Nk, D = _check_shapes(q, k, v)
    O = np.zeros((B, Hq, Nq, D))
    L = np.zeros((B, Hq, Nq, 1))
    M = np.full((B, Hq, Nq, 1), -np.inf)
    allowed_full = causal_allowed(Nq, Nk) if causal else np.ones((Nq, Nk), dtype=bool)
    for b in range(B):
        for h in range(Hq):
            g = kv_head_of(h, Hq, Hkv)
            for i in range(0, Nq, Br):
                Qb = q[b, h, i:i + Br]
                Ob = O[b, h, i:i + Br]
                Lb = L[b, h, i:i + Br]
                Mb = M[b, h, i:i + Br]
                for j in range(0, Nk, Bc):
                    Kb = k[b, g, j:j + Bc]
                    Vb = v[b, g, j:j + Bc]
                    S = scale * (Qb @ Kb.T)
                    S = np.where(allowed_full[i:i + Br, j:j + Bc], S, -np.inf)
                    M_new = np.maximum(Mb, S.max(axis=-1, keepdims=True))
                    # rows that have seen no visible key yet keep M = -inf
                    M_ref = np.where(np.isfinite(M_new), M_new, 0.0)
                    exp_S = np.where(np.isfinite(S), np.exp(S - M_ref), 0.0)
                    exp_M_diff = np.where(np.isfinite(Mb), np.exp(Mb - M_ref), 0.0)
                    L_new = exp_M_diff * Lb + exp_S.sum(axis=-1, keepdims=True)
                    old = exp_M_diff * Ob if keep_page_bug else exp_M_diff * Lb * Ob
                    denom = np.where(L_new > 0, L_new, 1.0)
                    Ob = np.where(L_new > 0, (old + exp_S @ Vb) / denom, 0.0)
                    Lb, Mb = L_new, M_new
                O[b, h, i:i + Br] = Ob
                L[b, h, i:i + Br] = Lb
                M[b, h, i:i + Br] = Mb
    with np.errstate(divide="ignore"):
        LSE = np.where(L[..., 0] > 0, M[..., 0] + np.log(np.where(L[..., 0] > 0, L[..., 0], 1.0)),
                       -np.inf)
    return O, LSE


def merge_partials(o_parts, lse_parts):
    """Merge softmax-normalised partial results over disjoint key sets.

    [unite] formula 2 (softmax merge), read as: with m = max of the parts' maxima,
    each part's unnormalised sum is rescaled by exp(m_part - m).  In LSE form a
    part s with normalised output O_s and log-sum-exp lse_s contributes weight
    exp(lse_s - lse) with lse = log(sum_s exp(lse_s)) (the maximum is subtracted
    before the exponentials).  Parts with lse = -inf carry no keys.

    o_parts [S, ..., D], lse_parts [S, ...]  ->  (O [..., D], LSE [...]).
    """
    o_parts = np.asarray(o_parts, dtype=np.float64)
    lse_parts = np.asarray(lse_parts, dtype=np.float64)
    m = np.max(lse_parts, axis=0)
    m_safe = np.where(np.isfinite(m), m, 0.0)
    w = np.where(np.isfinite(lse_parts), np.exp(lse_parts - m_safe), 0.0)
    tot = np.sum(w, axis=0)
    with np.errstate(divide="ignore"):
        lse = np.where(tot > 0, m_safe + np.log(np.where(tot > 0, tot, 1.0)), -np.inf)
    wn = np.where(tot > 0, w / np.where(tot > 0, tot, 1.0), 0.0)
    O = np.sum(wn[..., None] * o_parts, axis=0)
    return O, lse


def gather_paged_kv(cache, block_table, seq_len: int, b: int, page_size: int):
    """Contiguous [Hkv, seq_len, D] view of sequence b's keys (or values).

    [cabseo] "Paged attention": the cache is a pool of fixed-size pages and a
    per-sequence block table lists the pages holding its tokens in order.
    ``cache`` is [num_pages, page_size, Hkv, D]; token t of sequence b lives in
    page block_table[b, t // page_size], slot t % page_size.
    """
    t = np.arange(seq_len)
    pages = np.asarray(block_table)[b, t // page_size].astype(np.int64)
    slots = t % page_size
    tokens = np.asarray(cache)[pages, slots]              # [seq_len, Hkv, D]
    return np.transpose(tokens, (1, 0, 2)).astype(np.float64)


def decode_paged(q, kcache, vcache, block_table, seq_lens, scale: float, page_size: int):
    """One new query token per sequence attending over its cached keys/values.

    [cabseo] "Memory requirements" and "Autoregressive and memory-bound
    operations" (decode reads the whole KV cache for one query vector) and
    "Paged attention" (the cache is reached through a block table).  Each
    sequence's K and V are gathered into contiguous arrays and the definition
    ``attention`` is applied with Nq = 1 and no mask beyond the sequence length.

    q [B, Hq, D]; kcache, vcache [num_pages, page_size, Hkv, D];
    block_table [B, max_pages] int; seq_lens [B] int.
    Returns O [B, Hq, D] and LSE [B, Hq].
    """
    q = np.asarray(q, dtype=np.float64)
    B, Hq, D = q.shape
    Hkv = kcache.shape[2]
    O = np.zeros((B, Hq, D))
    LSE = np.full((B, Hq), -np.inf)
    for b in range(B):
        n = int(seq_lens[b])
        if n <= 0:
            continue
        kb = gather_paged_kv(kcache, block_table, n, b, page_size)
        vb = gather_paged_kv(vcache, block_table, n, b, page_size)
        o, lse = attention(q[b][None, :, None, :], kb[None], vb[None], scale, causal=False)
        O[b] = o[0, :, 0, :]
        LSE[b] = lse[0, :, 0]
    return O, LSE


def varlen_attention(q, k, v, cu_seqlens_q, cu_seqlens_k, scale: float, causal: bool):
    """Attention over a ragged batch packed without padding.

    [devh] example 3 combines the causal rule with a padding mask, and [cabseo]
    "Continuous batching" groups sequences of different lengths in one batch.
    Reading: a packed batch of B sequences is the padded batch with a key
    padding mask, where sequence b's queries see only sequence b's keys.
    Sequence b owns query rows [cu_seqlens_q[b], cu_seqlens_q[b+1]) and key rows
    [cu_seqlens_k[b], cu_seqlens_k[b+1]); the definition ``attention`` is
    applied to each sequence on its own (causal: bottom-right aligned within the
    sequence).

    q [total_q, Hq, D]; k, v [total_k, Hkv, D]; cu_seqlens_* int [B + 1].
    Returns O [total_q, Hq, D] and LSE [Hq, total_q] (natural log).
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    cq = np.asarray(cu_seqlens_q, dtype=np.int64)
    ck = np.asarray(cu_seqlens_k, dtype=np.int64)
    if cq.shape != ck.shape or cq.ndim != 1 or cq[0] != 0 or ck[0] != 0:
        raise ValueError("cu_seqlens must be [B + 1] offsets starting at 0")
    if np.any(np.diff(cq) < 0) or np.any(np.diff(ck) < 0):
        raise ValueError("cu_seqlens must be non-decreasing")
    total_q, Hq, D = q.shape
    O = np.zeros((total_q, Hq, D))
    LSE = np.full((Hq, total_q), -np.inf)
    for b in range(len(cq) - 1):
        q0, q1, k0, k1 = cq[b], cq[b + 1], ck[b], ck[b + 1]
        if q1 == q0:
            continue
        qb = np.transpose(q[q0:q1], (1, 0, 2))[None]      # [1, Hq, Nq_b, D]
        kb = np.transpose(k[k0:k1], (1, 0, 2))[None]      # [1, Hkv, Nk_b, D]
        vb = np.transpose(v[k0:k1], (1, 0, 2))[None]
        o, lse = attention(qb, kb, vb, scale, causal)
        O[q0:q1] = np.transpose(o[0], (1, 0, 2))
        LSE[:, q0:q1] = lse[0]
    return O, LSE


def paged_prefill(q, kcache, vcache, block_table, cu_seqlens_q, seq_lens_k, scale: float,
                  causal: bool, page_size: int):
    """Prefill of new query tokens against keys/values held in a paged cache.

    [cabseo] "Paged attention" (the cache is reached page by page through a
    block table) combined with the ragged batches of ``varlen_attention``:
    sequence b's queries are rows [cu_seqlens_q[b], cu_seqlens_q[b+1]) of q and
    its keys are the first seq_lens_k[b] tokens of its pages.  Reading: with
    ``causal`` the queries are the last Nq_b tokens of the sequence (bottom-right
    alignment), as when a prompt is prefilled in chunks.

    q [total_q, Hq, D]; kcache, vcache [num_pages, page_size, Hkv, D];
    block_table [B, max_pages] int; cu_seqlens_q [B + 1]; seq_lens_k [B].
    Returns O [total_q, Hq, D] and LSE [Hq, total_q].
    """
    q = np.asarray(q, dtype=np.float64)
    cq = np.asarray(cu_seqlens_q, dtype=np.int64)
    lens = np.asarray(seq_lens_k, dtype=np.int64)
    B = len(cq) - 1
    total_q, Hq, D = q.shape
    O = np.zeros((total_q, Hq, D))
    LSE = np.full((Hq, total_q), -np.inf)
    for b in range(B):
        q0, q1 = cq[b], cq[b + 1]
        if q1 == q0:
            continue
        n = int(lens[b])
        kb = gather_paged_kv(kcache, block_table, n, b, page_size)[None]   # [1, Hkv, n, D]
        vb = gather_paged_kv(vcache, block_table, n, b, page_size)[None]
        qb = np.transpose(q[q0:q1], (1, 0, 2))[None]
        o, lse = attention(qb, kb, vb, scale, causal)
        O[q0:q1] = np.transpose(o[0], (1, 0, 2))
        LSE[:, q0:q1] = lse[0]
    return O, LSE


def attention_backward(q, k, v, o, lse, do, scale: float, causal: bool):
    """Gradients of the attention output with respect to Q, K and V.

    [unite] section "Core Concepts", recomputation: instead of storing the
    attention matrix, the backward pass recomputes what it needs.  Reading: the
    probabilities are rebuilt from the saved row LSE as P = exp(scale * Q K^T -
    LSE) (masked entries 0), then the chain rule through O = P V and the row
    softmax gives
        dV = P^T dO,  dP = dO V^T,  dS = P * (dP - rowsum(dO * O)),
        dQ = scale * dS K,  dK = scale * dS^T Q,
    with dK, dV of a KV head summed over the query heads that share it (GQA).
    q, o, do [B, Hq, Nq, D]; k, v [B, Hkv, Nk, D]; lse [B, Hq, Nq] (natural log).
    Returns dQ, dK, dV in float64 with the shapes of q, k, v.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    o = np.asarray(o, dtype=np.float64)
    do = np.asarray(do, dtype=np.float64)
    lse = np.asarray(lse, dtype=np.float64)
    B, Hq, Hkv, Nq, Nk, D = _check_shapes(q, k, v)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    allowed = causal_allowed(Nq, Nk) if causal else np.ones((Nq, Nk), dtype=bool)
    for b in range(B):
        for h in range(Hq):
            g = kv_head_of(h, Hq, Hkv)
            s = scale * (q[b, h] @ k[b, g].T)
            finite = np.isfinite(lse[b, h])[:, None]
            p = np.where(allowed & finite, np.exp(s - np.where(finite, lse[b, h][:, None], 0.0)),
                         0.0)
            dv[b, g] += p.T @ do[b, h]
            dp = do[b, h] @ v[b, g].T
            delta = np.sum(do[b, h] * o[b, h], axis=1, keepdims=True)
            ds = p * (dp - delta)
            dq[b, h] = scale * (ds @ k[b, g])
            dk[b, g] += scale * (ds.T @ q[b, h])
    return dq, dk, dv
