"""Seeded synthetic inputs shared by the tests, the bench and the oracle checks.

This module only draws random numbers and lays them out; it holds none of the
attention arithmetic.  Everything is generated on the CPU with one
``torch.Generator`` per case so that the CUDA path and the fp64 oracle read the
very same bf16/fp16 values.

Recipe (prefill): one generator seeded with the case seed; Q, then K, then V,
each drawn head by head in (b, h) order as ``randn(N, D)`` in fp32, multiplied
by the case amplitude and rounded to the storage dtype with torch's
round-to-nearest-even conversion.  Sampled rows for long sequences are drawn
from the same generator after V.

Recipe (paged decode): one generator seeded with the case seed; the sequence
lengths ``randint(lo, hi + 1, (B,))``; a permutation of the page pool; each
sequence takes ceil(len / page_size) pages from the permutation in sequence
order (so no page is shared); then q ``randn(B, Hq, D)``; then the K pool and
the V pool, each drawn in chunks of 1024 pages as ``randn(c, page_size, Hkv, D)``.
Unused block-table entries are 0.

Recipe (paged prefill): one generator seeded with the case seed; key lengths
``randint(lo, hi + 1, (B,))`` (or listed); query counts listed or equal to the
key lengths; a permutation of the page pool handed out in sequence order as for
paged decode; then packed Q [total_q, Hq, D], then the K pool and the V pool
``randn(num_pages, 16, Hkv, D)``.

Recipe (backward): the prefill case's inputs, then the output gradient dO drawn
from the same generator after V as ``randn(B, Hq, Nq, D)`` rounded to bf16 (sampled
rows, where used, come after dO).

Recipe (FP8 forward): the bf16 inputs of the named prefill case, drawn as
above; the rotation's D signs from their own generator seeded with the case's
sign seed, ``rand(D) < 0.5`` giving -1.

Recipe (ragged prefill): one generator seeded with the case seed; the key
lengths ``randint(lo, hi + 1, (B,))`` unless the case lists them; query lengths
equal to the key lengths (or listed); then packed Q [total_q, Hq, D], K and V
[total_k, Hkv, D], each ``randn`` in fp32 rounded to the storage dtype.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

__all__ = ["PrefillCase", "DecodeCase", "VarlenCase", "PREFILL_CASES", "DECODE_CASES",
           "VARLEN_CASES", "PagedPrefillCase", "PAGED_PREFILL_CASES", "make_paged_prefill",
           "make_prefill",
           "make_decode", "make_varlen", "varlen_flops",
           "sample_rows", "hadamard_signs", "Fp8Case", "FP8_CASES", "make_dout"]

_DTYPES = {"bf16": torch.bfloat16, "fp16": torch.float16}


@dataclass(frozen=True)
class PrefillCase:
    name: str
    B: int
    Hq: int
    Hkv: int
    Nq: int
    Nk: int
    D: int
    dtype: str = "bf16"
    seed: int = 0
    causal: bool = False
    amp: float = 1.0
    scale: float = field(default=float("nan"))

    @property
    def softmax_scale(self) -> float:
        return 1.0 / math.sqrt(self.D) if math.isnan(self.scale) else self.scale

    @property
    def flops(self) -> float:
        """Attention FLOP count 4*B*Hq*Nq*Nk*D, halved under the causal mask."""
        f = 4.0 * self.B * self.Hq * self.Nq * self.Nk * self.D
        return f / 2 if self.causal else f

    @property
    def algorithmic_bytes(self) -> int:
        """Read Q, K, V once and write O (storage dtype) and LSE (fp32) once."""
        e = 2
        q = self.B * self.Hq * self.Nq * self.D * e
        kv = 2 * self.B * self.Hkv * self.Nk * self.D * e
        o = self.B * self.Hq * self.Nq * self.D * e
        lse = self.B * self.Hq * self.Nq * 4
        return q + kv + o + lse


@dataclass(frozen=True)
class DecodeCase:
    name: str
    B: int
    Hq: int
    Hkv: int
    D: int
    page_size: int
    len_lo: int
    len_hi: int
    num_pages: int
    seed: int
    dtype: str = "bf16"

    @property
    def softmax_scale(self) -> float:
        return 1.0 / math.sqrt(self.D)

    @property
    def max_pages_per_seq(self) -> int:
        return -(-self.len_hi // self.page_size)


# The workloads of the pages, synthetic (N(0,1) values; shapes as on the pages).
PREFILL_CASES = {
    "tiny_b1_h2_n256_d64": PrefillCase("tiny_b1_h2_n256_d64", 1, 2, 2, 256, 256, 64,
                                       "bf16", seed=0, causal=False),
    "mha_b2_h8_n4096_d64_fp16": PrefillCase("mha_b2_h8_n4096_d64_fp16", 2, 8, 8, 4096, 4096,
                                            64, "fp16", seed=1, causal=False, scale=0.125),
    "mha_b2_h8_n4096_d64_fp16_causal": PrefillCase("mha_b2_h8_n4096_d64_fp16_causal", 2, 8, 8,
                                                   4096, 4096, 64, "fp16", seed=1, causal=True,
                                                   scale=0.125),
    "gqa_b1_hq32_hkv8_n8192_d128_causal": PrefillCase("gqa_b1_hq32_hkv8_n8192_d128_causal", 1,
                                                      32, 8, 8192, 8192, 128, "bf16", seed=2,
                                                      causal=True),
    "gqa_b1_hq32_hkv8_n131072_d128_causal": PrefillCase(
        "gqa_b1_hq32_hkv8_n131072_d128_causal", 1, 32, 8, 131072, 131072, 128, "bf16",
        seed=3, causal=True, amp=0.5),
}

DECODE_CASES = {
    "decode_b64_hq32_hkv8_d128_page16": DecodeCase("decode_b64_hq32_hkv8_d128_page16", 64, 32,
                                                   8, 128, 16, 512, 8192, 40000, seed=4),
}


def _draw_heads(gen: torch.Generator, B: int, H: int, N: int, D: int, amp: float,
                dtype: torch.dtype) -> torch.Tensor:
    out = torch.empty((B, H, N, D), dtype=dtype)
    for b in range(B):
        for h in range(H):
            x = torch.randn((N, D), generator=gen, dtype=torch.float32)
            if amp != 1.0:
                x.mul_(amp)
            out[b, h] = x.to(dtype)
    return out


def make_prefill(case: PrefillCase, gen: torch.Generator | None = None):
    """Q [B,Hq,Nq,D], K and V [B,Hkv,Nk,D] on the CPU in the storage dtype.

    Returns (q, k, v, gen); ``gen`` is the generator after V, for follow-on draws.
    """
    dt = _DTYPES[case.dtype]
    if gen is None:
        gen = torch.Generator("cpu").manual_seed(case.seed)
    q = _draw_heads(gen, case.B, case.Hq, case.Nq, case.D, case.amp, dt)
    k = _draw_heads(gen, case.B, case.Hkv, case.Nk, case.D, case.amp, dt)
    v = _draw_heads(gen, case.B, case.Hkv, case.Nk, case.D, case.amp, dt)
    return q, k, v, gen


def sample_rows(case: PrefillCase, gen: torch.Generator, per_head: int,
                include_ends: bool = True):
    """(b, h, i) rows spread over every head: ``per_head`` positions per head drawn
    with ``randint(0, Nq)`` from ``gen``.  With ``include_ends`` the first two
    samples of (b=0, h=0) are replaced by rows 0 and Nq-1."""
    rows = []
    for b in range(case.B):
        for h in range(case.Hq):
            pos = torch.randint(0, case.Nq, (per_head,), generator=gen).tolist()
            rows.extend((b, h, int(i)) for i in pos)
    if include_ends and len(rows) >= 2:
        rows[0] = (0, 0, 0)
        rows[1] = (0, 0, case.Nq - 1)
    return rows


def make_decode(case: DecodeCase, with_pool: bool = True):
    """q [B,Hq,D], kcache/vcache [num_pages, page_size, Hkv, D], block_table
    [B, max_pages_per_seq] int32 and seq_lens [B] int32, all on the CPU."""
    dt = _DTYPES[case.dtype]
    gen = torch.Generator("cpu").manual_seed(case.seed)
    seq_lens = torch.randint(case.len_lo, case.len_hi + 1, (case.B,), generator=gen)
    perm = torch.randperm(case.num_pages, generator=gen)
    P = case.max_pages_per_seq
    block_table = torch.zeros((case.B, P), dtype=torch.int32)
    cursor = 0
    for b in range(case.B):
        n = -(-int(seq_lens[b]) // case.page_size)
        if cursor + n > case.num_pages:
            raise ValueError("page pool too small for the drawn sequence lengths")
        block_table[b, :n] = perm[cursor:cursor + n].to(torch.int32)
        cursor += n
    q = torch.randn((case.B, case.Hq, case.D), generator=gen, dtype=torch.float32).to(dt)
    kc = vc = None
    if with_pool:
        pools = []
        for _ in range(2):
            pool = torch.empty((case.num_pages, case.page_size, case.Hkv, case.D), dtype=dt)
            for c0 in range(0, case.num_pages, 1024):
                c = min(1024, case.num_pages - c0)
                pool[c0:c0 + c] = torch.randn((c, case.page_size, case.Hkv, case.D),
                                              generator=gen, dtype=torch.float32).to(dt)
            pools.append(pool)
        kc, vc = pools
    return q, kc, vc, block_table, seq_lens.to(torch.int32)


@dataclass(frozen=True)
class VarlenCase:
    """A ragged batch packed without padding: sequence b has nq[b] queries and
    nk[b] keys (drawn from [lo, hi] when not listed)."""
    name: str
    B: int
    Hq: int
    Hkv: int
    D: int
    dtype: str
    causal: bool
    seed: int
    lo: int = 1
    hi: int = 1
    nq: tuple = ()
    nk: tuple = ()

    @property
    def softmax_scale(self) -> float:
        return 1.0 / math.sqrt(self.D)


def varlen_lengths(case: VarlenCase, gen: torch.Generator):
    if case.nk:
        nk = torch.tensor(case.nk, dtype=torch.int64)
    else:
        nk = torch.randint(case.lo, case.hi + 1, (case.B,), generator=gen)
    nq = torch.tensor(case.nq, dtype=torch.int64) if case.nq else nk.clone()
    return nq, nk


def make_varlen(case: VarlenCase):
    """q [total_q, Hq, D], k, v [total_k, Hkv, D], cu_q, cu_k (int32 [B + 1]) on the CPU."""
    gen = torch.Generator("cpu").manual_seed(case.seed)
    nq, nk = varlen_lengths(case, gen)
    dt = torch.bfloat16 if case.dtype == "bf16" else torch.float16
    cu_q = torch.zeros(case.B + 1, dtype=torch.int32)
    cu_k = torch.zeros(case.B + 1, dtype=torch.int32)
    cu_q[1:] = torch.cumsum(nq, 0).to(torch.int32)
    cu_k[1:] = torch.cumsum(nk, 0).to(torch.int32)
    tq, tk = int(cu_q[-1]), int(cu_k[-1])
    q = torch.randn(tq, case.Hq, case.D, generator=gen).to(dt)
    k = torch.randn(tk, case.Hkv, case.D, generator=gen).to(dt)
    v = torch.randn(tk, case.Hkv, case.D, generator=gen).to(dt)
    return q, k, v, cu_q, cu_k


def varlen_flops(cu_q, cu_k, Hq: int, D: int, causal: bool) -> float:
    """4 * Hq * D * (visible query-key pairs) summed over the sequences."""
    total = 0
    for b in range(len(cu_q) - 1):
        nq = int(cu_q[b + 1] - cu_q[b])
        nk = int(cu_k[b + 1] - cu_k[b])
        if causal:
            # query i sees keys 0 .. i + nk - nq
            total += sum(min(nk, i + nk - nq + 1) for i in range(nq)) if nq else 0
        else:
            total += nq * nk
    return 4.0 * Hq * D * total


VARLEN_CASES = {
    # a serving-like mix: 16 sequences, lengths U[256, 8192], Llama-3-8B heads, causal
    "varlen_b16_hq32_hkv8_d128_causal": VarlenCase("varlen_b16_hq32_hkv8_d128_causal", 16, 32, 8,
                                                    128, "bf16", True, seed=5, lo=256, hi=8192),
}


@dataclass(frozen=True)
class PagedPrefillCase:
    """New queries of B sequences against their keys/values in a 16-token page
    pool: sequence b has nk[b] cached keys and its last nq[b] tokens query them."""
    name: str
    B: int
    Hq: int
    Hkv: int
    D: int
    causal: bool
    seed: int
    num_pages: int
    lo: int = 1
    hi: int = 1
    nq: tuple = ()
    nk: tuple = ()
    page_size: int = 16

    @property
    def softmax_scale(self) -> float:
        return 1.0 / math.sqrt(self.D)


def make_paged_prefill(case: PagedPrefillCase):
    """q [total_q, Hq, D], kcache, vcache [num_pages, 16, Hkv, D] (bf16), block_table
    [B, max_pages], cu_q [B + 1] and seq_lens_k [B] (int32), all on the CPU."""
    gen = torch.Generator("cpu").manual_seed(case.seed)
    if case.nk:
        nk = torch.tensor(case.nk, dtype=torch.int64)
    else:
        nk = torch.randint(case.lo, case.hi + 1, (case.B,), generator=gen)
    nq = torch.tensor(case.nq, dtype=torch.int64) if case.nq else nk.clone()
    npages = [(int(n) + case.page_size - 1) // case.page_size for n in nk]
    max_pages = max(1, max(npages))
    if sum(npages) > case.num_pages:
        raise ValueError("page pool too small for the drawn lengths")
    perm = torch.randperm(case.num_pages, generator=gen)
    table = torch.zeros(case.B, max_pages, dtype=torch.int32)
    used = 0
    for b, n in enumerate(npages):
        table[b, :n] = perm[used:used + n].to(torch.int32)
        used += n
    cu_q = torch.zeros(case.B + 1, dtype=torch.int32)
    cu_q[1:] = torch.cumsum(nq, 0).to(torch.int32)
    q = torch.randn(int(cu_q[-1]), case.Hq, case.D, generator=gen).to(torch.bfloat16)
    shape = (case.num_pages, case.page_size, case.Hkv, case.D)
    kc = torch.randn(shape, generator=gen).to(torch.bfloat16)
    vc = torch.randn(shape, generator=gen).to(torch.bfloat16)
    return q, kc, vc, table, cu_q, nk.to(torch.int32)


PAGED_PREFILL_CASES = {
    # chunked prefill: 16 sequences with 1024-8192 cached tokens each; the last
    # 512 tokens of every sequence are the new queries (causal), Llama-3-8B heads
    "paged_prefill_b16_chunk512_hq32_hkv8_d128": PagedPrefillCase(
        "paged_prefill_b16_chunk512_hq32_hkv8_d128", 16, 32, 8, 128, True, seed=6,
        num_pages=16 * 512, nq=(512,) * 16,
        nk=(1024, 8192, 2048, 4096, 3000, 6000, 5120, 1536, 7000, 2500, 4500, 8000, 1800, 3500,
            6500, 5000)),
}


def make_dout(case: PrefillCase, gen: torch.Generator) -> torch.Tensor:
    """Output gradient dO [B, Hq, Nq, D] for a backward pass, ``randn`` from ``gen``
    (the case's generator after V) rounded to bf16."""
    return torch.randn((case.B, case.Hq, case.Nq, case.D), generator=gen).to(torch.bfloat16)


def hadamard_signs(D: int, seed: int) -> torch.Tensor:
    """D random signs (+1.0 / -1.0, float32) for the Walsh-Hadamard rotation of
    an FP8 forward's queries and keys: ``rand(D) < 0.5`` from a generator seeded
    with ``seed`` gives -1."""
    g = torch.Generator("cpu").manual_seed(seed)
    return torch.where(torch.rand(D, generator=g) < 0.5, -1.0, 1.0).to(torch.float32)


@dataclass(frozen=True)
class Fp8Case:
    """An FP8 forward workload: the bf16 inputs of a prefill case, quantised to
    E4M3 by the library, with the rotation's signs drawn from ``sign_seed``
    (None: no rotation)."""
    name: str
    prefill: PrefillCase
    sign_seed: int | None = None


FP8_CASES = {
    "fp8_gqa_b1_hq32_hkv8_n8192_d128_causal": Fp8Case(
        "fp8_gqa_b1_hq32_hkv8_n8192_d128_causal",
        PREFILL_CASES["gqa_b1_hq32_hkv8_n8192_d128_causal"], sign_seed=12),
}
