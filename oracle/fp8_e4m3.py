"""fp64 oracle pieces for an FP8 (E4M3) attention forward.

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).  The pages name FP8 support
and "incoherent processing" (a technique that lowers the quantisation error of
low-precision formats) among FlashAttention-3's additions (unite.ai, "Flash
Attention: Revolutionizing Transformer Efficiency", section "Flash Attention-3")
without defining either.  Readings, each the plainest one the rest supports:

* FP8 means the E4M3 format of the FP8 formats used by tensor cores: 1 sign bit,
  4 exponent bits with bias 7, 3 mantissa bits, subnormals, no infinity, largest
  finite magnitude 448 = 1.75 * 2^8; conversion rounds to nearest, ties to even,
  and saturates finite values beyond 448 to +-448 (the hardware's satfinite
  conversion).
* A tensor is quantised with one fp32 scale per block of rows (the amax of the
  block divided by 448), so each block uses the whole E4M3 range.
* Incoherent processing multiplies Q and K along the head dimension by the same
  random orthogonal matrix (a Walsh-Hadamard matrix with random signs, divided
  by sqrt(D)) before quantisation; Q K^T is unchanged in exact arithmetic while
  outliers are spread over all coordinates.
* The FP8 forward's reference output is the definition applied to the
  dequantised inputs; the kernel's remaining error (P rounded before P V, the
  fp32 accumulation) is what its tolerance has to cover.

Parity status: pinned by tests/test_oracle_fp8.py (library conversion, closed
forms, orthogonality and the Q K^T invariance, exactness on representable
inputs).
"""
from __future__ import annotations

import numpy as np

from .attention_fp64 import attention

E4M3_MAX = 448.0
E4M3_MIN_NORMAL_EXP = -6      # smallest normal magnitude 2^-6
E4M3_MANTISSA_BITS = 3


def e4m3_round(x):
    """Nearest E4M3 value of each element (ties to even), saturating at +-448;
    NaN stays NaN."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    # exponent of the binade holding |x| (subnormals share the smallest normal's quantum)
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.clip(e, E4M3_MIN_NORMAL_EXP, 8)
    quantum = np.exp2(e - E4M3_MANTISSA_BITS)
    r = np.round(a / quantum) * quantum          # numpy rounds half to even
    r = np.minimum(r, E4M3_MAX)
    out = np.copysign(r, x)
    return np.where(np.isnan(x), np.nan, out)


def quantize_rows(x, block_rows: int, axis: int = -2):
    """Per-block E4M3 quantisation along `axis` (blocks of `block_rows` rows).

    Returns (codes as float64 E4M3 values, scales) with x ~= codes * scale of the
    row's block; scale = amax(block) / 448 (1 for an all-zero block)."""
    x = np.asarray(x, dtype=np.float64)
    xm = np.moveaxis(x, axis, -2)
    n = xm.shape[-2]
    nb = (n + block_rows - 1) // block_rows
    codes = np.empty_like(xm)
    scales = np.empty(xm.shape[:-2] + (nb,))
    for i in range(nb):
        blk = xm[..., i * block_rows:(i + 1) * block_rows, :]
        amax = np.max(np.abs(blk), axis=(-2, -1))
        s = np.where(amax > 0, amax / E4M3_MAX, 1.0)
        scales[..., i] = s
        codes[..., i * block_rows:(i + 1) * block_rows, :] = e4m3_round(blk / s[..., None, None])
    return np.moveaxis(codes, -2, axis), scales


def dequantize_rows(codes, scales, block_rows: int, axis: int = -2):
    codes = np.asarray(codes, dtype=np.float64)
    cm = np.moveaxis(codes, axis, -2)
    rep = np.repeat(scales, block_rows, axis=-1)[..., :cm.shape[-2]]
    return np.moveaxis(cm * rep[..., :, None], -2, axis)


def random_hadamard(D: int, seed: int):
    """Orthogonal D x D matrix: Sylvester's Walsh-Hadamard matrix with a random
    sign per row, divided by sqrt(D) (D a power of two)."""
    if D <= 0 or D & (D - 1):
        raise ValueError("D must be a power of two")
    Hm = np.array([[1.0]])
    while Hm.shape[0] < D:
        Hm = np.block([[Hm, Hm], [Hm, -Hm]])
    signs = np.where(np.random.default_rng(seed).random(D) < 0.5, -1.0, 1.0)
    return (signs[:, None] * Hm) / np.sqrt(D)


def fp8_attention_reference(q, k, v, scale: float, causal: bool, block_rows: int = 128,
                            rotate_seed: int | None = None):
    """The definition on E4M3-quantised inputs (q, k, v [B, H, N, D] real).

    With `rotate_seed`, q and k are first multiplied along D by the same random
    Hadamard matrix (incoherent processing).  Returns (O, LSE) of the dequantised
    inputs, in fp64."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    if rotate_seed is not None:
        Hm = random_hadamard(q.shape[-1], rotate_seed)
        q = q @ Hm
        k = k @ Hm
    deq = []
    for t in (q, k, v):
        codes, s = quantize_rows(t, block_rows)
        deq.append(dequantize_rows(codes, s, block_rows))
    return attention(deq[0], deq[1], deq[2], scale, causal)
