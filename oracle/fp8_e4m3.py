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
* A tensor is quantised with one fp32 scale per group of rows (the amax of the
  group divided by 448), so each group uses the whole E4M3 range.  Q and K use
  groups of 128 rows (one tile); V uses one group per (sequence, head): a
  per-tile V scale would have to multiply P V_j inside the tensor core's
  accumulation, while a per-head one is applied once to the finished output.
* Incoherent processing multiplies Q and K along the head dimension by the same
  random orthogonal matrix (a Walsh-Hadamard matrix with a random sign per row,
  divided by sqrt(D)) before quantisation; Q K^T is unchanged in exact
  arithmetic while outliers are spread over all coordinates.  The random signs
  are an input (drawn by the shared input generators).
* The FP8 forward's reference output is the definition applied to the
  dequantised inputs; the kernel's remaining error (P rounded to E4M3 before
  P V, the fp32 accumulation) is what its tolerance has to cover.
* Quantisation decides integers (the codes), so the `*_f32` functions take those
  decisions in the precision the kernel computes in: fp32 values, the
  Walsh-Hadamard butterflies in fp32 in increasing bit order, the reciprocal
  448 / amax rounded to fp32 once per group and one fp32 product per element,
  then the exact E4M3 rounding of that fp32 number.

Parity status: pinned by tests/test_oracle_fp8.py (library conversion and byte
decoding, closed forms, the Walsh-Hadamard matrix's entries, orthogonality and
the Q K^T invariance, agreement of the fp32 decisions with the fp64 definition,
exactness on representable inputs).
"""
from __future__ import annotations

import numpy as np

from .attention_fp64 import attention

E4M3_MAX = 448.0
E4M3_MIN_NORMAL_EXP = -6      # smallest normal magnitude 2^-6
E4M3_MANTISSA_BITS = 3
E4M3_BIAS = 7
QK_GROUP_ROWS = 128           # rows per scale of Q and K


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


def e4m3_from_bits(bits):
    """Values of E4M3 bytes: sign bit 7, exponent bits 3-6 (bias 7), mantissa bits
    0-2; exponent 0 is subnormal (mantissa * 2^-9); 0x7f and 0xff are NaN."""
    b = np.asarray(bits, dtype=np.int64) & 0xFF
    sign = np.where(b & 0x80, -1.0, 1.0)
    e = (b >> 3) & 0xF
    m = (b & 0x7).astype(np.float64)
    mag = np.where(e == 0, m * 2.0 ** (1 - E4M3_BIAS - E4M3_MANTISSA_BITS),
                   (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - E4M3_BIAS))
    return np.where((b & 0x7F) == 0x7F, np.nan, sign * mag)


def e4m3_to_bits(vals):
    """Bytes of E4M3 values (each must be exactly representable; the sign of a
    zero is kept)."""
    v = np.asarray(vals, dtype=np.float64)
    if np.isnan(v).any():
        raise ValueError("NaN has no single E4M3 byte here")
    sign = np.signbit(v).astype(np.int64) << 7
    a = np.abs(v)
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.where(a > 0, a, 1.0))).astype(np.int64)
    normal = a >= 2.0 ** E4M3_MIN_NORMAL_EXP
    sub_m = np.round(a * 2.0 ** 9).astype(np.int64)
    nor_m = np.round((a / np.exp2(e) - 1.0) * 8.0).astype(np.int64)
    field = np.where(normal, ((e + E4M3_BIAS) << 3) | nor_m, sub_m)
    out = sign | field
    bad = e4m3_from_bits(out) != v
    if bad.any():
        raise ValueError(f"{int(bad.sum())} values are not E4M3 numbers")
    return out.astype(np.uint8)


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


def sylvester_hadamard(D: int):
    """Sylvester's D x D Walsh-Hadamard matrix of +-1 entries (D a power of two)."""
    if D <= 0 or D & (D - 1):
        raise ValueError("D must be a power of two")
    Hm = np.array([[1.0]])
    while Hm.shape[0] < D:
        Hm = np.block([[Hm, Hm], [Hm, -Hm]])
    return Hm


def hadamard_rotation(signs):
    """Orthogonal D x D matrix diag(signs) H / sqrt(D) for a vector of D signs."""
    s = np.asarray(signs, dtype=np.float64).reshape(-1)
    return (s[:, None] * sylvester_hadamard(s.size)) / np.sqrt(s.size)


def walsh_hadamard_f32(x):
    """x H along the last axis in fp32: the fast Walsh-Hadamard transform, one
    butterfly stage per bit of the index in increasing order, each stage taking
    every pair (i, i + 2^b) with bit b of i clear to (x_i + x_j, x_i - x_j)."""
    y = np.array(x, dtype=np.float32, copy=True)
    D = y.shape[-1]
    if D <= 0 or D & (D - 1):
        raise ValueError("D must be a power of two")
    h = 1
    while h < D:
        v = y.reshape(y.shape[:-1] + (D // (2 * h), 2, h))
        a = v[..., 0, :].copy()
        c = v[..., 1, :].copy()
        v[..., 0, :] = a + c
        v[..., 1, :] = a - c
        h *= 2
    return y


def rotate_rows_f32(x, signs):
    """x diag(signs) H / sqrt(D) in fp32: each element times sign * fp32(1/sqrt(D))
    (one fp32 product), then the fp32 Walsh-Hadamard transform."""
    x32 = np.asarray(x, dtype=np.float32)
    D = x32.shape[-1]
    c = np.float32(1.0 / np.sqrt(D))
    mult = (np.asarray(signs, dtype=np.float32).reshape(-1) * c).astype(np.float32)
    return walsh_hadamard_f32(x32 * mult)


def quantize_rows_f32(x, group_rows: int):
    """E4M3 codes and fp32 scales of x [..., N, D] with the decisions in fp32.

    group_rows > 0: one scale per `group_rows` rows (the last group may be
    short); 0: one scale per [N, D] slice (1 for an empty slice).  Per group: amax = max |x| (fp32),
    r = fp32(448 / amax), scale = fp32(amax / 448) (both 1 when amax = 0), and
    code = E4M3(fp32(x * r)).  Returns (codes as float64 E4M3 values, scales as
    float32 [..., groups])."""
    x32 = np.asarray(x, dtype=np.float32)
    n = x32.shape[-2]
    if group_rows == 0:                      # one group per slice, an empty one has scale 1
        codes = np.zeros(x32.shape, dtype=np.float64)
        scales = np.ones(x32.shape[:-2] + (1,), dtype=np.float32)
        if n == 0:
            return codes, scales
    g = n if group_rows == 0 else group_rows
    ng = (n + g - 1) // g
    codes = np.empty(x32.shape, dtype=np.float64)
    scales = np.empty(x32.shape[:-2] + (ng,), dtype=np.float32)
    for i in range(ng):
        blk = x32[..., i * g:(i + 1) * g, :]
        amax = np.max(np.abs(blk), axis=(-2, -1)).astype(np.float32)
        pos = amax > 0
        safe = np.where(pos, amax, np.float32(1))
        r = np.where(pos, np.float32(E4M3_MAX) / safe, np.float32(1)).astype(np.float32)
        s = np.where(pos, safe / np.float32(E4M3_MAX), np.float32(1)).astype(np.float32)
        scales[..., i] = s
        prod = (blk * r[..., None, None]).astype(np.float32)
        codes[..., i * g:(i + 1) * g, :] = e4m3_round(prod.astype(np.float64))
    return codes, scales


def dequantize_f32_groups(codes, scales, group_rows: int):
    """codes * scale of each row's group, in float64."""
    codes = np.asarray(codes, dtype=np.float64)
    n = codes.shape[-2]
    g = n if group_rows == 0 else group_rows
    rep = np.repeat(np.asarray(scales, dtype=np.float64), g, axis=-1)[..., :n]
    return codes * rep[..., :, None]


def fp8_attention_reference(q, k, v, scale: float, causal: bool, block_rows: int = 128,
                            signs=None):
    """The definition on E4M3-quantised inputs (q, k, v [B, H, N, D] real), with
    the quantisation taken in float64.

    With `signs`, q and k are first multiplied along D by hadamard_rotation(signs)
    (incoherent processing).  q and k use groups of `block_rows` rows, v one
    group per [N, D] slice.  Returns (O, LSE) of the dequantised inputs, in fp64."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    if signs is not None:
        Hm = hadamard_rotation(signs)
        q = q @ Hm
        k = k @ Hm
    deq = []
    for t in (q, k):
        codes, s = quantize_rows(t, block_rows)
        deq.append(dequantize_rows(codes, s, block_rows))
    codes, s = quantize_rows(v, max(1, v.shape[-2]))
    deq.append(dequantize_rows(codes, s, max(1, v.shape[-2])))
    return attention(deq[0], deq[1], deq[2], scale, causal)


def fp8_quantise_inputs_f32(q, k, v, signs=None):
    """The kernel-precision quantisation of an FP8 forward's inputs: q, k (rotated
    when `signs` is given) in 128-row groups and v per [N, D] slice.  Returns
    ((q codes, q scales), (k codes, k scales), (v codes, v scales))."""
    q32 = np.asarray(q, dtype=np.float32)
    k32 = np.asarray(k, dtype=np.float32)
    if signs is not None:
        q32 = rotate_rows_f32(q32, signs)
        k32 = rotate_rows_f32(k32, signs)
    return (quantize_rows_f32(q32, QK_GROUP_ROWS), quantize_rows_f32(k32, QK_GROUP_ROWS),
            quantize_rows_f32(v, 0))


def fp8_attention_f32_decisions(q, k, v, scale: float, causal: bool, signs=None):
    """The definition on the inputs as fp8_quantise_inputs_f32 quantises them.

    Returns (O, LSE, (qd, kd, vd)): fp64 output and LSE of the dequantised
    inputs, and those dequantised inputs (for error bounds)."""
    (qc, qs), (kc, ks), (vc, vs) = fp8_quantise_inputs_f32(q, k, v, signs)
    qd = dequantize_f32_groups(qc, qs, QK_GROUP_ROWS)
    kd = dequantize_f32_groups(kc, ks, QK_GROUP_ROWS)
    vd = dequantize_f32_groups(vc, vs, 0)
    O, L = attention(qd, kd, vd, scale, causal)
    return O, L, (qd, kd, vd)
