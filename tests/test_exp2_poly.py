"""The forward kernel's FMA-pipe exp2 (exp2_fma_pair in csrc/ptx_sm100.cuh),
re-evaluated step by step in float32 on the CPU with the coefficients read from
the source, against the exact 2^x: its relative error must stay below 1e-4 over
the kernel's input range [-125, 8] (2^-125 stands in below that), far under the
2^-9 rounding of P to bf16 that follows."""
import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(__file__), "..", "exact_tiled_attention_40_b200", "csrc",
                   "ptx_sm100.cuh")


def coefficients():
    body = open(SRC).read().split("exp2_fma_pair", 1)[1].split("}", 1)[0]
    hexes = re.findall(r"f2_pack\((0x[0-9a-fA-Fp.+-]+)f,", body)
    vals = [float.fromhex(h) for h in hexes]
    assert len(vals) == 4, vals
    c3, c2, c1, c0 = vals          # order of appearance in the Horner steps
    return np.float32(c0), np.float32(c1), np.float32(c2), np.float32(c3)


def exp2_like_kernel(x):
    c0, c1, c2, c3 = coefficients()
    x = np.maximum(x.astype(np.float32), np.float32(-125.0))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    f = (x - (t - magic).astype(np.float32)).astype(np.float32)
    p = (f * c3 + c2).astype(np.float32)
    p = (p * f + c1).astype(np.float32)
    p = (p * f + c0).astype(np.float32)
    bits = p.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << 23)
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def test_relative_error_over_kernel_range():
    x = np.concatenate([np.linspace(-125.0, 8.0, 400001), np.arange(-125, 9) + 0.5,
                        np.arange(-125, 9).astype(np.float64)])
    y = exp2_like_kernel(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float32).astype(np.float64))
    rel = np.abs(y - ref) / ref
    assert rel.max() < 1e-4, rel.max()


def test_clamps_tiny_inputs_to_a_normal_number():
    y = exp2_like_kernel(np.array([-1000.0, -126.0, -np.inf], dtype=np.float32))
    assert np.all(np.isfinite(y)) and np.all(y > 0) and np.all(y < 3e-38)
