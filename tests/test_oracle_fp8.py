"""Pins of the FP8 (E4M3) oracle pieces: against torch's E4M3 conversion (a
library routine), the format's closed forms, the orthogonality of the random
Hadamard matrix and the invariance of Q K^T under it, and exactness when the
inputs are already representable."""
import numpy as np
import torch

import oracle
from oracle import fp8_e4m3 as f8


def test_rounding_matches_library_conversion_inside_the_range():
    rng = np.random.default_rng(120)
    x = np.concatenate([rng.standard_normal(20000) * s for s in (1e-3, 0.05, 1, 20, 150)])
    x = x[np.abs(x) < 464]                       # beyond this torch gives NaN, we saturate
    ref = torch.from_numpy(x).to(torch.float32).to(torch.float8_e4m3fn).double().numpy()
    # the float32 step is exact for these doubles' nearest E4M3 except at exact ties,
    # which random doubles do not hit
    np.testing.assert_array_equal(f8.e4m3_round(x), ref)


def test_closed_forms():
    r = f8.e4m3_round
    assert r(448.0) == 448.0 and r(1e6) == 448.0 and r(-1e6) == -448.0     # saturation
    assert r(2.0 ** -9) == 2.0 ** -9                      # smallest subnormal
    assert r(2.0 ** -10) == 0.0                           # tie between 0 and 2^-9 -> even (0)
    assert r(1.0625) == 1.0 and r(1.1875) == 1.25         # ties to even mantissa
    assert r(-3.3) == -3.25
    assert np.isnan(r(np.nan))
    # every finite E4M3 value is a fixed point
    vals = [m * 2.0 ** (e - 3) for e in range(-6, 9) for m in range(8, 16)]
    vals += [m * 2.0 ** -9 for m in range(0, 8)]
    vals = np.array([v for v in vals if v <= 448.0])
    np.testing.assert_array_equal(r(vals), vals)
    np.testing.assert_array_equal(r(-vals), -vals)


def test_block_quantisation_round_trip_error_is_within_half_a_unit():
    rng = np.random.default_rng(121)
    x = rng.standard_normal((2, 3, 300, 16)) * np.exp(rng.standard_normal((2, 3, 300, 1)))
    codes, s = f8.quantize_rows(x, 128)
    assert s.shape == (2, 3, 3)
    assert np.all(np.abs(codes) <= 448.0)
    back = f8.dequantize_rows(codes, s, 128)
    # relative error of a normal E4M3 value is at most 2^-4; subnormal ones within 2^-10 * scale
    rep = np.repeat(s, 128, axis=-1)[..., :300, None]
    assert np.all(np.abs(back - x) <= np.maximum(np.abs(x) * 2.0 ** -4, rep * 2.0 ** -10) + 1e-15)


def test_random_hadamard_is_orthogonal_and_keeps_scores():
    Hm = f8.random_hadamard(64, 122)
    np.testing.assert_allclose(Hm @ Hm.T, np.eye(64), atol=1e-12)
    rng = np.random.default_rng(123)
    q = rng.standard_normal((40, 64))
    k = rng.standard_normal((50, 64))
    np.testing.assert_allclose((q @ Hm) @ (k @ Hm).T, q @ k.T, atol=1e-10)
    assert not np.allclose(f8.random_hadamard(64, 124), Hm)     # the seed matters


def test_representable_inputs_give_the_exact_definition():
    """Inputs already on the E4M3 grid with block amax 448 quantise without error."""
    rng = np.random.default_rng(125)
    def grid(shape):
        x = f8.e4m3_round(rng.standard_normal(shape) * 40)
        x[..., 0, 0] = 448.0                          # block amax 448 -> scale 1
        return x
    q, k, v = grid((1, 2, 100, 16)), grid((1, 1, 100, 16)), grid((1, 1, 100, 16))
    O, L = f8.fp8_attention_reference(q, k, v, 0.01, True, block_rows=128)
    O_ref, L_ref = oracle.attention(q, k, v, 0.01, True)
    np.testing.assert_allclose(O, O_ref, atol=1e-12)
    np.testing.assert_allclose(L, L_ref, atol=1e-12)


def test_incoherent_processing_lowers_the_error_for_outlier_features():
    """With a few large coordinates (outliers) in Q and K, the rotation spreads
    them and the FP8 scores come closer to the exact ones."""
    rng = np.random.default_rng(126)
    q = rng.standard_normal((1, 1, 256, 64))
    k = rng.standard_normal((1, 1, 256, 64))
    q[..., 3] *= 60.0
    k[..., 3] *= 60.0
    v = rng.standard_normal((1, 1, 256, 64))
    O, _ = oracle.attention(q, k, v, 0.02, False)
    O_plain, _ = f8.fp8_attention_reference(q, k, v, 0.02, False)
    O_rot, _ = f8.fp8_attention_reference(q, k, v, 0.02, False, rotate_seed=127)
    assert np.abs(O_rot - O).max() < np.abs(O_plain - O).max()
