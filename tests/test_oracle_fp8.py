"""Pins of the FP8 (E4M3) oracle pieces: against torch's E4M3 conversion and
byte view (library routines), the format's closed forms, the Walsh-Hadamard
matrix's entries in closed form, orthogonality and the invariance of Q K^T
under the rotation, agreement of the fp32-decision quantiser with the fp64
definition, and exactness when the inputs are already representable."""
import numpy as np
import pytest
import torch

import oracle
from oracle import fp8_e4m3 as f8
from exact_tiled_attention_40_b200.inputs import hadamard_signs


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


def test_byte_decoding_matches_the_library_view_of_all_256_bytes():
    b = np.arange(256)
    lib = torch.from_numpy(b.astype(np.uint8)).view(torch.float8_e4m3fn).double().numpy()
    ours = f8.e4m3_from_bits(b)
    np.testing.assert_array_equal(np.isnan(ours), np.isnan(lib))
    ok = ~np.isnan(lib)
    np.testing.assert_array_equal(ours[ok], lib[ok])
    np.testing.assert_array_equal(np.signbit(ours[ok]), np.signbit(lib[ok]))   # -0 is 0x80
    # encoding inverts decoding on every non-NaN byte
    np.testing.assert_array_equal(f8.e4m3_to_bits(ours[ok]), b[ok])
    assert f8.e4m3_to_bits([448.0, -448.0, 2.0 ** -9, -0.0]).tolist() == [0x7E, 0xFE, 0x01, 0x80]
    with pytest.raises(ValueError):
        f8.e4m3_to_bits([1.1])                    # not an E4M3 number


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


@pytest.mark.parametrize("D", [2, 4, 64, 128])
def test_walsh_hadamard_transform_gives_the_closed_form_entries(D):
    """Row i of the transform of the identity is H[i, j] = (-1)^popcount(i & j)."""
    closed = np.array([[(-1.0) ** bin(i & j).count("1") for j in range(D)] for i in range(D)])
    np.testing.assert_array_equal(f8.sylvester_hadamard(D), closed)
    np.testing.assert_array_equal(f8.walsh_hadamard_f32(np.eye(D)), closed)


def test_walsh_hadamard_f32_is_the_matrix_product_up_to_fp32_rounding():
    rng = np.random.default_rng(128)
    x = rng.standard_normal((50, 128)).astype(np.float32)
    exact = x.astype(np.float64) @ f8.sylvester_hadamard(128)
    got = f8.walsh_hadamard_f32(x)
    assert got.dtype == np.float32
    # seven stages, each one fp32 rounding of a partial sum of at most |x| summed
    bound = 7 * 2.0 ** -24 * (np.abs(x).astype(np.float64).sum(-1, keepdims=True))
    assert np.all(np.abs(got - exact) <= bound)


def test_hadamard_rotation_is_orthogonal_and_keeps_scores():
    s = hadamard_signs(64, 122).numpy()
    Hm = f8.hadamard_rotation(s)
    np.testing.assert_allclose(Hm @ Hm.T, np.eye(64), atol=1e-12)
    rng = np.random.default_rng(123)
    q = rng.standard_normal((40, 64))
    k = rng.standard_normal((50, 64))
    np.testing.assert_allclose((q @ Hm) @ (k @ Hm).T, q @ k.T, atol=1e-10)
    assert not np.allclose(f8.hadamard_rotation(hadamard_signs(64, 124).numpy()), Hm)
    # the fp32 rotation is the same map up to fp32 rounding
    x = rng.standard_normal((30, 64)).astype(np.float32)
    np.testing.assert_allclose(f8.rotate_rows_f32(x, s), x.astype(np.float64) @ Hm,
                               rtol=0, atol=1e-5)


def test_fp32_decisions_agree_with_the_fp64_definition():
    """The kernel-precision quantiser picks the fp64 definition's code except,
    rarely, one step away where fp32 rounding moves a value across a rounding
    boundary; its scales are amax / 448 to fp32 accuracy."""
    rng = np.random.default_rng(129)
    x = (rng.standard_normal((2, 2, 300, 64)) * 3).astype(np.float32)
    c32, s32 = f8.quantize_rows_f32(x, 128)
    c64, s64 = f8.quantize_rows(x.astype(np.float64), 128)
    assert s32.shape == s64.shape == (2, 2, 3) and s32.dtype == np.float32
    np.testing.assert_allclose(s32, s64, rtol=2.0 ** -23, atol=0)
    diff = c32 != c64
    assert diff.mean() < 1e-3
    # one E4M3 quantum apart where they differ
    q = np.exp2(np.clip(np.floor(np.log2(np.maximum(np.abs(c64[diff]), 2.0 ** -9))), -6, 8) - 3)
    assert np.all(np.abs(c32[diff] - c64[diff]) <= q * 1.0000001)
    # whole-slice groups: one scale per [N, D] slice
    cs, ss = f8.quantize_rows_f32(x, 0)
    assert ss.shape == (2, 2, 1)
    np.testing.assert_allclose(ss[..., 0], np.abs(x).max(axis=(-2, -1)) / 448.0, rtol=2.0 ** -23)


def test_fp32_quantiser_closed_forms():
    g = f8.e4m3_round(np.random.default_rng(130).standard_normal((1, 200, 16)) * 30)
    g[0, 5, 3] = 448.0                          # every group's amax is 448: r = s = 1
    g[0, 130, 0] = -448.0
    c, s = f8.quantize_rows_f32(g, 128)
    np.testing.assert_array_equal(s, np.ones((1, 2), np.float32))
    np.testing.assert_array_equal(c, g)         # grid values are their own codes
    z = np.zeros((1, 130, 8), np.float32)
    z[0, 129, 0] = -0.0
    c, s = f8.quantize_rows_f32(z, 128)
    np.testing.assert_array_equal(s, np.ones((1, 2), np.float32))   # zero group: scale 1
    assert np.all(c == 0)
    # an empty slice: no codes, scale 1 (one group per slice)
    c, s = f8.quantize_rows_f32(np.zeros((2, 0, 8), np.float32), 0)
    assert c.shape == (2, 0, 8) and s.shape == (2, 1) and np.all(s == 1)
    c, s = f8.quantize_rows_f32(np.zeros((2, 0, 8), np.float32), 128)
    assert s.shape == (2, 0)
    # a value far below the group's amax rounds to zero with its sign kept
    t = np.array([[[448.0, -1e-6]]], np.float32)
    c, _ = f8.quantize_rows_f32(t, 128)
    assert c[0, 0, 1] == 0 and np.signbit(c[0, 0, 1])


def test_representable_inputs_give_the_exact_definition():
    """Inputs already on the E4M3 grid with group amax 448 quantise without error."""
    rng = np.random.default_rng(125)

    def grid(shape):
        x = f8.e4m3_round(rng.standard_normal(shape) * 40)
        x[..., 0, 0] = 448.0                          # group amax 448 -> scale 1
        return x
    q, k, v = grid((1, 2, 100, 16)), grid((1, 1, 100, 16)), grid((1, 1, 100, 16))
    O_ref, L_ref = oracle.attention(q, k, v, 0.01, True)
    O, L = f8.fp8_attention_reference(q, k, v, 0.01, True, block_rows=128)
    np.testing.assert_allclose(O, O_ref, atol=1e-12)
    np.testing.assert_allclose(L, L_ref, atol=1e-12)
    O2, L2, _ = f8.fp8_attention_f32_decisions(q, k, v, 0.01, True)
    np.testing.assert_allclose(O2, O_ref, atol=1e-12)
    np.testing.assert_allclose(L2, L_ref, atol=1e-12)


def test_fp32_and_fp64_quantisation_give_nearly_the_same_attention():
    rng = np.random.default_rng(131)
    q, k, v = (rng.standard_normal((1, 2, 200, 64)) for _ in range(3))
    s = hadamard_signs(64, 132).numpy()
    O64, L64 = f8.fp8_attention_reference(q, k, v, 0.125, False, signs=s)
    O32, L32, _ = f8.fp8_attention_f32_decisions(q, k, v, 0.125, False, signs=s)
    assert np.abs(O32 - O64).max() < 2e-3
    assert np.abs(L32 - L64).max() < 1e-3


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
    O_rot, _ = f8.fp8_attention_reference(q, k, v, 0.02, False,
                                          signs=hadamard_signs(64, 127).numpy())
    assert np.abs(O_rot - O).max() < np.abs(O_plain - O).max()
    O_rot32, _, _ = f8.fp8_attention_f32_decisions(q, k, v, 0.02, False,
                                                    signs=hadamard_signs(64, 127).numpy())
    assert np.abs(O_rot32 - O).max() < np.abs(O_plain - O).max()
