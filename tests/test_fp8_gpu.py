"""Parity of the E4M3 quantiser and the FP8 forward (through the C ABI) with the
oracle.

Quantiser: codes and scales are integer and bit decisions, compared bit for
bit with oracle.fp8_e4m3's fp32-decision quantiser on the same bf16 inputs.

FP8 forward: the oracle is the definition in fp64 on the dequantised inputs
(the oracle's own quantisation of the same bf16 tensors, which the first tests
show to equal the library's).  The kernel's remaining error is the rounding of
P to E4M3 before P V; the tolerances derive from it:
  * every element: |dO_d| <= sum_j max(2^-4 w_j, 2^-16 w_max) |v_jd|
    + 2^-8 |O_d| + 1e-4 (w the softmax weights): the kernel writes
    p = 2^(x - m_ref + 6) with its lazy reference m_ref at or below the row
    maximum, so the row's largest p is 2^6 or more; a normal E4M3 entry is
    within 2^-4 relative of p and a subnormal one (below 2^-6) within 2^-10
    absolute, i.e. 2^-16 w_max; the bf16 output rounding adds 2^-8 |O| and
    1e-4 covers fp32 arithmetic;
  * in aggregate: the rounding errors are independent, so
    sqrt(sum dO^2 / sum E^2) <= 0.06 with E^2 = sum_j w_j^2 v_j^2 (a uniform
    relative error within 2^-4 has standard deviation 0.036);
  * LSE is computed from the unrounded p: |dLSE| <= 2e-4 + 2^-13 S_abs, with
    S_abs = max_j scale * sum_d |q_d k_jd|, allowing the tensor core's fp32
    accumulation of the E4M3 products a relative error of 2^-13.
"""

import numpy as np
import pytest
import torch

import oracle
from oracle import fp8_e4m3 as f8
from exact_tiled_attention_40_b200 import fa
from exact_tiled_attention_40_b200.inputs import (FP8_CASES, PrefillCase, hadamard_signs,
                                                  make_prefill, sample_rows)

pytestmark = pytest.mark.gpu


def f32(t):
    return t.float().numpy()


def run_quant(x, group_rows, signs):
    dev = torch.device("cuda", 0)
    codes, scales = fa.quantize_e4m3(x.to(dev), group_rows,
                                     None if signs is None else signs.to(dev))
    torch.cuda.synchronize()
    assert fa.device_status() == 0, fa.last_error()
    return codes.cpu().numpy(), scales.cpu().numpy()


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("group_rows", [128, 0])
@pytest.mark.parametrize("rotate", [False, True])
def test_quantiser_codes_and_scales_are_bit_exact(cuda_device, D, group_rows, rotate):
    g = torch.Generator().manual_seed(40 + D + group_rows + int(rotate))
    x = (torch.randn((3, 300, D), generator=g) * torch.exp(torch.randn((3, 300, 1), generator=g)))
    x[1, 7, 5] = 60.0                                   # an outlier
    x[2].zero_()                                        # an all-zero slice: scale 1
    x = x.to(torch.bfloat16)
    signs = hadamard_signs(D, 41) if rotate else None
    codes, scales = run_quant(x, group_rows, signs)
    xr = f32(x) if signs is None else f8.rotate_rows_f32(f32(x), signs.numpy())
    c_ref, s_ref = f8.quantize_rows_f32(xr, group_rows)
    np.testing.assert_array_equal(codes, f8.e4m3_to_bits(c_ref))
    np.testing.assert_array_equal(scales.reshape(s_ref.shape), s_ref)


def test_quantiser_edge_sizes(cuda_device):
    """One row, a ragged last group, and N = 0 (scales still written)."""
    for N in (1, 129):
        x = torch.randn((2, N, 128), generator=torch.Generator().manual_seed(N)).to(torch.bfloat16)
        for gr in (128, 0):
            codes, scales = run_quant(x, gr, None)
            c_ref, s_ref = f8.quantize_rows_f32(f32(x), gr)
            np.testing.assert_array_equal(codes, f8.e4m3_to_bits(c_ref))
            np.testing.assert_array_equal(scales.reshape(s_ref.shape), s_ref)
    x = torch.empty((3, 0, 128), dtype=torch.bfloat16)
    _, scales = run_quant(x, 0, None)
    _, s_ref = f8.quantize_rows_f32(f32(x), 0)
    np.testing.assert_array_equal(scales, s_ref.reshape(3))


def fp8_bounds(qd, kd, vd, scale, causal, rows=None):
    """Per-element bounds of the FP8 forward's error (see the module docstring):
    (P rounding bound, E2, S_abs) for all rows, or for the sampled (b, h, i) rows."""
    B, Hq, Nq, D = qd.shape
    Hkv, Nk = kd.shape[1], kd.shape[2]
    if rows is None:
        rows = [(b, h, i) for b in range(B) for h in range(Hq) for i in range(Nq)]
    A = np.zeros((len(rows), D))
    E2 = np.zeros((len(rows), D))
    S_abs = np.zeros(len(rows))
    for r, (b, h, i) in enumerate(rows):
        g = oracle.kv_head_of(h, Hq, Hkv)
        n = min(Nk, i + (Nk - Nq) + 1) if causal else Nk
        if n <= 0:
            continue
        s = scale * (kd[b, g, :n] @ qd[b, h, i])
        w, _, _ = oracle.softmax_rows(s[None, :])
        w = w[0]
        A[r] = np.maximum(w * 2.0 ** -4, w.max() * 2.0 ** -16) @ np.abs(vd[b, g, :n])
        E2[r] = (w * w) @ (vd[b, g, :n] ** 2)
        S_abs[r] = scale * np.max(np.abs(kd[b, g, :n]) @ np.abs(qd[b, h, i]))
    return A, E2, S_abs


def check_fp8(o, lse, O_ref, L_ref, A, E2, S_abs):
    dO = np.abs(o - O_ref)
    tol = A + 2.0 ** -8 * np.abs(O_ref) + 1e-4
    worst = float((dO / tol).max())
    agg = float(np.sqrt((dO ** 2).sum() / max(E2.sum(), 1e-300)))
    dL = np.abs(lse - L_ref)
    fin = np.isfinite(L_ref)
    assert np.array_equal(np.isfinite(lse), fin)
    tol_l = 2e-4 + 2.0 ** -13 * S_abs
    assert worst <= 1.0, ("element bound", worst)
    assert agg <= 0.06, ("aggregate", agg)
    assert np.all(dL[fin] <= tol_l[fin]), ("lse", float(dL[fin].max()))
    return worst, agg


def run_fp8(q, k, v, scale, causal, signs):
    dev = torch.device("cuda", 0)
    o, lse = fa.attention_fp8(q.to(dev), k.to(dev), v.to(dev), scale, causal,
                              None if signs is None else signs.to(dev))
    torch.cuda.synchronize()
    assert fa.device_status() == 0, fa.last_error()
    return o.float().cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64)


SMALL = [
    (PrefillCase("fp8_tile", 1, 2, 1, 128, 128, 128, seed=50), None),
    (PrefillCase("fp8_ragged_causal", 1, 4, 2, 300, 300, 128, seed=51, causal=True), 52),
    (PrefillCase("fp8_ragged_plain", 2, 2, 2, 200, 520, 128, seed=53), 54),
    (PrefillCase("fp8_q_shorter_causal", 1, 4, 1, 100, 513, 128, seed=55, causal=True), None),
    (PrefillCase("fp8_many_tiles", 1, 2, 2, 1024, 1024, 128, seed=56, causal=True), 57),
    (PrefillCase("fp8_seven", 1, 2, 1, 7, 7, 128, seed=58, causal=True), None),
    (PrefillCase("fp8_peaked", 1, 2, 2, 384, 384, 128, seed=59, scale=1.0), 60),
]


@pytest.mark.parametrize("case,sign_seed", SMALL, ids=lambda c: getattr(c, "name", str(c)))
def test_fp8_forward_matches_oracle_within_derived_bounds(cuda_device, case, sign_seed):
    q, k, v, _ = make_prefill(case)
    signs = None if sign_seed is None else hadamard_signs(case.D, sign_seed)
    o, lse = run_fp8(q, k, v, case.softmax_scale, case.causal, signs)
    O_ref, L_ref, (qd, kd, vd) = f8.fp8_attention_f32_decisions(
        f32(q), f32(k), f32(v), case.softmax_scale, case.causal,
        None if signs is None else signs.numpy())
    A, E2, S_abs = fp8_bounds(qd, kd, vd, case.softmax_scale, case.causal)
    check_fp8(o.reshape(-1, case.D), lse.reshape(-1), O_ref.reshape(-1, case.D),
              L_ref.reshape(-1), A, E2, S_abs)


def test_fp8_zero_queries_average_the_values(cuda_device):
    """Q = 0: every weight is 1 / Nk, so O is the mean of the dequantised V."""
    case = PrefillCase("fp8_zero_q", 1, 2, 1, 130, 260, 128, seed=61)
    q, k, v, _ = make_prefill(case)
    q.zero_()
    o, lse = run_fp8(q, k, v, case.softmax_scale, False, None)
    _, _, (_, _, vd) = f8.fp8_attention_f32_decisions(f32(q), f32(k), f32(v),
                                                      case.softmax_scale, False)
    mean = vd.mean(axis=2, keepdims=True)
    # P = 2^6 exactly for every key: no P rounding, only the bf16 output rounding
    assert np.abs(o - mean[:, [0, 0]]).max() <= 2.0 ** -8 * np.abs(mean).max() + 1e-6
    np.testing.assert_allclose(lse, np.log(260.0), atol=1e-5)


def test_fp8_empty_keys_give_zero_output(cuda_device):
    dev = torch.device("cuda", 0)
    q8 = torch.zeros((1, 2, 5, 128), dtype=torch.uint8, device=dev)
    k8 = torch.zeros((1, 1, 0, 128), dtype=torch.uint8, device=dev)
    qs = torch.ones((2, 1), device=dev)
    ks = torch.ones((1, 0), device=dev)
    vs = torch.ones((1,), device=dev)
    o, lse = fa.attention_fp8_quantised(q8, k8, k8, qs, ks, vs, 0.1, False)
    torch.cuda.synchronize()
    assert torch.all(o == 0) and torch.all(torch.isneginf(lse))


def test_fp8_full_size_workload_sampled_rows(cuda_device):
    """The FP8 workload at full size (B1 Hq32 Hkv8 N8192 D128 causal, rotated),
    in the launch configuration the benchmark times: the codes bit-exact, and
    512 sampled rows within the derived bounds."""
    c = FP8_CASES["fp8_gqa_b1_hq32_hkv8_n8192_d128_causal"]
    case = c.prefill
    q, k, v, gen = make_prefill(case)
    rows = sample_rows(case, gen, 16)
    signs = hadamard_signs(case.D, c.sign_seed)
    dev = torch.device("cuda", 0)
    qg, kg, vg, sg = q.to(dev), k.to(dev), v.to(dev), signs.to(dev)
    q8, qs = fa.quantize_e4m3(qg, 128, sg)
    k8, ks = fa.quantize_e4m3(kg, 128, sg)
    v8, vs = fa.quantize_e4m3(vg, 0)
    o, lse = fa.attention_fp8_quantised(q8, k8, v8, qs, ks, vs, case.softmax_scale, True)
    torch.cuda.synchronize()
    assert fa.device_status() == 0, fa.last_error()
    (qc, qsr), (kc, ksr), (vc, vsr) = f8.fp8_quantise_inputs_f32(f32(q), f32(k), f32(v),
                                                                signs.numpy())
    np.testing.assert_array_equal(q8.cpu().numpy(), f8.e4m3_to_bits(qc))
    np.testing.assert_array_equal(k8.cpu().numpy(), f8.e4m3_to_bits(kc))
    np.testing.assert_array_equal(v8.cpu().numpy(), f8.e4m3_to_bits(vc))
    np.testing.assert_array_equal(qs.cpu().numpy().reshape(qsr.shape), qsr)
    qd = f8.dequantize_f32_groups(qc, qsr, 128)
    kd = f8.dequantize_f32_groups(kc, ksr, 128)
    vd = f8.dequantize_f32_groups(vc, vsr, 0)
    O_ref, L_ref = oracle.attention_rows(qd, kd, vd, case.softmax_scale, True, rows)
    A, E2, S_abs = fp8_bounds(qd, kd, vd, case.softmax_scale, True, rows)
    og = o.float().cpu().numpy().astype(np.float64)
    lg = lse.cpu().numpy().astype(np.float64)
    o_s = np.stack([og[b, h, i] for b, h, i in rows])
    l_s = np.array([lg[b, h, i] for b, h, i in rows])
    check_fp8(o_s, l_s, O_ref, L_ref, A, E2, S_abs)
