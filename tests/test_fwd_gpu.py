"""Parity of fa_fwd / fa_fwd_fp16 (through the C ABI) with the fp64 oracle.

Tolerances: max |dO| <= 2e-2 and max |dLSE| <= 1e-3 against the fp64 oracle on
the same bf16/fp16 inputs (bf16 I/O, fp32 accumulation, P rounded to the input
type before the P V product).
"""
import numpy as np
import pytest
import torch

import oracle
from exact_tiled_attention_40_b200 import fa
from exact_tiled_attention_40_b200.inputs import PREFILL_CASES, PrefillCase, make_prefill, sample_rows

pytestmark = pytest.mark.gpu
TOL_O = 2e-2
TOL_LSE = 1e-3


def f64(t):
    return t.float().double().numpy()


def run_gpu(case, q, k, v):
    dev = torch.device("cuda", 0)
    o, lse = fa.attention(q.to(dev), k.to(dev), v.to(dev), case.softmax_scale, case.causal)
    torch.cuda.synchronize()
    assert fa.device_status() == 0, fa.last_error()
    return o.cpu(), lse.cpu()


def derived_tol_o(v):
    """O tolerance for inputs scaled beyond unit variance: rounding O to the
    16-bit output type costs <= 2^-8 |O| <= 2^-8 max|V|, and rounding P before
    the P V product costs <= 2^-8 max|V| (weights sum to 1), so 2^-7 max|V|."""
    return max(TOL_O, 2.0 ** -7 * float(v.float().abs().max()))


def check_full(case, tol_o=TOL_O):
    q, k, v, _ = make_prefill(case)
    o, lse = run_gpu(case, q, k, v)
    O_ref, L_ref = oracle.attention(f64(q), f64(k), f64(v), case.softmax_scale, case.causal)
    dO = np.abs(f64(o) - O_ref).max()
    dL = np.abs(lse.double().numpy() - L_ref).max()
    tol = derived_tol_o(v) if tol_o is None else tol_o
    assert dO <= tol and dL <= TOL_LSE, (case, dO, dL, tol)
    return dO, dL


SMALL = [
    PrefillCase("one_tile", 1, 1, 1, 128, 128, 64, seed=10),
    PrefillCase("ragged_200", 1, 2, 2, 200, 200, 128, seed=11),
    PrefillCase("ragged_causal", 1, 2, 1, 300, 300, 128, seed=12, causal=True),
    PrefillCase("single_row", 2, 2, 2, 1, 1, 64, seed=13),
    PrefillCase("seven", 1, 4, 2, 7, 7, 128, seed=14, causal=True),
    PrefillCase("tile_plus_one", 1, 2, 1, 129, 129, 64, seed=15, causal=True),
    PrefillCase("q_shorter_causal", 1, 4, 1, 100, 513, 128, seed=16, causal=True),
    PrefillCase("q_shorter_plain", 2, 2, 2, 77, 390, 64, seed=17),
    PrefillCase("gqa8", 1, 8, 1, 384, 384, 128, seed=18, causal=True),
    PrefillCase("fp16_d128", 1, 2, 2, 260, 260, 128, "fp16", seed=19, causal=True),
    PrefillCase("fp16_d64", 2, 2, 1, 520, 300, 64, "fp16", seed=20),
    PrefillCase("peaked_rescale", 1, 2, 2, 512, 512, 128, seed=24, scale=2.0),
    PrefillCase("peaked_rescale_causal", 1, 2, 1, 640, 640, 64, seed=25, causal=True,
                scale=1.5),
    PrefillCase("many_tiles", 1, 2, 2, 1024, 1024, 128, seed=22, causal=True),
]


@pytest.mark.parametrize("case", SMALL, ids=lambda c: c.name)
def test_small_cases_match_oracle(cuda_device, case):
    check_full(case)


def test_amplified_inputs_within_derived_tolerance(cuda_device):
    """Values of amplitude 2 and a sharp softmax: exercises the lazy rescale.
    The inputs lie outside the unit-variance workloads the 2e-2 bound is stated
    for, so O is checked against the bound derived from the output arithmetic
    (derived_tol_o: 2^-7 max|V|, about 0.07 here); the measured error is printed
    beside it."""
    case = PrefillCase("scale_big", 1, 2, 2, 256, 256, 64, seed=21, scale=0.9, amp=2.0)
    q, k, v, _ = make_prefill(case)
    dO, dL = check_full(case, tol_o=None)
    print(f"scale_big: max|dO| = {dO:.3e} against the derived bound {derived_tol_o(v):.3e}; "
          f"max|dLSE| = {dL:.3e}")


def test_tiny_workload(cuda_device):
    check_full(PREFILL_CASES["tiny_b1_h2_n256_d64"])


@pytest.mark.parametrize("name", ["mha_b2_h8_n4096_d64_fp16", "mha_b2_h8_n4096_d64_fp16_causal"])
def test_mha_fp16_workload_full_compare(cuda_device, name):
    check_full(PREFILL_CASES[name])


def check_sampled(case, per_head):
    q, k, v, gen = make_prefill(case)
    rows = sample_rows(case, gen, per_head)
    o, lse = run_gpu(case, q, k, v)
    kd, vd = f64(k), f64(v)            # converted once; rows then read their prefixes
    qd = q.float().double().numpy()
    O_ref, L_ref = oracle.attention_rows(qd, kd, vd, case.softmax_scale, case.causal, rows)
    idx = tuple(np.array(rows).T)
    got_o = o.float().double().numpy()[idx]
    got_l = lse.double().numpy()[idx]
    dO = np.abs(got_o - O_ref).max()
    dL = np.abs(got_l - L_ref).max()
    assert dO <= TOL_O and dL <= TOL_LSE, (case.name, dO, dL)
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()


def test_llama3_8b_gqa_causal_workload_full_compare(cuda_device):
    """Every one of the 262,144 output rows (32 heads x 8192 queries) against the
    oracle's materialised-score attention, element by element."""
    dO, dL = check_full(PREFILL_CASES["gqa_b1_hq32_hkv8_n8192_d128_causal"])
    print(f"gqa_b1_hq32_hkv8_n8192_d128_causal: max|dO| = {dO:.3e}, max|dLSE| = {dL:.3e}")


def test_long_context_131072_workload_sampled(cuda_device):
    check_sampled(PREFILL_CASES["gqa_b1_hq32_hkv8_n131072_d128_causal"], 16)


def test_empty_keys_give_zero_output(cuda_device):
    dev = torch.device("cuda", 0)
    q = torch.randn(1, 2, 5, 64, device=dev).bfloat16()
    k = torch.empty(1, 2, 0, 64, device=dev, dtype=torch.bfloat16)
    o, lse = fa.attention(q, k, k.clone(), 0.125, False)
    torch.cuda.synchronize()
    assert torch.all(o == 0) and torch.all(lse == float("-inf"))


def test_repeat_runs_are_bitwise_identical(cuda_device):
    case = PrefillCase("det", 1, 4, 2, 640, 640, 128, seed=23, causal=True)
    q, k, v, _ = make_prefill(case)
    dev = torch.device("cuda", 0)
    q, k, v = q.to(dev), k.to(dev), v.to(dev)
    o1, l1 = fa.attention(q, k, v, case.softmax_scale, True)
    o2, l2 = fa.attention(q, k, v, case.softmax_scale, True)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
