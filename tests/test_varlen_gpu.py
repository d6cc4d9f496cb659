"""Parity of fa_fwd_varlen (through the C ABI) with the fp64 ragged-batch oracle."""
import numpy as np
import pytest
import torch

import oracle
from exact_tiled_attention_40_b200 import fa
from exact_tiled_attention_40_b200.inputs import VARLEN_CASES, VarlenCase, make_varlen

pytestmark = pytest.mark.gpu
TOL_O = 2e-2
TOL_LSE = 1e-3


def f64(t):
    return t.float().double().numpy()


def run(case, q, k, v, cu_q, cu_k):
    dev = torch.device("cuda", 0)
    nq = (cu_q[1:] - cu_q[:-1]).max().item() if len(cu_q) > 1 else 0
    nk = (cu_k[1:] - cu_k[:-1]).max().item() if len(cu_k) > 1 else 0
    o, lse = fa.attention_varlen(q.to(dev), k.to(dev), v.to(dev), cu_q.to(dev), cu_k.to(dev),
                                 max(nq, 1), max(nk, 1), case.softmax_scale, case.causal)
    torch.cuda.synchronize()
    return o.cpu(), lse.cpu()


def check(case):
    q, k, v, cu_q, cu_k = make_varlen(case)
    o, lse = run(case, q, k, v, cu_q, cu_k)
    assert fa.device_status() == 0, fa.last_error()
    O_ref, L_ref = oracle.varlen_attention(f64(q), f64(k), f64(v), cu_q.numpy(), cu_k.numpy(),
                                           case.softmax_scale, case.causal)
    dO = np.abs(f64(o) - O_ref).max() if O_ref.size else 0.0
    live = np.isfinite(L_ref)
    dL = np.abs(lse.double().numpy()[live] - L_ref[live]).max() if live.any() else 0.0
    assert dO <= TOL_O and dL <= TOL_LSE, (case.name, dO, dL)
    assert np.all(lse.numpy()[~live] == -np.inf)
    return o, lse


@pytest.mark.parametrize("causal", [False, True])
def test_ragged_gqa_bf16_d128(cuda_device, causal):
    # lengths straddle the 128-row tiles and the 256-row tile pairs; one sequence is empty
    lens = (1, 128, 300, 0, 517, 64, 1000, 255)
    check(VarlenCase("ragged", len(lens), 8, 2, 128, "bf16", causal, seed=90, nq=lens, nk=lens))


def test_queries_shorter_than_keys_bottom_right(cuda_device):
    check(VarlenCase("suffix", 3, 4, 4, 128, "bf16", True, seed=91, nq=(100, 7, 300),
                     nk=(400, 7, 301)))


def test_sequence_without_keys_non_causal(cuda_device):
    o, lse = check(VarlenCase("nokeys", 3, 4, 2, 64, "bf16", False, seed=92, nq=(200, 5, 129),
                              nk=(333, 0, 256)))
    assert torch.all(o[200:205] == 0)


def test_more_sequences_than_the_sorted_list_holds(cuda_device):
    """1500 short sequences: past the 1024 whose work the kernel sorts in
    shared memory, so the CTAs walk the (pair, sequence) items in plain order."""
    check(VarlenCase("many", 1500, 4, 2, 64, "bf16", True, seed=96, lo=1, hi=300))


def test_mha_fp16_d64(cuda_device):
    check(VarlenCase("fp16", 5, 8, 8, 64, "fp16", True, seed=93, lo=1, hi=700))


def test_serving_mix_sampled_rows(cuda_device):
    """The 16-sequence, 32-head workload at full size, checked on sampled rows."""
    case = VARLEN_CASES["varlen_b16_hq32_hkv8_d128_causal"]
    q, k, v, cu_q, cu_k = make_varlen(case)
    o, lse = run(case, q, k, v, cu_q, cu_k)
    assert fa.device_status() == 0, fa.last_error()
    rng = np.random.default_rng(94)
    for b in range(case.B):
        q0, q1, k0, k1 = (int(x) for x in (cu_q[b], cu_q[b + 1], cu_k[b], cu_k[b + 1]))
        qb = np.transpose(f64(q[q0:q1]), (1, 0, 2))[None]
        kb = np.transpose(f64(k[k0:k1]), (1, 0, 2))[None]
        vb = np.transpose(f64(v[k0:k1]), (1, 0, 2))[None]
        rows = [(0, int(h), int(i)) for h, i in zip(rng.integers(0, case.Hq, 4),
                                                    rng.integers(0, q1 - q0, 4))]
        rows += [(0, 0, 0), (0, case.Hq - 1, q1 - q0 - 1)]
        O_ref, L_ref = oracle.attention_rows(qb, kb, vb, case.softmax_scale, True, rows)
        got_o = np.stack([f64(o[q0 + i, h]) for _, h, i in rows])
        got_l = np.array([float(lse[h, q0 + i]) for _, h, i in rows])
        assert np.abs(got_o - O_ref).max() <= TOL_O, b
        assert np.abs(got_l - L_ref).max() <= TOL_LSE, b


def test_bad_offsets_are_reported_and_skipped(cuda_device):
    """Offsets that decrease are caught by the kernel (device error word); the
    valid sequences are still computed."""
    case = VarlenCase("bad", 3, 4, 2, 128, "bf16", False, seed=95, nq=(50, 40, 60),
                      nk=(70, 30, 20))
    q, k, v, cu_q, cu_k = make_varlen(case)
    bad_k = cu_k.clone()
    bad_k[2] = bad_k[1] - 5                       # sequence 1 has negative key length
    o, lse = run(case, q, k, v, cu_q, bad_k)
    assert fa.device_status() == 5                # FA_ERR_DEVICE_INDEX
    O_ref, L_ref = oracle.varlen_attention(f64(q), f64(k), f64(v), cu_q.numpy(), cu_k.numpy(),
                                           case.softmax_scale, False)
    assert np.abs(f64(o[:50]) - O_ref[:50]).max() <= TOL_O      # sequence 0 unaffected
