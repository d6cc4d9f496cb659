"""Parity of fa_bwd (through the C ABI) with oracle.attention_backward.

Inputs: q, k, v and the output gradient dO drawn by the shared generators; o
and lse are the oracle forward's (o rounded to bf16, lse to fp32), and the
oracle backward reads the same rounded values.  Tolerance, derived from the
kernel's arithmetic (bf16 keeps 8 significant bits: rounding to nearest is
within 2^-8 relative): P and dS are rounded to bf16 before their tensor-core
products (2^-8 each), every output is rounded to bf16 (2^-8 of the result,
itself at most the sum of its terms' magnitudes), and the fp32 recomputation of
P costs < 1e-4 relative.  So for every element
    |d dV_jd| <= (2^-7 + 1e-4) sum_i P_ij |dO_id|,
    |d dK_jd| <= (2^-7 + 1e-4) scale sum_i |dS_ij| |Q_id|,
    |d dQ_id| <= (2^-7 + 1e-4) scale sum_j |dS_ij| |K_jd|,
plus 1e-6 (summed over the query heads of a KV head for dK, dV).
"""

import numpy as np
import pytest
import torch

import oracle
from exact_tiled_attention_40_b200 import fa
from exact_tiled_attention_40_b200.inputs import (PREFILL_CASES, PrefillCase, make_dout,
                                                  make_prefill, sample_rows)

pytestmark = pytest.mark.gpu

U = 2.0 ** -7 + 1e-4


def f64(t):
    return t.float().double().numpy()


def bounds(q, k, v, o, lse, do, scale, causal):
    """Magnitude sums bounding each gradient element's rounding error."""
    B, Hq, Nq, D = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    G = Hq // Hkv
    bq = np.zeros(q.shape)
    bk = np.zeros(k.shape)
    bv = np.zeros(v.shape)
    allowed = oracle.causal_allowed(Nq, Nk) if causal else np.ones((Nq, Nk), bool)
    for b in range(B):
        for h in range(Hq):
            g = h // G
            s = scale * q[b, h] @ k[b, g].T
            P = np.where(allowed, np.exp(s - lse[b, h][:, None]), 0.0)
            dP = do[b, h] @ v[b, g].T
            delta = np.sum(do[b, h] * o[b, h], axis=1)
            dS = np.abs(P * (dP - delta[:, None]))
            bv[b, g] += P.T @ np.abs(do[b, h])
            bk[b, g] += scale * dS.T @ np.abs(q[b, h])
            bq[b, h] = scale * dS @ np.abs(k[b, g])
    return bq, bk, bv


def run_case(case):
    q, k, v, gen = make_prefill(case)
    do = make_dout(case, gen)
    O, L = oracle.attention(f64(q), f64(k), f64(v), case.softmax_scale, case.causal)
    o = torch.from_numpy(O).to(torch.bfloat16)
    lse = torch.from_numpy(L).to(torch.float32)
    dev = torch.device("cuda", 0)
    dq, dk, dv = fa.attention_backward(q.to(dev), k.to(dev), v.to(dev), o.to(dev), lse.to(dev),
                                       do.to(dev), case.softmax_scale, case.causal)
    torch.cuda.synchronize()
    assert fa.device_status() == 0, fa.last_error()
    ref = oracle.attention_backward(f64(q), f64(k), f64(v), f64(o), lse.double().numpy(), f64(do),
                                    case.softmax_scale, case.causal)
    bq, bk, bv = bounds(f64(q), f64(k), f64(v), f64(o), lse.double().numpy(), f64(do),
                        case.softmax_scale, case.causal)
    for got, want, bnd, name in ((dq, ref[0], bq, "dQ"), (dk, ref[1], bk, "dK"),
                                 (dv, ref[2], bv, "dV")):
        err = np.abs(f64(got.cpu()) - want)
        worst = float((err / (U * bnd + 1e-6)).max())
        assert worst <= 1.0, (case.name, name, worst, float(err.max()))


SMALL = [
    PrefillCase("bwd_tile", 1, 2, 1, 128, 128, 64, seed=90),
    PrefillCase("bwd_ragged_causal", 1, 4, 2, 300, 300, 128, seed=91, causal=True),
    PrefillCase("bwd_ragged_plain", 2, 2, 2, 200, 520, 64, seed=92),
    PrefillCase("bwd_q_shorter_causal", 1, 4, 1, 100, 513, 128, seed=93, causal=True),
    PrefillCase("bwd_many_tiles", 1, 2, 2, 640, 640, 128, seed=94, causal=True),
    PrefillCase("bwd_seven", 1, 2, 1, 7, 7, 128, seed=95, causal=True),
    PrefillCase("bwd_gqa8", 1, 8, 1, 256, 256, 64, seed=96, causal=True),
]


@pytest.mark.parametrize("case", SMALL, ids=lambda c: c.name)
def test_backward_matches_oracle_within_derived_bounds(cuda_device, case):
    run_case(case)


def test_backward_keys_no_query_sees_get_zero(cuda_device):
    """No queries (Nq = 0): dK = dV = 0 over every key."""
    dev = torch.device("cuda", 0)
    k = torch.randn((1, 1, 200, 64), device=dev).to(torch.bfloat16)
    dk = torch.full_like(k, 7.0)
    dv = torch.full_like(k, 7.0)
    fa.fa_bwd(None, k, k, None, None, None, None, dk, dv, None, 1, 2, 1, 0, 200, 64, 0.125,
              False, stream=torch.cuda.current_stream(dev).cuda_stream)
    torch.cuda.synchronize()
    assert torch.all(dk == 0) and torch.all(dv == 0)


def test_full_size_sampled_dq_rows_and_the_dv_sum(cuda_device):
    """B1 Hq32 Hkv8 N8192 D128 causal, as the forward benchmark's workload.

    The oracle cannot run the whole forward here, so o and lse come from the
    library's forward, except at 64 sampled rows, which get the oracle's o and
    lse; dQ of a row depends only on that row's o, lse and dO (and all of K, V),
    so those rows of dQ are compared with the oracle.  dV is checked through an
    identity that holds for any o: the rows of P sum to 1, so
    sum_j dV_j = sum over the group's heads and queries of dO_i."""
    case = PREFILL_CASES["gqa_b1_hq32_hkv8_n8192_d128_causal"]
    q, k, v, gen = make_prefill(case)
    do = make_dout(case, gen)
    rows = sample_rows(case, gen, 2)
    dev = torch.device("cuda", 0)
    qg, kg, vg, dog = q.to(dev), k.to(dev), v.to(dev), do.to(dev)
    o, lse = fa.attention(qg, kg, vg, case.softmax_scale, True)
    O_r, L_r = oracle.attention_rows(f64(q), f64(k), f64(v), case.softmax_scale, True, rows)
    for n, (b, h, i) in enumerate(rows):
        o[b, h, i] = torch.from_numpy(O_r[n]).to(torch.bfloat16).to(dev)
        lse[b, h, i] = float(np.float32(L_r[n]))
    dq, dk, dv = fa.attention_backward(qg, kg, vg, o, lse, dog, case.softmax_scale, True)
    torch.cuda.synchronize()
    assert fa.device_status() == 0, fa.last_error()
    G = case.Hq // case.Hkv
    scale = case.softmax_scale
    for n, (b, h, i) in enumerate(rows):
        g = h // G
        n_vis = i + 1
        kk = f64(k[b, g, :n_vis])
        vv = f64(v[b, g, :n_vis])
        qi = f64(q[b, h, i])
        oi = f64(o[b, h, i].cpu())
        doi = f64(do[b, h, i])
        li = float(lse[b, h, i].cpu())
        # one row of the oracle backward: the row as a 1-query problem over its visible keys
        ref = oracle.attention_backward(qi[None, None, None], kk[None, None], vv[None, None],
                                        oi[None, None, None], np.array([[[li]]]),
                                        doi[None, None, None], scale, False)
        P = np.exp(scale * kk @ qi - li)
        dS = np.abs(P * (vv @ doi - doi @ oi))
        bnd = scale * dS @ np.abs(kk)
        err = np.abs(f64(dq[b, h, i].cpu()) - ref[0][0, 0, 0])
        assert np.all(err <= U * bnd + 1e-6), (b, h, i, float(err.max()))
    lhs = dv.float().sum(dim=2).double().cpu().numpy()              # [B, Hkv, D]
    rhs = do.float().double().numpy().reshape(case.B, case.Hkv, G, case.Nq, case.D).sum((2, 3))
    mag = np.abs(do.float().double().numpy()).reshape(case.B, case.Hkv, G, case.Nq,
                                                      case.D).sum((2, 3))
    assert np.all(np.abs(lhs - rhs) <= U * mag + 1e-3)
