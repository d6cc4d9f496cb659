"""Parity of fa_fwd_paged (through the C ABI) with the fp64 paged-prefill oracle."""
import numpy as np
import pytest
import torch

import oracle
from exact_tiled_attention_40_b200 import fa
from exact_tiled_attention_40_b200.inputs import PagedPrefillCase, make_paged_prefill

pytestmark = pytest.mark.gpu
TOL_O = 2e-2
TOL_LSE = 1e-3


def f64(t):
    return t.float().double().numpy()


def run(case, q, kc, vc, table, cu_q, lens):
    dev = torch.device("cuda", 0)
    max_q = int((cu_q[1:] - cu_q[:-1]).max())
    o, lse = fa.prefill_paged(q.to(dev), kc.to(dev), vc.to(dev), table.to(dev), cu_q.to(dev),
                              lens.to(dev), max(max_q, 1), case.softmax_scale, case.causal)
    torch.cuda.synchronize()
    return o.cpu(), lse.cpu()


def check(case):
    q, kc, vc, table, cu_q, lens = make_paged_prefill(case)
    o, lse = run(case, q, kc, vc, table, cu_q, lens)
    assert fa.device_status() == 0, fa.last_error()
    O_ref, L_ref = oracle.paged_prefill(f64(q), kc.float().numpy(), vc.float().numpy(),
                                        table.numpy(), cu_q.numpy(), lens.numpy(),
                                        case.softmax_scale, case.causal, case.page_size)
    dO = np.abs(f64(o) - O_ref).max() if O_ref.size else 0.0
    live = np.isfinite(L_ref)
    dL = np.abs(lse.double().numpy()[live] - L_ref[live]).max() if live.any() else 0.0
    assert dO <= TOL_O and dL <= TOL_LSE, (case.name, dO, dL)


def test_chunked_prefill_causal_gqa(cuda_device):
    # the last Nq_b tokens of each sequence query its cached prefix (partial last pages)
    check(PagedPrefillCase("chunk", 4, 8, 2, 128, True, seed=110, num_pages=400,
                           nq=(128, 1, 300, 37), nk=(700, 5, 300, 1000)))


def test_full_prompt_non_causal(cuda_device):
    check(PagedPrefillCase("full", 3, 4, 4, 128, False, seed=111, num_pages=200,
                           nq=(50, 260, 3), nk=(50, 260, 1100)))


def test_more_sequences_than_the_sorted_list_holds(cuda_device):
    """1100 sequences (past the 1024 the kernel sorts) of up to 100 cached
    keys, each querying all of them."""
    check(PagedPrefillCase("many", 1100, 4, 2, 128, True, seed=114, num_pages=8000, lo=1,
                           hi=100))


def test_head_dim_64(cuda_device):
    check(PagedPrefillCase("d64", 5, 8, 2, 64, True, seed=112, num_pages=500, lo=1, hi=900))


def test_out_of_range_page_is_reported(cuda_device):
    case = PagedPrefillCase("badpage", 2, 4, 2, 128, True, seed=113, num_pages=100,
                            nq=(20, 30), nk=(60, 90))
    q, kc, vc, table, cu_q, lens = make_paged_prefill(case)
    table[1, 2] = case.num_pages + 7
    run(case, q, kc, vc, table, cu_q, lens)
    assert fa.device_status() == 5          # FA_ERR_DEVICE_INDEX
