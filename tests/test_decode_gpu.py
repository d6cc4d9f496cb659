"""Parity of fa_decode_paged (through the C ABI) with the fp64 paged-decode oracle."""
import numpy as np
import pytest
import torch

import oracle
from exact_tiled_attention_40_b200 import fa
from exact_tiled_attention_40_b200.inputs import DECODE_CASES, DecodeCase, make_decode

pytestmark = pytest.mark.gpu
TOL_O = 2e-2
TOL_LSE = 1e-3


def f64(t):
    return t.float().double().numpy()


def run(case, q, kc, vc, table, lens):
    dev = torch.device("cuda", 0)
    o, lse = fa.decode_paged(q.to(dev), kc.to(dev), vc.to(dev), table.to(dev), lens.to(dev),
                             case.softmax_scale)
    torch.cuda.synchronize()
    return o.cpu(), lse.cpu()


def check(case, q, kc, vc, table, lens):
    o, lse = run(case, q, kc, vc, table, lens)
    assert fa.device_status() == 0, fa.last_error()
    O_ref, L_ref = oracle.decode_paged(f64(q), kc.float().numpy(), vc.float().numpy(),
                                       table.numpy(), lens.numpy(), case.softmax_scale,
                                       case.page_size)
    live = lens.numpy() > 0
    dO = np.abs(f64(o) - O_ref).max()
    dL = np.abs(lse.double().numpy()[live] - L_ref[live]).max() if live.any() else 0.0
    assert dO <= TOL_O and dL <= TOL_LSE, (case.name, dO, dL)
    assert np.all(lse.numpy()[~live] == -np.inf)


@pytest.mark.parametrize("Hq,Hkv", [(8, 2), (4, 4), (8, 4), (16, 2), (32, 16)])
def test_small_decode_matches_oracle(cuda_device, Hq, Hkv):
    case = DecodeCase("small", 5, Hq, Hkv, 128, 16, 1, 700, 300, seed=40 + Hq + Hkv)
    q, kc, vc, table, lens = make_decode(case)
    lens[0] = 1        # single token
    lens[1] = 16       # exactly one page
    lens[2] = 17       # one page plus one token
    check(case, q, kc, vc, table, lens)


def test_fewer_cache_chunks_than_sms(cuda_device):
    """Short sequences: far fewer 8-token chunks than SMs, so most persistent
    CTAs get an empty share and the merge must skip them."""
    case = DecodeCase("short", 6, 16, 4, 128, 16, 1, 20, 40, seed=52)
    check(case, *make_decode(case))


def test_many_sequences_offsets_in_global_memory(cuda_device):
    """5000 short sequences: more than the 4096 whose half-page offsets the
    stream kernel's producer keeps in shared memory, so it searches them in
    global memory, and the merge runs 5000 blocks."""
    case = DecodeCase("many", 5000, 8, 2, 128, 16, 1, 40, 16000, seed=53)
    check(case, *make_decode(case))


def test_zero_length_sequence(cuda_device):
    case = DecodeCase("zero", 3, 8, 2, 128, 16, 5, 40, 20, seed=50)
    q, kc, vc, table, lens = make_decode(case)
    lens[1] = 0
    o, _ = run(case, q, kc, vc, table, lens)
    assert torch.all(o[1] == 0)
    check(case, q, kc, vc, table, lens)


def test_decode_workload_b64(cuda_device):
    check(DECODE_CASES["decode_b64_hq32_hkv8_d128_page16"],
          *make_decode(DECODE_CASES["decode_b64_hq32_hkv8_d128_page16"]))


def test_out_of_range_page_is_reported_not_read(cuda_device):
    """An entry past the pool is skipped by the kernel's own bounds check and
    reported through the device error word."""
    case = DecodeCase("badpage", 2, 8, 2, 128, 16, 40, 60, 20, seed=51)
    q, kc, vc, table, lens = make_decode(case)
    table[0, 1] = case.num_pages + 5
    run(case, q, kc, vc, table, lens)
    assert fa.device_status() == 5          # FA_ERR_DEVICE_INDEX
    assert fa.device_status() == 0          # the word is cleared by the read
