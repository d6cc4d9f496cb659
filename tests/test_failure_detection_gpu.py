"""Failure detection without a GPU fault: a bounded in-kernel wait that nothing
satisfies gives up after its limit, the host reads FA_ERR_DEVICE_TIMEOUT from
fa_device_status(), and the context stays usable (a forward right after it
still matches the oracle).  Out-of-range indices read from device memory are
covered by tests/test_decode_gpu.py and tests/test_varlen_gpu.py.
"""

import numpy as np
import pytest
import torch

import oracle
from exact_tiled_attention_40_b200 import fa
from exact_tiled_attention_40_b200.inputs import PrefillCase, make_prefill

pytestmark = pytest.mark.gpu


def test_a_wait_that_runs_out_is_reported_and_the_context_survives(cuda_device):
    assert fa.device_status() == 0, fa.last_error()
    status, gave_up = fa.selftest_wait_timeout(20000, cuda_device)
    assert gave_up
    assert status == 4, (status, fa.last_error())          # FA_ERR_DEVICE_TIMEOUT
    assert fa.device_status() == 0                           # the word was cleared
    case = PrefillCase("after_timeout", 1, 2, 1, 200, 200, 64, seed=110, causal=True)
    q, k, v, _ = make_prefill(case)
    o, lse = fa.attention(q.to(cuda_device), k.to(cuda_device), v.to(cuda_device),
                          case.softmax_scale, True)
    torch.cuda.synchronize()
    O_ref, L_ref = oracle.attention(q.float().double().numpy(), k.float().double().numpy(),
                                    v.float().double().numpy(), case.softmax_scale, True)
    assert np.abs(o.cpu().float().double().numpy() - O_ref).max() <= 2e-2
    assert np.abs(lse.cpu().double().numpy() - L_ref).max() <= 1e-3
    assert fa.device_status() == 0
