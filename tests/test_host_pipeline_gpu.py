"""fa_fwd_host (inputs and outputs in host memory, copies overlapped with the
forward chunk by chunk) gives exactly fa_fwd's result: the same kernel runs on
each chunk's slice, so O and LSE must match bit for bit; the shapes cover the
chunk plans (groups of one sequence, several sequences per chunk, a ragged
last chunk, no keys).
"""

import pytest
import torch

from exact_tiled_attention_40_b200 import fa
from exact_tiled_attention_40_b200.inputs import PrefillCase, make_prefill

pytestmark = pytest.mark.gpu

CASES = [
    PrefillCase("host_groups", 1, 32, 8, 1024, 1024, 128, seed=100, causal=True),
    PrefillCase("host_three_seqs", 3, 8, 8, 300, 300, 64, seed=101),
    PrefillCase("host_many_seqs", 11, 4, 2, 260, 400, 128, seed=102, causal=True),
    PrefillCase("host_two_groups", 1, 4, 2, 333, 333, 64, seed=103, causal=True),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: c.name)
def test_host_pipeline_equals_the_device_forward(cuda_device, case):
    q, k, v, _ = make_prefill(case)
    o_ref, l_ref = fa.attention(q.to(cuda_device), k.to(cuda_device), v.to(cuda_device),
                                case.softmax_scale, case.causal)
    o, l = fa.attention_from_host(q.pin_memory(), k.pin_memory(), v.pin_memory(),
                                  case.softmax_scale, case.causal, device=cuda_device)
    torch.cuda.synchronize()
    assert fa.device_status() == 0, fa.last_error()
    assert torch.equal(o, o_ref.cpu())
    assert torch.equal(l, l_ref.cpu())
