"""fa_decode_paged_noalloc: paged decode for callers that cannot allocate device
memory while decoding (for example a serving engine that reserved nearly all
device memory for weights and the KV-cache pool up front, or a runtime that
forbids allocations after start-up).  Its chunk partials live in a fixed
scratch array inside the library instead of a per-call workspace.

The GPU test calls it through the C ABI twice in a row, on different inputs,
and checks each result against fa_decode_paged (the allocating entry point)
within the decode tests' tolerances.  This file is collected last on purpose.
"""
import numpy as np
import pytest
import torch

from exact_tiled_attention_40_b200 import fa
from exact_tiled_attention_40_b200.inputs import DECODE_CASES, DecodeCase, make_decode

TOL_O = 2e-2
TOL_LSE = 1e-3
FAKE = 0x10000


def test_oversized_problem_is_rejected_before_touching_the_device():
    lib = fa.lib()
    # (148 + B) * Hq = 44,736 > 32,513 rows: the partials cannot fit the fixed scratch.
    rc = lib.fa_decode_paged_noalloc(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1250, 32, 8, 128, 16,
                                     0.1, None, 4, 100, None)
    assert rc == 1                                         # FA_ERR_INVALID_ARG
    msg = lib.fa_last_error_string().decode()
    assert "scratch" in msg and "16777216" in msg


def _inputs(case, dev, edit=None):
    q, kc, vc, table, lens = make_decode(case)
    if edit:
        edit(lens)
    return tuple(t.to(dev) for t in (q, kc, vc, table, lens))


@pytest.mark.gpu
def test_two_calls_match_the_allocating_entry_point(cuda_device):
    dev = cuda_device
    big = DECODE_CASES["decode_b64_hq32_hkv8_d128_page16"]        # chunking widened to fit
    small = DecodeCase("noalloc_small", 5, 16, 2, 128, 16, 1, 900, 400, seed=70)

    def short_first(lens):
        lens[0] = 1
        lens[1] = 0

    cases = [(big, _inputs(big, dev)), (small, _inputs(small, dev, short_first))]
    refs = []
    for case, (q, kc, vc, table, lens) in cases:
        refs.append(fa.decode_paged(q, kc, vc, table, lens, case.softmax_scale))
    torch.cuda.synchronize()
    assert fa.device_status() == 0, fa.last_error()

    for call, (case, (q, kc, vc, table, lens)) in enumerate(cases):
        o = torch.full_like(q, float("nan"))
        lse = torch.full((case.B, case.Hq), float("nan"), dtype=torch.float32, device=dev)
        torch.cuda.synchronize()
        free_before = torch.cuda.mem_get_info(dev)[0]
        fa.decode_paged_noalloc(q, kc, vc, table, lens, o, lse, case.softmax_scale)
        torch.cuda.synchronize()
        free_after = torch.cuda.mem_get_info(dev)[0]
        assert fa.device_status() == 0, fa.last_error()
        if call > 0:                   # after the first call's one-time set-up
            assert free_after == free_before
        o_ref, lse_ref = refs[call]
        dO = (o.float() - o_ref.float()).abs().max().item()
        live = lens > 0
        dL = (lse[live] - lse_ref[live]).abs().max().item()
        assert dO <= TOL_O and dL <= TOL_LSE, (case.name, dO, dL)
        assert torch.all(lse[~live] == float("-inf"))
        assert torch.isfinite(o.float()).all()
