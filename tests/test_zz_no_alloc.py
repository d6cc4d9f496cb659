"""fa_decode_paged_noalloc: paged decode for callers that cannot allocate device
memory while decoding (for example a serving engine that reserved nearly all
device memory for weights and the KV-cache pool up front, or a runtime that
forbids allocations after start-up).  Its chunk partials live in a fixed
scratch array inside the library instead of a per-call workspace.

The GPU test calls it through the C ABI on several problems in a row, each
chosen to take one of the ways the plan is fitted to the array, and checks
every result against fa_decode_paged (the allocating entry point) and against
the fp64 oracle, within the decode tests' tolerances.  This file is collected
last on purpose.
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from exact_tiled_attention_40_b200 import fa
from exact_tiled_attention_40_b200.inputs import DECODE_CASES, DecodeCase, make_decode

TOL_O = 2e-2
TOL_LSE = 1e-3
FAKE = 0x10000


def test_oversized_problem_is_rejected_before_touching_the_device():
    lib = fa.lib()
    # B * Hq = 40,000 partial rows of 516 bytes exceed 16 MiB even with one chunk
    # per sequence, so no schedule fits the fixed scratch.
    rc = lib.fa_decode_paged_noalloc(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1250, 32, 8, 128, 16,
                                     0.1, None, 4, 100, None)
    assert rc == 1                                         # FA_ERR_INVALID_ARG
    msg = lib.fa_last_error_string().decode()
    assert "scratch" in msg and "16777216" in msg


def _inputs(case, dev, table_width=None, edit=None):
    """The case's inputs on `dev`; `table_width` pads the block table with unused
    zero entries (a wider table means a larger max_pages_per_seq for the same
    lengths)."""
    q, kc, vc, table, lens = make_decode(case)
    if edit:
        edit(lens)
    if table_width:
        table = F.pad(table, (0, table_width - table.shape[1])).contiguous()
    return tuple(t.to(dev) for t in (q, kc, vc, table, lens))


def _short_first(lens):
    lens[0] = 1
    lens[1] = 0


# (case, block-table width, edit, how the plan fits the 16 MiB array), at 148 SMs:
CASES = [
    # persistent schedule as fa_decode_paged plans it (592 dynamic-unit slots fit in 740)
    (DECODE_CASES["decode_b64_hq32_hkv8_d128_page16"], None, None),
    # persistent schedule that fits as fa_decode_paged plans it, short sequences first
    (DecodeCase("noalloc_small", 5, 16, 2, 128, 16, 1, 900, 400, seed=70), None, _short_first),
    # persistent schedule with the slots trimmed to one dynamic unit per CTA (cap 167)
    (DecodeCase("noalloc_b350", 350, 32, 8, 128, 16, 1, 300, 7200, seed=71), 512, None),
    # (148 + 900) * 32 rows do not fit: direct schedule instead, one chunk per sequence
    (DecodeCase("noalloc_b900", 900, 32, 8, 128, 16, 1, 64, 4000, seed=72), None, None),
    # Hkv = 16, direct schedule: 32-page chunks would need 65,536 rows (32,513 fit);
    # widened to 128-page chunks, 16,384 rows
    (DecodeCase("noalloc_hkv16", 128, 32, 16, 128, 16, 1, 600, 5200, seed=73), 512, None),
]


@pytest.mark.gpu
def test_calls_in_a_row_match_the_allocating_entry_point_and_the_oracle(cuda_device):
    dev = cuda_device
    inputs = [_inputs(case, dev, width, edit) for case, width, edit in CASES]
    refs = []
    for (case, _, _), (q, kc, vc, table, lens) in zip(CASES, inputs):
        refs.append(fa.decode_paged(q, kc, vc, table, lens, case.softmax_scale))
    torch.cuda.synchronize()
    assert fa.device_status() == 0, fa.last_error()

    for call, ((case, _, _), (q, kc, vc, table, lens)) in enumerate(zip(CASES, inputs)):
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
        live = lens > 0
        assert torch.all(lse[~live] == float("-inf"))
        assert torch.isfinite(o.float()).all()

        o_ref, lse_ref = refs[call]
        dO = (o.float() - o_ref.float()).abs().max().item()
        dL = (lse[live] - lse_ref[live]).abs().max().item()
        assert dO <= TOL_O and dL <= TOL_LSE, (case.name, "vs fa_decode_paged", dO, dL)

        O_or, L_or = oracle.decode_paged(q.cpu().double().numpy(), kc.cpu().float().numpy(),
                                         vc.cpu().float().numpy(), table.cpu().numpy(),
                                         lens.cpu().numpy(), case.softmax_scale, 16)
        dO = float(np.abs(o.cpu().double().numpy() - O_or).max())
        lv = live.cpu().numpy()
        dL = float(np.abs(lse.cpu().double().numpy()[lv] - L_or[lv]).max())
        assert dO <= TOL_O and dL <= TOL_LSE, (case.name, "vs oracle", dO, dL)
