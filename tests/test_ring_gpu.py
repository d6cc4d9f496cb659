"""The library's merge kernel and the sequence-sharded forward on one B200.

fa_merge_partials is compared with the oracle's LSE merge (fp32 arithmetic:
1e-5); the ring forward with the library's per-chunk forward and merge is run
as one rank (no exchange) and as four ranks one after another on the same
device with their K/V chunks handed in per step (no rank waits for another),
and compared with the fp64 oracle on the whole sequence within the forward's
tolerances (max |dO| <= 2e-2, max |dLSE| <= 1e-3).
"""

import numpy as np
import pytest
import torch

import oracle
from exact_tiled_attention_40_b200 import fa, ring
from exact_tiled_attention_40_b200.inputs import PrefillCase, make_prefill

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("D", [64, 128])
def test_merge_kernel_matches_the_oracle_merge(cuda_device, D):
    g = torch.Generator().manual_seed(80 + D)
    rows = 1000
    o_acc = torch.randn((rows, D), generator=g)
    lse_acc = torch.randn((rows,), generator=g) * 3
    o_part = torch.randn((rows, D), generator=g).to(torch.bfloat16)
    lse_part = torch.randn((rows,), generator=g) * 3
    lse_acc[::7] = -float("inf")
    lse_part[::11] = -float("inf")
    o_acc[::77] = 0.0
    o_part[::77] = 0
    dev = cuda_device
    a, la = o_acc.to(dev), lse_acc.to(dev)
    out = torch.empty((rows, D), dtype=torch.bfloat16, device=dev)
    fa.merge_partials(a, la, o_part.to(dev), lse_part.to(dev), first=False, o_out=out)
    torch.cuda.synchronize()
    O_ref, L_ref = oracle.merge_partials(
        [o_acc.double().numpy(), o_part.double().numpy()],
        [lse_acc.double().numpy(), lse_part.double().numpy()])
    np.testing.assert_allclose(a.cpu().double().numpy(), O_ref, atol=1e-5, rtol=1e-5)
    L = la.cpu().double().numpy()
    assert np.array_equal(np.isneginf(L), np.isneginf(L_ref))
    fin = np.isfinite(L_ref)
    np.testing.assert_allclose(L[fin], L_ref[fin], atol=1e-5)
    ob = out.cpu().double().numpy()
    assert np.all(np.abs(ob - O_ref) <= 2.0 ** -8 * np.abs(O_ref) + 1e-5)
    # first: the accumulator becomes the part
    b, lb = torch.empty_like(a), torch.empty_like(la)
    fa.merge_partials(b, lb, o_part.to(dev), lse_part.to(dev), first=True)
    torch.cuda.synchronize()
    assert torch.equal(b.cpu(), o_part.float())
    assert torch.equal(lb.cpu(), lse_part)


def _check(case, world):
    q, k, v, _ = make_prefill(case)
    dev = torch.device("cuda", 0)
    qg, kg, vg = q.to(dev), k.to(dev), v.to(dev)
    ks = [ring.zigzag_shard(kg, r, world) for r in range(world)]
    vs = [ring.zigzag_shard(vg, r, world) for r in range(world)]
    outs, lses = [], []
    for r in range(world):
        o, lse = ring.ring_attention(
            ring.zigzag_shard(qg, r, world), ks[r], vs[r], case.causal, case.softmax_scale,
            rank=r, world=world, fetch=lambda s, r=r: (ks[(r - s) % world], vs[(r - s) % world]))
        outs.append(o)
        lses.append(lse)
    torch.cuda.synchronize()
    assert fa.device_status() == 0, fa.last_error()
    O = ring.zigzag_unshard(outs).cpu().float().double().numpy()
    L = ring.zigzag_unshard(lses, dim=-1).cpu().double().numpy()
    O_ref, L_ref = oracle.attention(q.float().double().numpy(), k.float().double().numpy(),
                                    v.float().double().numpy(), case.softmax_scale, case.causal)
    assert np.abs(O - O_ref).max() <= 2e-2
    assert np.abs(L - L_ref).max() <= 1e-3


@pytest.mark.parametrize("world", [1, 4])
@pytest.mark.parametrize("causal", [True, False])
def test_sequence_sharded_forward_matches_the_oracle(cuda_device, world, causal):
    case = PrefillCase("ring", 1, 4, 2, 1024, 1024, 128, seed=81, causal=causal)
    _check(case, world)


def test_sequence_sharded_forward_with_short_chunks(cuda_device):
    """Chunks of 40 rows: every chunk pair is a ragged single tile."""
    _check(PrefillCase("ring_short", 2, 2, 1, 320, 320, 64, seed=82, causal=True), 4)
