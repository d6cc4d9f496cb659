"""Every entry point whose LSE output may be NULL (include/fa.h) run without it:
O must be bit-identical to the same call that also writes LSE, and the device
error word must stay clear.  The O arithmetic does not depend on whether LSE
leaves the kernel, so any difference would be a write through the missing
pointer or a changed code path."""
import pytest
import torch

from exact_tiled_attention_40_b200 import fa
from exact_tiled_attention_40_b200.inputs import (DecodeCase, PagedPrefillCase, PrefillCase,
                                                  VarlenCase, make_decode, make_paged_prefill,
                                                  make_prefill, make_varlen)

pytestmark = pytest.mark.gpu


def same_o(with_lse, without_lse):
    o1, l1 = with_lse
    o2, l2 = without_lse
    torch.cuda.synchronize()
    assert fa.device_status() == 0, fa.last_error()
    assert l1 is not None and l2 is None
    assert torch.equal(o1, o2)


@pytest.mark.parametrize("case", [
    PrefillCase("nolse_bulk", 1, 4, 2, 256, 256, 128, seed=130, causal=True),   # LSE by bulk copy
    PrefillCase("nolse_rows", 1, 2, 1, 201, 333, 128, seed=131),                # per-row LSE stores
    PrefillCase("nolse_fp16", 2, 2, 2, 130, 130, 64, "fp16", seed=132, causal=True),
], ids=lambda c: c.name)
def test_dense_forward(cuda_device, case):
    q, k, v, _ = make_prefill(case)
    dev = torch.device("cuda", 0)
    q, k, v = q.to(dev), k.to(dev), v.to(dev)
    same_o(fa.attention(q, k, v, case.softmax_scale, case.causal),
           fa.attention(q, k, v, case.softmax_scale, case.causal, return_lse=False))


def test_ragged_forward(cuda_device):
    case = VarlenCase("nolse_varlen", 4, 4, 2, 128, "bf16", True, seed=133, lo=1, hi=400)
    q, k, v, cu_q, cu_k = make_varlen(case)
    dev = torch.device("cuda", 0)
    q, k, v, cu_q, cu_k = (t.to(dev) for t in (q, k, v, cu_q, cu_k))
    mq = int((cu_q[1:] - cu_q[:-1]).max())
    mk = int((cu_k[1:] - cu_k[:-1]).max())
    same_o(fa.attention_varlen(q, k, v, cu_q, cu_k, mq, mk, case.softmax_scale, True),
           fa.attention_varlen(q, k, v, cu_q, cu_k, mq, mk, case.softmax_scale, True,
                               return_lse=False))


def test_paged_prefill(cuda_device):
    case = PagedPrefillCase("nolse_paged", 3, 4, 2, 128, True, seed=134, num_pages=200, lo=1,
                            hi=700)
    q, kc, vc, table, cu_q, lens = make_paged_prefill(case)
    dev = torch.device("cuda", 0)
    q, kc, vc, table, cu_q, lens = (t.to(dev) for t in (q, kc, vc, table, cu_q, lens))
    mq = int((cu_q[1:] - cu_q[:-1]).max())
    same_o(fa.prefill_paged(q, kc, vc, table, cu_q, lens, mq, case.softmax_scale, True),
           fa.prefill_paged(q, kc, vc, table, cu_q, lens, mq, case.softmax_scale, True,
                            return_lse=False))


def test_fp8_forward(cuda_device):
    case = PrefillCase("nolse_fp8", 1, 4, 2, 300, 300, 128, seed=135, causal=True)
    q, k, v, _ = make_prefill(case)
    dev = torch.device("cuda", 0)
    q, k, v = q.to(dev), k.to(dev), v.to(dev)
    same_o(fa.attention_fp8(q, k, v, case.softmax_scale, True),
           fa.attention_fp8(q, k, v, case.softmax_scale, True, return_lse=False))


@pytest.mark.parametrize("Hq,Hkv", [(8, 2), (32, 16)], ids=["streamed", "direct"])
def test_decode(cuda_device, Hq, Hkv):
    case = DecodeCase("nolse_decode", 6, Hq, Hkv, 128, 16, 1, 900, 400, seed=136)
    q, kc, vc, table, lens = (t.to(torch.device("cuda", 0)) for t in make_decode(case))
    same_o(fa.decode_paged(q, kc, vc, table, lens, case.softmax_scale),
           fa.decode_paged(q, kc, vc, table, lens, case.softmax_scale, return_lse=False))
