"""Out-of-bounds detection without a sanitizer: every tensor a call reads or writes
sits in the middle of a larger allocation whose margins hold a canary pattern
(NaN for inputs, so a stray read shows up in the results; a fixed bit pattern
for outputs, so a stray write shows up in the margins).  After the call the
margins must be untouched and the results must still match the oracle.
"""

import numpy as np
import pytest
import torch

import oracle
from exact_tiled_attention_40_b200 import fa
from exact_tiled_attention_40_b200.inputs import (DecodeCase, PrefillCase, VarlenCase,
                                                  make_decode, make_dout, make_prefill,
                                                  make_varlen)

pytestmark = pytest.mark.gpu

PAD_BYTES = 8192          # margin on each side (a multiple of 16: alignment is kept)


class Guarded:
    """A tensor of `shape` inside an allocation with PAD_BYTES of canary on each side."""

    def __init__(self, shape, dtype, dev, canary_bits, init=None):
        item = torch.empty((), dtype=dtype).element_size()
        self.pad = PAD_BYTES // item
        n = int(np.prod(shape)) if len(shape) else 1
        self.n = n
        ibits = {1: torch.uint8, 2: torch.int16, 4: torch.int32}[item]
        self.full = torch.empty(n + 2 * self.pad, dtype=dtype, device=dev)
        self.full.view(ibits).fill_(canary_bits)
        self.bits = ibits
        self.canary = canary_bits
        self.t = self.full[self.pad:self.pad + n].view(shape)
        if init is not None:
            self.t.copy_(init)

    def margins_intact(self):
        b = self.full.view(self.bits)
        head, tail = b[:self.pad], b[self.pad + self.n:]
        return bool(torch.all(head == self.canary)) and bool(torch.all(tail == self.canary))


BF16_NAN = 0x7FC1                # a bf16 NaN, as int16 bits
OUT_BITS16 = 0x5A5A
OUT_BITS32 = 0x5A5A5A5A


def f64(t):
    return t.float().double().cpu().numpy()


FP16_NAN = 0x7E01                # an fp16 NaN, as int16 bits


@pytest.mark.parametrize("case", [
    # rows past Nq = 300 in the last query tile: the O tensor map clips them; LSE rows
    # leave by bulk copies (Nq % 4 == 0)
    PrefillCase("canary_fwd", 2, 4, 2, 300, 300, 128, seed=120, causal=True),
    # fp16, D = 64, Nq = 77 (not a multiple of 4: LSE by plain stores), more keys than queries
    PrefillCase("canary_fwd_fp16", 2, 2, 1, 77, 390, 64, "fp16", seed=122),
], ids=lambda c: c.name)
def test_forward_touches_nothing_outside_its_tensors(cuda_device, case):
    q, k, v, _ = make_prefill(case)
    dev = cuda_device
    dt, nan = (torch.bfloat16, BF16_NAN) if case.dtype == "bf16" else (torch.float16, FP16_NAN)
    gq = Guarded(q.shape, dt, dev, nan, q)
    gk = Guarded(k.shape, dt, dev, nan, k)
    gv = Guarded(v.shape, dt, dev, nan, v)
    go = Guarded(q.shape, dt, dev, OUT_BITS16)
    gl = Guarded((case.B, case.Hq, case.Nq), torch.float32, dev, OUT_BITS32)
    fa.fa_fwd(gq.t, gk.t, gv.t, go.t, gl.t, case.B, case.Hq, case.Hkv, case.Nq, case.Nk, case.D,
              case.softmax_scale, case.causal)
    torch.cuda.synchronize()
    assert fa.device_status() == 0, fa.last_error()
    assert go.margins_intact() and gl.margins_intact()
    O, L = oracle.attention(f64(q), f64(k), f64(v), case.softmax_scale, case.causal)
    assert np.abs(f64(go.t) - O).max() <= 2e-2
    assert np.abs(f64(gl.t) - L).max() <= 1e-3


def test_ragged_forward_touches_nothing_outside_its_tensors(cuda_device):
    case = VarlenCase("canary_varlen", 5, 4, 2, 128, "bf16", True, 121, lo=20, hi=400)
    q, k, v, cu_q, cu_k = make_varlen(case)
    dev = cuda_device
    gq = Guarded(q.shape, torch.bfloat16, dev, BF16_NAN, q)
    gk = Guarded(k.shape, torch.bfloat16, dev, BF16_NAN, k)
    gv = Guarded(v.shape, torch.bfloat16, dev, BF16_NAN, v)
    go = Guarded(q.shape, torch.bfloat16, dev, OUT_BITS16)
    gl = Guarded((case.Hq, q.shape[0]), torch.float32, dev, OUT_BITS32)
    cq, ck = cu_q.to(dev), cu_k.to(dev)
    max_q = int((cu_q[1:] - cu_q[:-1]).max())
    max_k = int((cu_k[1:] - cu_k[:-1]).max())
    fa.fa_fwd_varlen(gq.t, gk.t, gv.t, go.t, gl.t, cq, ck, case.B, case.Hq, case.Hkv, max_q, max_k,
                     q.shape[0], k.shape[0], case.D, case.softmax_scale, True)
    torch.cuda.synchronize()
    assert fa.device_status() == 0, fa.last_error()
    assert go.margins_intact() and gl.margins_intact()
    O, L = oracle.varlen_attention(f64(q), f64(k), f64(v), cu_q.numpy(), cu_k.numpy(),
                                   case.softmax_scale, True)
    assert np.abs(f64(go.t) - O).max() <= 2e-2
    assert np.abs(f64(gl.t) - L).max() <= 1e-3


def test_decode_touches_nothing_outside_its_tensors(cuda_device):
    case = DecodeCase("canary_decode", 5, 8, 2, 128, 16, 1, 300, 200, seed=122)
    q, kc, vc, table, lens = make_decode(case)
    dev = cuda_device
    gq = Guarded(q.shape, torch.bfloat16, dev, BF16_NAN, q)
    go = Guarded(q.shape, torch.bfloat16, dev, OUT_BITS16)
    gl = Guarded((case.B, case.Hq), torch.float32, dev, OUT_BITS32)
    fa.fa_decode_paged(gq.t, kc.to(dev), vc.to(dev), table.to(dev), lens.to(dev), go.t, case.B,
                       case.Hq, case.Hkv, case.D, case.page_size, case.softmax_scale,
                       table.shape[1], case.num_pages, gl.t)
    torch.cuda.synchronize()
    assert fa.device_status() == 0, fa.last_error()
    assert go.margins_intact() and gl.margins_intact()
    O, L = oracle.decode_paged(f64(q), kc.float().numpy(), vc.float().numpy(), table.numpy(),
                               lens.numpy(), case.softmax_scale, 16)
    assert np.abs(f64(go.t) - O).max() <= 2e-2
    assert np.abs(f64(gl.t) - L).max() <= 1e-3


def test_backward_touches_nothing_outside_its_tensors(cuda_device):
    case = PrefillCase("canary_bwd", 1, 4, 2, 300, 300, 64, seed=123, causal=True)
    q, k, v, gen = make_prefill(case)
    do = make_dout(case, gen)
    dev = cuda_device
    o, lse = fa.attention(q.to(dev), k.to(dev), v.to(dev), case.softmax_scale, True)
    gdq = Guarded(q.shape, torch.bfloat16, dev, OUT_BITS16)
    gdk = Guarded(k.shape, torch.bfloat16, dev, OUT_BITS16)
    gdv = Guarded(v.shape, torch.bfloat16, dev, OUT_BITS16)
    gde = Guarded((case.B, case.Hq, case.Nq), torch.float32, dev, OUT_BITS32)
    fa.fa_bwd(q.to(dev), k.to(dev), v.to(dev), o, lse, do.to(dev), gdq.t, gdk.t, gdv.t, gde.t,
              case.B, case.Hq, case.Hkv, case.Nq, case.Nk, case.D, case.softmax_scale, True)
    torch.cuda.synchronize()
    assert fa.device_status() == 0, fa.last_error()
    for g in (gdq, gdk, gdv, gde):
        assert g.margins_intact()
    for g in (gdq, gdk, gdv):
        assert torch.isfinite(g.t.float()).all()
