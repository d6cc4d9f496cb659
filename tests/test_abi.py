"""The C-ABI library loads, exports every declared entry point, and validates
arguments on the host (no GPU needed: nothing here launches a kernel)."""
import ctypes

import pytest
import torch

from exact_tiled_attention_40_b200 import fa

E = {v: k for k, v in fa.STATUS.items()}
FAKE = 0x10000   # 16-byte aligned fake device address; validation never dereferences it


@pytest.fixture(scope="module")
def lib():
    return fa.lib()


def test_every_header_symbol_is_exported(lib):
    names = fa.header_symbols()
    assert set(names) >= {"fa_fwd", "fa_fwd_fp16", "fa_decode_paged", "fa_last_error_string",
                          "fa_device_status", "fa_release", "fa_version"}
    for n in names:
        assert hasattr(lib, n), n
    assert lib.fa_version() >= 100


def fwd(lib, B=1, Hq=2, Hkv=1, Nq=8, Nk=8, D=64, scale=0.125, causal=0, q=FAKE, o=FAKE,
        k=FAKE, v=FAKE):
    return lib.fa_fwd(q, k, v, o, None, B, Hq, Hkv, Nq, Nk, D, scale, causal, None)


@pytest.mark.parametrize("kw,code", [
    (dict(B=-1), "FA_ERR_INVALID_ARG"),
    (dict(D=96), "FA_ERR_UNSUPPORTED"),
    (dict(Hq=3, Hkv=2), "FA_ERR_INVALID_ARG"),
    (dict(Hkv=0), "FA_ERR_INVALID_ARG"),
    (dict(causal=1, Nq=9, Nk=8), "FA_ERR_INVALID_ARG"),
    (dict(scale=0.0), "FA_ERR_INVALID_ARG"),
    (dict(scale=float("nan")), "FA_ERR_INVALID_ARG"),
    (dict(scale=-1.0), "FA_ERR_INVALID_ARG"),
    (dict(q=0), "FA_ERR_INVALID_ARG"),
    (dict(k=0), "FA_ERR_INVALID_ARG"),
    (dict(o=FAKE + 8), "FA_ERR_INVALID_ARG"),
])
def test_fwd_rejects_bad_arguments_on_the_host(lib, kw, code):
    assert fwd(lib, **kw) == E[code]
    assert lib.fa_last_error_string().decode() != ""


def test_fwd_empty_problem_is_a_noop(lib):
    assert fwd(lib, B=0) == 0
    assert fwd(lib, Nq=0) == 0
    assert fwd(lib, Hq=0) == 0


def dec(lib, B=2, Hq=8, Hkv=2, D=128, page=16, scale=0.1, maxp=4, npages=10, ptr=FAKE):
    return lib.fa_decode_paged(ptr, ptr, ptr, ptr, ptr, ptr, B, Hq, Hkv, D, page, scale, None,
                               maxp, npages, None)


@pytest.mark.parametrize("kw,code", [
    (dict(D=64), "FA_ERR_UNSUPPORTED"),
    (dict(page=32), "FA_ERR_UNSUPPORTED"),
    (dict(Hq=32, Hkv=1), "FA_ERR_UNSUPPORTED"),
    (dict(Hq=6, Hkv=4), "FA_ERR_INVALID_ARG"),
    (dict(maxp=0), "FA_ERR_INVALID_ARG"),
    (dict(npages=-1), "FA_ERR_INVALID_ARG"),
    (dict(ptr=0), "FA_ERR_INVALID_ARG"),
    (dict(ptr=FAKE + 4), "FA_ERR_INVALID_ARG"),
    (dict(scale=0.0), "FA_ERR_INVALID_ARG"),
])
def test_decode_rejects_bad_arguments_on_the_host(lib, kw, code):
    assert dec(lib, **kw) == E[code]


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device path")
def test_valid_call_without_a_device_fails_loudly(lib):
    assert fwd(lib) == E["FA_ERR_NO_DEVICE"]
    assert dec(lib) == E["FA_ERR_NO_DEVICE"]
    with pytest.raises(fa.FAError):
        fa._check(fwd(lib), "fa_fwd")


def varlen(lib, B=2, Hq=4, Hkv=2, max_q=9, max_k=9, tq=12, tk=14, D=128, scale=0.1, causal=0,
           q=FAKE, k=FAKE, v=FAKE, o=FAKE, cuq=FAKE, cuk=FAKE):
    return lib.fa_fwd_varlen(q, k, v, o, None, cuq, cuk, B, Hq, Hkv, max_q, max_k, tq, tk, D,
                             scale, causal, None)


@pytest.mark.parametrize("kw,code", [
    (dict(B=-1), "FA_ERR_INVALID_ARG"),
    (dict(tq=-3), "FA_ERR_INVALID_ARG"),
    (dict(D=80), "FA_ERR_UNSUPPORTED"),
    (dict(Hq=5), "FA_ERR_INVALID_ARG"),
    (dict(cuq=None), "FA_ERR_INVALID_ARG"),
    (dict(cuk=None), "FA_ERR_INVALID_ARG"),
    (dict(k=None), "FA_ERR_INVALID_ARG"),
    (dict(q=FAKE + 2), "FA_ERR_INVALID_ARG"),
    (dict(scale=-1.0), "FA_ERR_INVALID_ARG"),
])
def test_varlen_rejects_bad_arguments_on_the_host(lib, kw, code):
    assert varlen(lib, **kw) == E[code]
    assert lib.fa_last_error_string()


def test_varlen_empty_batch_is_a_noop(lib):
    assert varlen(lib, B=0) == 0
    assert varlen(lib, tq=0) == 0
    assert varlen(lib, max_q=0) == 0


# The next three calls pass validation, so on a machine with a GPU they would launch
# kernels on the fake addresses: they run only where no device exists.
NO_DEVICE_ONLY = pytest.mark.skipif(torch.cuda.is_available(),
                                    reason="fake pointers must never reach a device")


@NO_DEVICE_ONLY
def test_varlen_without_keys_passes_validation(lib):
    assert varlen(lib, tk=0, k=None, v=None, q=FAKE) == E["FA_ERR_NO_DEVICE"]


def paged(lib, B=2, Hq=4, Hkv=2, max_q=9, maxp=4, npages=10, tq=12, D=128, page=16, scale=0.1,
          causal=1, q=FAKE, kc=FAKE, vc=FAKE, table=FAKE, o=FAKE, cuq=FAKE, lens=FAKE):
    return lib.fa_fwd_paged(q, kc, vc, table, o, None, cuq, lens, B, Hq, Hkv, max_q, maxp, npages,
                            tq, D, page, scale, causal, None)


@pytest.mark.parametrize("kw,code", [
    (dict(B=-1), "FA_ERR_INVALID_ARG"),
    (dict(D=96), "FA_ERR_UNSUPPORTED"),
    (dict(page=32), "FA_ERR_UNSUPPORTED"),
    (dict(Hq=3), "FA_ERR_INVALID_ARG"),
    (dict(maxp=0), "FA_ERR_INVALID_ARG"),
    (dict(npages=0), "FA_ERR_INVALID_ARG"),
    (dict(table=None), "FA_ERR_INVALID_ARG"),
    (dict(lens=None), "FA_ERR_INVALID_ARG"),
    (dict(kc=FAKE + 4), "FA_ERR_INVALID_ARG"),
    (dict(scale=float("inf")), "FA_ERR_INVALID_ARG"),
])
def test_paged_prefill_rejects_bad_arguments_on_the_host(lib, kw, code):
    assert paged(lib, **kw) == E[code]
    assert lib.fa_last_error_string()


def test_paged_prefill_empty_batch_is_a_noop(lib):
    assert paged(lib, B=0) == 0
    assert paged(lib, tq=0) == 0


def quant(lib, x=FAKE, codes=FAKE, scales=FAKE, Z=4, N=300, D=128, group=128, signs=None):
    return lib.fa_quantize_e4m3(x, codes, scales, Z, N, D, group, signs, None)


@pytest.mark.parametrize("kw,code", [
    (dict(Z=-1), "FA_ERR_INVALID_ARG"),
    (dict(N=-5), "FA_ERR_INVALID_ARG"),
    (dict(D=96), "FA_ERR_UNSUPPORTED"),
    (dict(group=64), "FA_ERR_UNSUPPORTED"),
    (dict(Z=70000), "FA_ERR_UNSUPPORTED"),
    (dict(x=None), "FA_ERR_INVALID_ARG"),
    (dict(codes=None), "FA_ERR_INVALID_ARG"),
    (dict(scales=None), "FA_ERR_INVALID_ARG"),
    (dict(x=FAKE + 8), "FA_ERR_INVALID_ARG"),
    (dict(codes=FAKE + 1), "FA_ERR_INVALID_ARG"),
])
def test_quantize_rejects_bad_arguments_on_the_host(lib, kw, code):
    assert quant(lib, **kw) == E[code]
    assert lib.fa_last_error_string()


def test_quantize_of_no_slices_is_a_noop(lib):
    assert quant(lib, Z=0) == 0


@NO_DEVICE_ONLY
def test_quantize_empty_slices_need_no_data_pointers(lib):
    # N == 0 still writes scales (1 per slice for group 0), so it reaches the device
    assert quant(lib, N=0, x=None, codes=None, group=0) == E["FA_ERR_NO_DEVICE"]


def fp8(lib, B=1, Hq=2, Hkv=1, Nq=8, Nk=8, D=128, scale=0.1, causal=0, q=FAKE, k=FAKE,
        v=FAKE, qs=FAKE, ks=FAKE, vs=FAKE, o=FAKE):
    return lib.fa_fwd_fp8(q, k, v, qs, ks, vs, o, None, B, Hq, Hkv, Nq, Nk, D, scale, causal,
                          None)


@pytest.mark.parametrize("kw,code", [
    (dict(B=-1), "FA_ERR_INVALID_ARG"),
    (dict(D=64), "FA_ERR_UNSUPPORTED"),
    (dict(D=96), "FA_ERR_UNSUPPORTED"),
    (dict(Hq=3, Hkv=2), "FA_ERR_INVALID_ARG"),
    (dict(causal=1, Nq=9, Nk=8), "FA_ERR_INVALID_ARG"),
    (dict(scale=0.0), "FA_ERR_INVALID_ARG"),
    (dict(q=0), "FA_ERR_INVALID_ARG"),
    (dict(v=FAKE + 4), "FA_ERR_INVALID_ARG"),
    (dict(qs=None), "FA_ERR_INVALID_ARG"),
    (dict(ks=None), "FA_ERR_INVALID_ARG"),
    (dict(vs=None), "FA_ERR_INVALID_ARG"),
])
def test_fp8_forward_rejects_bad_arguments_on_the_host(lib, kw, code):
    assert fp8(lib, **kw) == E[code]
    assert lib.fa_last_error_string()


def test_fp8_forward_empty_problem_is_a_noop(lib):
    assert fp8(lib, B=0) == 0
    assert fp8(lib, Nq=0) == 0


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device path")
def test_fp8_calls_without_a_device_fail_loudly(lib):
    assert fp8(lib) == E["FA_ERR_NO_DEVICE"]
    assert quant(lib) == E["FA_ERR_NO_DEVICE"]


def merge(lib, oa=FAKE, la=FAKE, op=FAKE, lp=FAKE, out=None, rows=10, D=128, first=0):
    return lib.fa_merge_partials(oa, la, op, lp, out, rows, D, first, None)


@pytest.mark.parametrize("kw,code", [
    (dict(rows=-1), "FA_ERR_INVALID_ARG"),
    (dict(D=96), "FA_ERR_UNSUPPORTED"),
    (dict(oa=None), "FA_ERR_INVALID_ARG"),
    (dict(lp=None), "FA_ERR_INVALID_ARG"),
    (dict(op=FAKE + 2), "FA_ERR_INVALID_ARG"),
    (dict(out=FAKE + 4), "FA_ERR_INVALID_ARG"),
])
def test_merge_rejects_bad_arguments_on_the_host(lib, kw, code):
    assert merge(lib, **kw) == E[code]


def test_merge_of_no_rows_is_a_noop(lib):
    assert merge(lib, rows=0, oa=None, op=None) == 0


def bwd(lib, B=1, Hq=2, Hkv=1, Nq=8, Nk=8, D=128, scale=0.1, causal=0, q=FAKE, k=FAKE, v=FAKE,
        o=FAKE, lse=FAKE, do=FAKE, dq=FAKE, dk=FAKE, dv=FAKE, delta=FAKE):
    return lib.fa_bwd(q, k, v, o, lse, do, dq, dk, dv, delta, B, Hq, Hkv, Nq, Nk, D, scale,
                      causal, None)


@pytest.mark.parametrize("kw,code", [
    (dict(B=-1), "FA_ERR_INVALID_ARG"),
    (dict(D=96), "FA_ERR_UNSUPPORTED"),
    (dict(Hq=3, Hkv=2), "FA_ERR_INVALID_ARG"),
    (dict(causal=1, Nq=9, Nk=8), "FA_ERR_INVALID_ARG"),
    (dict(scale=0.0), "FA_ERR_INVALID_ARG"),
    (dict(lse=None), "FA_ERR_INVALID_ARG"),
    (dict(delta=None), "FA_ERR_INVALID_ARG"),
    (dict(dk=None), "FA_ERR_INVALID_ARG"),
    (dict(do=FAKE + 2), "FA_ERR_INVALID_ARG"),
    (dict(dv=FAKE + 8), "FA_ERR_INVALID_ARG"),
])
def test_bwd_rejects_bad_arguments_on_the_host(lib, kw, code):
    assert bwd(lib, **kw) == E[code]


def test_bwd_empty_problems(lib):
    assert bwd(lib, B=0) == 0
    assert bwd(lib, Nq=0, Nk=0) == 0


@NO_DEVICE_ONLY
def test_bwd_without_queries_still_reaches_the_device(lib):
    # no queries but keys: dK = dV = 0 must still be written
    assert bwd(lib, Nq=0, q=None, o=None, lse=None, do=None, dq=None,
               delta=None) == E["FA_ERR_NO_DEVICE"]


def fwd_host(lib, B=1, Hq=2, Hkv=1, Nq=8, Nk=8, D=128, scale=0.1, causal=0, qh=FAKE, kh=FAKE,
             vh=FAKE, oh=FAKE, lh=FAKE, q=FAKE, k=FAKE, v=FAKE, o=FAKE, l=FAKE):
    return lib.fa_fwd_host(qh, kh, vh, oh, lh, q, k, v, o, l, B, Hq, Hkv, Nq, Nk, D, scale, causal,
                           None)


@pytest.mark.parametrize("kw,code", [
    (dict(B=-1), "FA_ERR_INVALID_ARG"),
    (dict(D=96), "FA_ERR_UNSUPPORTED"),
    (dict(Hq=3, Hkv=2), "FA_ERR_INVALID_ARG"),
    (dict(qh=None), "FA_ERR_INVALID_ARG"),
    (dict(vh=None), "FA_ERR_INVALID_ARG"),
    (dict(oh=None), "FA_ERR_INVALID_ARG"),
    (dict(lh=None), "FA_ERR_INVALID_ARG"),     # lse_host and lse_dev: both or neither
    (dict(q=FAKE + 4), "FA_ERR_INVALID_ARG"),
])
def test_fwd_host_rejects_bad_arguments_on_the_host(lib, kw, code):
    assert fwd_host(lib, **kw) == E[code]


def test_fwd_host_empty_problem_is_a_noop(lib):
    assert fwd_host(lib, B=0) == 0
    assert fwd_host(lib, Nq=0) == 0


@pytest.mark.parametrize("limit,ptr", [(0, None), (2_000_000, None), (100, FAKE + 2)])
def test_wait_selftest_rejects_bad_arguments(lib, limit, ptr):
    assert lib.fa_selftest_wait_timeout(limit, ptr, None) == E["FA_ERR_INVALID_ARG"]


@NO_DEVICE_ONLY
def test_wait_selftest_needs_a_device(lib):
    assert lib.fa_selftest_wait_timeout(100, None, None) == E["FA_ERR_NO_DEVICE"]
