"""Thin Python binding of the C ABI in include/fa.h (argument marshalling only).

Every function forwards device pointers, sizes and the current CUDA stream to
``libfa_sm100.so``; all arithmetic runs in that library's sm_100a kernels.
There is no fallback: if the library or a CUDA device is missing, calls raise.
PyTorch is used for device memory and streams only.
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
# FA_LIBRARY may name another build of the same ABI (e.g. the FA_DEBUG build).
LIB_PATH = os.environ.get("FA_LIBRARY") or os.path.join(HERE, "libfa_sm100.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "fa.h")

FA_OK = 0
STATUS = {0: "FA_OK", 1: "FA_ERR_INVALID_ARG", 2: "FA_ERR_UNSUPPORTED", 3: "FA_ERR_CUDA",
          4: "FA_ERR_DEVICE_TIMEOUT", 5: "FA_ERR_DEVICE_INDEX", 6: "FA_ERR_NO_DEVICE",
          7: "FA_ERR_DEVICE_DIVERGED"}

_lib = None

_P = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float
_SIGS = {
    "fa_fwd": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _I, _P]),
    "fa_fwd_fp16": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _I, _P]),
    "fa_fwd_varlen": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _F, _I,
                           _P]),
    "fa_fwd_varlen_fp16": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _F,
                                _I, _P]),
    "fa_fwd_paged": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _I,
                          _F, _I, _P]),
    "fa_fwd_host": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _I,
                         _P]),
    "fa_quantize_e4m3": (_I, [_P, _P, _P, _I, _I, _I, _I, _P, _P]),
    "fa_fwd_fp8": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _I, _P]),
    "fa_merge_partials": (_I, [_P, _P, _P, _P, _P, ctypes.c_longlong, _I, _I, _P]),
    "fa_bwd": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _I, _P]),
    "fa_decode_paged": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _P, _I, _I, _P]),
    "fa_decode_paged_noalloc": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _P, _I, _I,
                                     _P]),
    "fa_selftest_wait_timeout": (_I, [ctypes.c_uint, _P, _P]),
    "fa_last_error_string": (ctypes.c_char_p, []),
    "fa_device_status": (_I, []),
    "fa_release": (None, []),
    "fa_version": (_I, []),
}


class FAError(RuntimeError):
    def __init__(self, code: int, where: str, msg: str):
        super().__init__(f"{where}: {STATUS.get(code, code)}: {msg}")
        self.code = code


def lib() -> ctypes.CDLL:
    """Load the shared library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise FAError(-1, "load", f"{LIB_PATH} is missing; run "
                          "`python -m exact_tiled_attention_40_b200.build`")
        l = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(l, name)
            fn.restype = res
            fn.argtypes = args
        _lib = l
    return _lib


def header_symbols() -> list[str]:
    """Names of the functions declared in include/fa.h."""
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\**\s+\**(fa_\w+)\s*\(", text, re.M)))


def _check(code: int, where: str):
    if code != FA_OK:
        raise FAError(code, where, lib().fa_last_error_string().decode())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def fa_fwd(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, D, scale, causal, stream=None):
    """Raw call of the C entry point (bf16 or fp16 chosen from q's dtype)."""
    fn = lib().fa_fwd if q.dtype == torch.bfloat16 else lib().fa_fwd_fp16
    s = _stream(q.device) if stream is None else ctypes.c_void_p(stream)
    _check(fn(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Hq, Hkv, Nq, Nk, D,
              float(scale), int(bool(causal)), s), "fa_fwd")


def attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, scale: float | None = None,
              causal: bool = False, return_lse: bool = True):
    """O, LSE for q [B,Hq,Nq,D] and k, v [B,Hkv,Nk,D] (bf16 or fp16, contiguous CUDA)."""
    if not (q.is_cuda and k.is_cuda and v.is_cuda):
        raise FAError(1, "attention", "tensors must live on a CUDA device")
    if q.dtype not in (torch.bfloat16, torch.float16) or k.dtype != q.dtype or v.dtype != q.dtype:
        raise FAError(1, "attention", "q, k, v must share dtype bf16 or fp16")
    q, k, v = q.contiguous(), k.contiguous(), v.contiguous()
    B, Hq, Nq, D = q.shape
    _, Hkv, Nk, _ = k.shape
    if scale is None:
        scale = D ** -0.5
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q.device) if return_lse else None
    fa_fwd(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, D, scale, causal)
    return o, lse


def fa_fwd_varlen(q, k, v, o, lse, cu_q, cu_k, B, Hq, Hkv, max_q, max_k, total_q, total_k, D,
                  scale, causal, stream=None):
    """Raw call of the ragged-batch entry point (bf16 or fp16 chosen from q's dtype)."""
    fn = lib().fa_fwd_varlen if q.dtype == torch.bfloat16 else lib().fa_fwd_varlen_fp16
    s = _stream(q.device) if stream is None else ctypes.c_void_p(stream)
    _check(fn(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(cu_q), _ptr(cu_k), B, Hq, Hkv,
              max_q, max_k, total_q, total_k, D, float(scale), int(bool(causal)), s),
           "fa_fwd_varlen")


def attention_varlen(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, cu_seqlens_q: torch.Tensor,
                     cu_seqlens_k: torch.Tensor, max_seqlen_q: int, max_seqlen_k: int,
                     scale: float | None = None, causal: bool = False, return_lse: bool = True):
    """O [total_q,Hq,D] (and LSE [Hq,total_q]) for a ragged batch packed as
    q [total_q,Hq,D], k, v [total_k,Hkv,D] with int32 offsets cu_seqlens_* [B+1]."""
    for t in (q, k, v, cu_seqlens_q, cu_seqlens_k):
        if not t.is_cuda:
            raise FAError(1, "attention_varlen", "tensors must live on a CUDA device")
    if q.dtype not in (torch.bfloat16, torch.float16) or k.dtype != q.dtype or v.dtype != q.dtype:
        raise FAError(1, "attention_varlen", "q, k, v must share dtype bf16 or fp16")
    if cu_seqlens_q.dtype != torch.int32 or cu_seqlens_k.dtype != torch.int32:
        raise FAError(1, "attention_varlen", "cu_seqlens must be int32")
    q, k, v = q.contiguous(), k.contiguous(), v.contiguous()
    total_q, Hq, D = q.shape
    total_k, Hkv, _ = k.shape
    B = cu_seqlens_q.numel() - 1
    if scale is None:
        scale = D ** -0.5
    o = torch.empty_like(q)
    lse = torch.empty((Hq, total_q), dtype=torch.float32, device=q.device) if return_lse else None
    fa_fwd_varlen(q, k, v, o, lse, cu_seqlens_q.contiguous(), cu_seqlens_k.contiguous(), B, Hq,
                  Hkv, int(max_seqlen_q), int(max_seqlen_k), total_q, total_k, D, scale, causal)
    return o, lse


def fa_fwd_paged(q, kcache, vcache, block_table, o, lse, cu_q, seq_lens_k, B, Hq, Hkv, max_q,
                 max_pages_per_seq, num_pages, total_q, D, page_size, scale, causal, stream=None):
    """Raw call of the paged-prefill entry point (bf16)."""
    s = _stream(q.device) if stream is None else ctypes.c_void_p(stream)
    _check(lib().fa_fwd_paged(_ptr(q), _ptr(kcache), _ptr(vcache), _ptr(block_table), _ptr(o),
                              _ptr(lse), _ptr(cu_q), _ptr(seq_lens_k), B, Hq, Hkv, max_q,
                              max_pages_per_seq, num_pages, total_q, D, page_size, float(scale),
                              int(bool(causal)), s), "fa_fwd_paged")


def prefill_paged(q, kcache, vcache, block_table, cu_seqlens_q, seq_lens_k, max_seqlen_q,
                  scale=None, causal=True, return_lse=True):
    """O [total_q,Hq,D] (and LSE [Hq,total_q]) for packed new queries q [total_q,Hq,D]
    against a paged bf16 cache [num_pages,16,Hkv,D] (int32 block table and lengths)."""
    for t in (q, kcache, vcache, block_table, cu_seqlens_q, seq_lens_k):
        if not t.is_cuda:
            raise FAError(1, "prefill_paged", "tensors must live on a CUDA device")
    total_q, Hq, D = q.shape
    num_pages, page_size, Hkv, _ = kcache.shape
    B = cu_seqlens_q.numel() - 1
    if scale is None:
        scale = D ** -0.5
    o = torch.empty_like(q)
    lse = torch.empty((Hq, total_q), dtype=torch.float32, device=q.device) if return_lse else None
    fa_fwd_paged(q.contiguous(), kcache, vcache, block_table.contiguous(), o, lse,
                 cu_seqlens_q.contiguous(), seq_lens_k.contiguous(), B, Hq, Hkv,
                 int(max_seqlen_q), block_table.shape[1], num_pages, total_q, D, page_size, scale,
                 causal)
    return o, lse


def fa_fwd_host(q_host, k_host, v_host, o_host, lse_host, q, k, v, o, lse, B, Hq, Hkv, Nq, Nk,
                D, scale, causal, stream=None):
    """Raw call of the host-buffer forward (bf16): *_host are CPU tensors, the others
    the device staging tensors of the same shapes."""
    s = _stream(q.device) if stream is None else ctypes.c_void_p(stream)
    _check(lib().fa_fwd_host(_ptr(q_host), _ptr(k_host), _ptr(v_host), _ptr(o_host),
                             _ptr(lse_host), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Hq,
                             Hkv, Nq, Nk, D, float(scale), int(bool(causal)), s), "fa_fwd_host")


def attention_from_host(q_host, k_host, v_host, scale=None, causal=False, device=None,
                        staging=None):
    """O and LSE in pinned host memory for bf16 q_host [B,Hq,Nq,D], k_host, v_host
    [B,Hkv,Nk,D] (contiguous, preferably pinned CPU tensors); the copies overlap the
    forward chunk by chunk.  `staging` = (q, k, v, o, lse) device tensors to reuse.
    Asynchronous like every call here: the host outputs are complete once the
    current stream has passed this call (e.g. after torch.cuda.synchronize())."""
    for t in (q_host, k_host, v_host):
        if t.is_cuda or t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise FAError(1, "attention_from_host", "contiguous bf16 CPU tensors expected")
    device = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    B, Hq, Nq, D = q_host.shape
    _, Hkv, Nk, _ = k_host.shape
    if scale is None:
        scale = D ** -0.5
    if staging is None:
        staging = (torch.empty(q_host.shape, dtype=torch.bfloat16, device=device),
                   torch.empty(k_host.shape, dtype=torch.bfloat16, device=device),
                   torch.empty(v_host.shape, dtype=torch.bfloat16, device=device),
                   torch.empty(q_host.shape, dtype=torch.bfloat16, device=device),
                   torch.empty((B, Hq, Nq), dtype=torch.float32, device=device))
    o_host = torch.empty(q_host.shape, dtype=torch.bfloat16, pin_memory=True)
    lse_host = torch.empty((B, Hq, Nq), dtype=torch.float32, pin_memory=True)
    q, k, v, o, lse = staging
    fa_fwd_host(q_host, k_host, v_host, o_host, lse_host, q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, D,
                scale, causal)
    return o_host, lse_host


def fa_quantize_e4m3(x, codes, scales, Z, N, D, group_rows, signs=None, stream=None):
    """Raw call of the E4M3 quantiser's C entry point."""
    s = _stream(x.device) if stream is None else ctypes.c_void_p(stream)
    _check(lib().fa_quantize_e4m3(_ptr(x), _ptr(codes), _ptr(scales), Z, N, D, group_rows,
                                  _ptr(signs), s), "fa_quantize_e4m3")


def quantize_e4m3(x: torch.Tensor, group_rows: int = 128, signs: torch.Tensor | None = None):
    """E4M3 codes (uint8, x's shape) and fp32 scales of a bf16 CUDA tensor x [..., N, D]:
    scales [prod(...), ceil(N / 128)] for group_rows 128, [prod(...)] for 0.  With
    signs [D] (+-1 fp32), rows are rotated by diag(signs) H / sqrt(D) first."""
    if not x.is_cuda or x.dtype != torch.bfloat16:
        raise FAError(1, "quantize_e4m3", "x must be a bf16 CUDA tensor")
    if signs is not None and (not signs.is_cuda or signs.dtype != torch.float32):
        raise FAError(1, "quantize_e4m3", "signs must be an fp32 CUDA tensor")
    x = x.contiguous()
    *lead, N, D = x.shape
    Z = 1
    for d in lead:
        Z *= d
    codes = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    shape = (Z, -(-N // 128)) if group_rows == 128 else (Z,)
    scales = torch.empty(shape, dtype=torch.float32, device=x.device)
    fa_quantize_e4m3(x, codes, scales, Z, N, D, group_rows,
                     None if signs is None else signs.contiguous())
    return codes, scales


def fa_fwd_fp8(q8, k8, v8, q_scale, k_scale, v_scale, o, lse, B, Hq, Hkv, Nq, Nk, D, scale,
               causal, stream=None):
    """Raw call of the FP8 forward's C entry point."""
    s = _stream(q8.device) if stream is None else ctypes.c_void_p(stream)
    _check(lib().fa_fwd_fp8(_ptr(q8), _ptr(k8), _ptr(v8), _ptr(q_scale), _ptr(k_scale),
                            _ptr(v_scale), _ptr(o), _ptr(lse), B, Hq, Hkv, Nq, Nk, D, float(scale),
                            int(bool(causal)), s), "fa_fwd_fp8")


def attention_fp8_quantised(q8, k8, v8, q_scale, k_scale, v_scale, scale=None, causal=False,
                            return_lse=True):
    """O (bf16) and LSE from E4M3 codes q8 [B,Hq,Nq,128], k8, v8 [B,Hkv,Nk,128] (uint8) with
    the scales quantize_e4m3 writes (q, k in 128-row groups, v per slice)."""
    for t in (q8, k8, v8, q_scale, k_scale, v_scale):
        if not t.is_cuda:
            raise FAError(1, "attention_fp8", "tensors must live on a CUDA device")
    if q8.dtype != torch.uint8 or k8.dtype != torch.uint8 or v8.dtype != torch.uint8:
        raise FAError(1, "attention_fp8", "codes must be uint8")
    B, Hq, Nq, D = q8.shape
    _, Hkv, Nk, _ = k8.shape
    if k8.shape != v8.shape or k8.shape[0] != B or k8.shape[3] != D:
        raise FAError(1, "attention_fp8", "k8, v8 must be [B, Hkv, Nk, D] like q8's B and D")
    want = {"q_scale": (q_scale, B * Hq * (-(-Nq // 128))),
            "k_scale": (k_scale, B * Hkv * (-(-Nk // 128))), "v_scale": (v_scale, B * Hkv)}
    for name, (t, n) in want.items():
        if t.dtype != torch.float32 or t.numel() != n:
            raise FAError(1, "attention_fp8", f"{name} must hold {n} fp32 scales")
    if scale is None:
        scale = D ** -0.5
    o = torch.empty((B, Hq, Nq, D), dtype=torch.bfloat16, device=q8.device)
    lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q8.device) if return_lse else None
    fa_fwd_fp8(q8.contiguous(), k8.contiguous(), v8.contiguous(), q_scale.contiguous(),
               k_scale.contiguous(), v_scale.contiguous(), o, lse, B, Hq, Hkv, Nq, Nk, D, scale,
               causal)
    return o, lse


def attention_fp8(q, k, v, scale=None, causal=False, signs=None, return_lse=True):
    """FP8 attention of bf16 q [B,Hq,Nq,128], k, v [B,Hkv,Nk,128]: q and k quantised in
    128-row groups (rotated by the Walsh-Hadamard map with `signs` when given), v per
    (sequence, head), then the E4M3 forward.  Returns (O bf16, LSE fp32)."""
    q8, qs = quantize_e4m3(q, 128, signs)
    k8, ks = quantize_e4m3(k, 128, signs)
    v8, vs = quantize_e4m3(v, 0)
    return attention_fp8_quantised(q8, k8, v8, qs, ks, vs, scale, causal, return_lse)


def fa_bwd(q, k, v, o, lse, dout, dq, dk, dv, delta, B, Hq, Hkv, Nq, Nk, D, scale, causal,
           stream=None):
    """Raw call of the backward's C entry point."""
    s = _stream(q.device) if stream is None else ctypes.c_void_p(stream)
    _check(lib().fa_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dout), _ptr(dq),
                        _ptr(dk), _ptr(dv), _ptr(delta), B, Hq, Hkv, Nq, Nk, D, float(scale),
                        int(bool(causal)), s), "fa_bwd")


def attention_backward(q, k, v, o, lse, dout, scale=None, causal=False):
    """(dQ, dK, dV) bf16 of attention(q, k, v) for the output gradient dout, given the
    forward's o and lse (q, o, dout [B,Hq,Nq,D]; k, v [B,Hkv,Nk,D]; bf16 CUDA)."""
    for t in (q, k, v, o, lse, dout):
        if not t.is_cuda:
            raise FAError(1, "attention_backward", "tensors must live on a CUDA device")
    if any(t.dtype != torch.bfloat16 for t in (q, k, v, o, dout)) or lse.dtype != torch.float32:
        raise FAError(1, "attention_backward", "bf16 q, k, v, o, dout and fp32 lse expected")
    q, k, v, o, dout, lse = (t.contiguous() for t in (q, k, v, o, dout, lse))
    B, Hq, Nq, D = q.shape
    _, Hkv, Nk, _ = k.shape
    if scale is None:
        scale = D ** -0.5
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    delta = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q.device)
    fa_bwd(q, k, v, o, lse, dout, dq, dk, dv, delta, B, Hq, Hkv, Nq, Nk, D, scale, causal)
    return dq, dk, dv


def merge_partials(o_acc, lse_acc, o_part, lse_part, first=False, o_out=None, stream=None):
    """Fold a partial result (o_part bf16 [..., D], lse_part fp32 [...]) into the fp32
    accumulator (o_acc [..., D], lse_acc [...]) by their LSE, in place; with `o_out`
    (bf16, o_part's shape) the merged rows are also written there."""
    for t in (o_acc, lse_acc, o_part, lse_part):
        if not t.is_cuda or not t.is_contiguous():
            raise FAError(1, "merge_partials", "tensors must be contiguous CUDA tensors")
    if o_acc.dtype != torch.float32 or lse_acc.dtype != torch.float32 or \
            lse_part.dtype != torch.float32 or o_part.dtype != torch.bfloat16:
        raise FAError(1, "merge_partials", "o_acc, lse fp32 and o_part bf16 expected")
    if o_acc.shape != o_part.shape or lse_acc.shape != lse_part.shape or \
            o_part.shape[:-1] != lse_part.shape:
        raise FAError(1, "merge_partials", "shape mismatch")
    if o_out is not None and (o_out.shape != o_part.shape or o_out.dtype != torch.bfloat16
                              or not o_out.is_contiguous()):
        raise FAError(1, "merge_partials", "o_out must be a contiguous bf16 tensor like o_part")
    D = o_part.shape[-1]
    rows = lse_part.numel()
    s = _stream(o_part.device) if stream is None else ctypes.c_void_p(stream)
    _check(lib().fa_merge_partials(_ptr(o_acc), _ptr(lse_acc), _ptr(o_part), _ptr(lse_part),
                                   _ptr(o_out), rows, D, int(bool(first)), s),
           "fa_merge_partials")


def fa_decode_paged(q, kcache, vcache, block_table, seq_lens, o, B, Hq, Hkv, D, page_size, scale,
                    max_pages_per_seq, num_pages, lse=None, stream=None):
    """Raw call of the C entry point."""
    s = _stream(q.device) if stream is None else ctypes.c_void_p(stream)
    _check(lib().fa_decode_paged(_ptr(q), _ptr(kcache), _ptr(vcache), _ptr(block_table),
                                 _ptr(seq_lens), _ptr(o), B, Hq, Hkv, D, page_size, float(scale),
                                 s, max_pages_per_seq, num_pages, _ptr(lse)), "fa_decode_paged")


def decode_paged(q, kcache, vcache, block_table, seq_lens, scale=None, return_lse=True):
    """O [B,Hq,D] (and LSE [B,Hq]) for one query token per sequence over a paged cache."""
    B, Hq, D = q.shape
    num_pages, page_size, Hkv, _ = kcache.shape
    if scale is None:
        scale = D ** -0.5
    if block_table.dtype != torch.int32 or seq_lens.dtype != torch.int32:
        raise FAError(1, "decode_paged", "block_table and seq_lens must be int32")
    block_table = block_table.contiguous()
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device) if return_lse else None
    fa_decode_paged(q.contiguous(), kcache.contiguous(), vcache.contiguous(), block_table,
                    seq_lens.contiguous(), o, B, Hq, Hkv, D, page_size, scale,
                    block_table.shape[1], num_pages, lse)
    return o, lse


def decode_paged_noalloc(q, kcache, vcache, block_table, seq_lens, o, lse=None, scale=None,
                         stream=None):
    """fa_decode_paged_noalloc: same result as decode_paged, written into the
    caller's o (and lse); the library allocates no device memory for it."""
    B, Hq, D = q.shape
    num_pages, page_size, Hkv, _ = kcache.shape
    if scale is None:
        scale = D ** -0.5
    s = _stream(q.device) if stream is None else ctypes.c_void_p(stream)
    _check(lib().fa_decode_paged_noalloc(_ptr(q), _ptr(kcache), _ptr(vcache), _ptr(block_table),
                                         _ptr(seq_lens), _ptr(o), B, Hq, Hkv, D, page_size,
                                         float(scale), s, block_table.shape[1], num_pages,
                                         _ptr(lse)), "fa_decode_paged_noalloc")


def device_status() -> int:
    """Synchronise and read/clear the device error word (FA_* code)."""
    return lib().fa_device_status()


def selftest_wait_timeout(limit_us: int = 20000, device=None):
    """Run the bounded-wait self-test (a wait nothing satisfies, given up after
    limit_us) and return (fa_device_status() code, whether the wait gave up)."""
    device = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    flag = torch.full((1,), -1, dtype=torch.int32, device=device)
    _check(lib().fa_selftest_wait_timeout(int(limit_us), _ptr(flag), _stream(device)),
           "fa_selftest_wait_timeout")
    status = device_status()
    return status, int(flag.item()) == 1


def last_error() -> str:
    return lib().fa_last_error_string().decode()


def release():
    lib().fa_release()
