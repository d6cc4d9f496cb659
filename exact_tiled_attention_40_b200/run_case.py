"""Run one named workload through the library and print per-launch times.

    python -m exact_tiled_attention_40_b200.run_case --case gqa_b1_hq32_hkv8_n8192_d128_causal
    python -m exact_tiled_attention_40_b200.run_case --case decode_b64_hq32_hkv8_d128_page16
    python -m exact_tiled_attention_40_b200.run_case --case gqa_b1_hq32_hkv8_n8192_d128_causal --op bwd
    python -m exact_tiled_attention_40_b200.run_case --case fp8_gqa_b1_hq32_hkv8_n8192_d128_causal
    python -m exact_tiled_attention_40_b200.run_case --case fp8_gqa_b1_hq32_hkv8_n8192_d128_causal --op quantize

--op bwd times fa_bwd on a prefill case (its inputs: the library forward's O and
LSE and a seeded output gradient); its rate counts the backward's five matrix
products, 2.5 times the forward's FLOPs.  For an FP8 case the inputs are
quantised once before timing and fa_fwd_fp8 is timed (--op quantize times
fa_quantize_e4m3 of Q, K and V instead, in GB/s of bf16 read and codes written).

Inputs come from the seeded generator and stay resident on the device; a
256 MiB buffer is written before every launch so no launch finds its inputs in
L2 (--clean-l2 also reads another 256 MiB after it, so that no dirty line of the
flush is left for the launch to write back: see l2flush.py).  Each launch is timed with CUDA events on the launching stream.  Handy for
profiling one kernel on one workload.
"""
from __future__ import annotations

import argparse
import json
import statistics

import torch

from . import fa
from .inputs import (DECODE_CASES, FP8_CASES, PAGED_PREFILL_CASES, PREFILL_CASES, VARLEN_CASES,
                     hadamard_signs, make_decode, make_dout, make_paged_prefill, make_prefill,
                     make_varlen, varlen_flops)
from .l2flush import L2Flush


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--case", required=True,
                    choices=sorted(PREFILL_CASES) + sorted(DECODE_CASES) + sorted(VARLEN_CASES)
                    + sorted(PAGED_PREFILL_CASES) + sorted(FP8_CASES))
    ap.add_argument("--op", default="fwd", choices=["fwd", "bwd", "quantize"])
    ap.add_argument("--iters", type=int, default=5)
    ap.add_argument("--clean-l2", action="store_true")
    args = ap.parse_args()
    dev = torch.device("cuda", 0)
    flush = L2Flush(dev)
    stream = torch.cuda.current_stream(dev)
    if args.op == "bwd":
        c = PREFILL_CASES[args.case]
        q, k, v, gen = make_prefill(c)
        do = make_dout(c, gen)
        q, k, v, do = q.to(dev), k.to(dev), v.to(dev), do.to(dev)
        o, lse = fa.attention(q, k, v, c.softmax_scale, c.causal)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        delta = torch.empty((c.B, c.Hq, c.Nq), dtype=torch.float32, device=dev)

        def launch():
            fa.fa_bwd(q, k, v, o, lse, do, dq, dk, dv, delta, c.B, c.Hq, c.Hkv, c.Nq, c.Nk, c.D,
                      c.softmax_scale, c.causal, stream=stream.cuda_stream)
        work, unit = 2.5 * c.flops / 1e12, "TFLOP/s"
    elif args.case in FP8_CASES:
        f = FP8_CASES[args.case]
        c = f.prefill
        q, k, v, _ = make_prefill(c)
        q, k, v = q.to(dev), k.to(dev), v.to(dev)
        signs = None if f.sign_seed is None else hadamard_signs(c.D, f.sign_seed).to(dev)
        q8, qs = fa.quantize_e4m3(q, 128, signs)
        k8, ks = fa.quantize_e4m3(k, 128, signs)
        v8, vs = fa.quantize_e4m3(v, 0)
        o = torch.empty(q.shape, dtype=torch.bfloat16, device=dev)
        lse = torch.empty((c.B, c.Hq, c.Nq), dtype=torch.float32, device=dev)
        if args.op == "quantize":
            def launch():
                s_ = stream.cuda_stream
                fa.fa_quantize_e4m3(q, q8, qs, c.B * c.Hq, c.Nq, c.D, 128, signs, stream=s_)
                fa.fa_quantize_e4m3(k, k8, ks, c.B * c.Hkv, c.Nk, c.D, 128, signs, stream=s_)
                fa.fa_quantize_e4m3(v, v8, vs, c.B * c.Hkv, c.Nk, c.D, 0, None, stream=s_)
            elems = q.numel() + k.numel() + v.numel()
            work, unit = 3 * elems / 1e9, "GB/s"
        else:
            def launch():
                fa.fa_fwd_fp8(q8, k8, v8, qs, ks, vs, o, lse, c.B, c.Hq, c.Hkv, c.Nq, c.Nk, c.D,
                              c.softmax_scale, c.causal, stream=stream.cuda_stream)
            work, unit = c.flops / 1e12, "TFLOP/s"
    elif args.case in PREFILL_CASES:
        c = PREFILL_CASES[args.case]
        q, k, v, _ = make_prefill(c)
        q, k, v = q.to(dev), k.to(dev), v.to(dev)
        o = torch.empty_like(q)
        lse = torch.empty((c.B, c.Hq, c.Nq), dtype=torch.float32, device=dev)

        def launch():
            fa.fa_fwd(q, k, v, o, lse, c.B, c.Hq, c.Hkv, c.Nq, c.Nk, c.D, c.softmax_scale,
                      c.causal, stream=stream.cuda_stream)
        work, unit = c.flops / 1e12, "TFLOP/s"
    elif args.case in PAGED_PREFILL_CASES:
        c = PAGED_PREFILL_CASES[args.case]
        q, kc, vc, table, cu_q, lens = make_paged_prefill(c)
        cu_k = torch.zeros_like(cu_q)
        cu_k[1:] = torch.cumsum(lens, 0)
        flops = varlen_flops(cu_q, cu_k, c.Hq, c.D, c.causal)
        max_q = int((cu_q[1:] - cu_q[:-1]).max())
        q, kc, vc, table, cu_q, lens = (t.to(dev) for t in (q, kc, vc, table, cu_q, lens))
        o = torch.empty_like(q)
        lse = torch.empty((c.Hq, q.shape[0]), dtype=torch.float32, device=dev)

        def launch():
            fa.fa_fwd_paged(q, kc, vc, table, o, lse, cu_q, lens, c.B, c.Hq, c.Hkv, max_q,
                            table.shape[1], c.num_pages, q.shape[0], c.D, c.page_size,
                            c.softmax_scale, c.causal, stream=stream.cuda_stream)
        work, unit = flops / 1e12, "TFLOP/s"
    elif args.case in VARLEN_CASES:
        c = VARLEN_CASES[args.case]
        q, k, v, cu_q, cu_k = make_varlen(c)
        flops = varlen_flops(cu_q, cu_k, c.Hq, c.D, c.causal)
        max_q = int((cu_q[1:] - cu_q[:-1]).max())
        max_k = int((cu_k[1:] - cu_k[:-1]).max())
        q, k, v, cu_q, cu_k = (t.to(dev) for t in (q, k, v, cu_q, cu_k))
        o = torch.empty_like(q)
        lse = torch.empty((c.Hq, q.shape[0]), dtype=torch.float32, device=dev)

        def launch():
            fa.fa_fwd_varlen(q, k, v, o, lse, cu_q, cu_k, c.B, c.Hq, c.Hkv, max_q, max_k,
                             q.shape[0], k.shape[0], c.D, c.softmax_scale, c.causal,
                             stream=stream.cuda_stream)
        work, unit = flops / 1e12, "TFLOP/s"
    else:
        c = DECODE_CASES[args.case]
        q, kc, vc, table, lens = make_decode(c)
        q, kc, vc, table, lens = (t.to(dev) for t in (q, kc, vc, table, lens))
        o = torch.empty_like(q)
        lse = torch.empty((c.B, c.Hq), dtype=torch.float32, device=dev)

        def launch():
            fa.fa_decode_paged(q, kc, vc, table, lens, o, c.B, c.Hq, c.Hkv, c.D, c.page_size,
                               c.softmax_scale, table.shape[1], c.num_pages, lse,
                               stream=stream.cuda_stream)
        work, unit = int(lens.sum()) * c.Hkv * c.D * 2 * 2 / 1e9, "GB/s"
    times = []
    for i in range(args.iters):
        flush(i, clean=args.clean_l2)
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        launch()
        b.record(stream)
        b.synchronize()
        times.append(a.elapsed_time(b))
    if fa.device_status() != 0:
        raise SystemExit(fa.last_error())
    best = min(times)
    print(json.dumps({"case": args.case, "ms": times, "best_ms": best,
                      "median_ms": statistics.median(times),
                      "rate_at_median": work / (statistics.median(times) * 1e-3), "unit": unit}))


if __name__ == "__main__":
    main()
