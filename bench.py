#!/usr/bin/env python
"""Benchmark of the exact tiled attention hot path on B200.

One step = one pass of the whole path over one batch of synthetic input:
  * prefill: fa_fwd on the Llama-3-8B-shaped GQA causal workload
    (B=1, Hq=32, Hkv=8, Nq=Nk=8192, D=128, bf16, scale 1/sqrt(128));
  * decode:  fa_decode_paged on the paged-cache workload (B=64 sequences,
    Hq=32, Hkv=8, D=128, pages of 16 tokens, lengths U[512, 8192], pool of
    40000 pages, bf16).
Each kernel launch is timed with CUDA events on the launching stream; a 256 MiB
buffer is written before every launch so no launch finds its inputs in L2.  The
decode is also timed (outside the timed region) after a clean flush that reads
another 256 MiB after the write: the write leaves L2 full of dirty lines whose
write-back lands inside a bandwidth-bound launch.

``value`` is prefill TFLOP/s (4*B*Hq*Nq*Nk*D / 2 for causal) summed over ranks
and divided by the slowest rank's prefill time; the decode KV GB/s is reported
beside it.  Multi-GPU runs are weak-scaled replicas (each rank runs the same
per-rank workload on its own inputs; the path has no exchange step).

Rows beyond the headline (``"widened"``, rank 0 at N=1, timed outside the
headline's region, each with its roofline fraction): ragged and paged prefill,
the (2, 8, 4096, 64) fp16 workload with and without the causal mask, the
131072-token causal GQA workload, the FP8 forward and its quantiser, and the
backward.  ``--headline-only`` skips them.

``--impl reference`` times the fp64 CPU oracle on a bounded sample of the same
workloads (rank 0 only).
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import re
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from exact_tiled_attention_40_b200.inputs import (  # noqa: E402
    DECODE_CASES, PAGED_PREFILL_CASES, PREFILL_CASES, VARLEN_CASES, make_decode,
    make_paged_prefill, make_prefill, make_varlen, varlen_flops)
from exact_tiled_attention_40_b200.l2flush import FLUSH_BYTES, L2Flush  # noqa: E402

METRIC = "attention TFLOP/s & % BF16 tensor peak (prefill); decode KV GB/s & % HBM peak"
PREFILL = PREFILL_CASES["gqa_b1_hq32_hkv8_n8192_d128_causal"]
DECODE = DECODE_CASES["decode_b64_hq32_hkv8_d128_page16"]
RAGGED = VARLEN_CASES["varlen_b16_hq32_hkv8_d128_causal"]
PAGED = PAGED_PREFILL_CASES["paged_prefill_b16_chunk512_hq32_hkv8_d128"]
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash(name: str) -> str:
    """Hash of a kernel source file's code: comments and blank lines removed, so
    that an edit of the comments alone does not retire a recorded measurement."""
    with open(os.path.join(ROOT, "exact_tiled_attention_40_b200", "csrc", name)) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    lines = [re.sub(r"//.*$", "", ln).rstrip() for ln in text.splitlines()]
    code = "\n".join(ln for ln in lines if ln.strip())
    return hashlib.sha256(code.encode()).hexdigest()[:16]


def recorded_traffic(kernel: str, source: str):
    """DRAM bytes per launch recorded from an ncu capture of the current source,
    or None when no capture matches the source as it is now."""
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(path):
        return None
    h = kernel_source_hash(source)
    for line in open(path):
        parts = line.split()
        if len(parts) >= 3 and parts[0] == kernel and parts[1] == h:
            return float(parts[2])
    return None


class ClockSampler:
    """Samples SM clocks and throttle reasons with nvidia-smi every 20 ms while
    running; the summary keeps the samples taken inside the timed region
    (mark() brackets it), or all of them when none fell inside (a region shorter
    than the sampling interval), and says which."""
    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    INTERVAL_MS = 20

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.window = None
        out_dir = os.environ.get("FA_BENCH_OUT", os.path.join(ROOT, "bench_out"))
        self.path = os.path.join(out_dir, f"clocks_rank{index}.csv")

    def __enter__(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", str(self.INTERVAL_MS)],
                stdout=self.f, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.f.close()

    def mark(self, start: float, end: float):
        """The timed region in wall-clock seconds (time.time())."""
        self.window = (start, end)

    @staticmethod
    def parse(lines, window=None):
        """Summary of nvidia-smi CSV lines (FIELDS order); `window` = (start, end)
        in seconds since the epoch selects the samples taken inside it."""
        import datetime
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        rows = []
        for line in lines:
            cols = [c.strip() for c in line.split(",")]
            if len(cols) < 9:
                continue
            try:
                ts = datetime.datetime.strptime(cols[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                rows.append((ts, float(cols[1]), float(cols[2]),
                             [n for n, c in zip(names, cols[5:9]) if c.lower().startswith("active")]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        inside = [r for r in rows if window and window[0] <= r[0] <= window[1]]
        used, where = (inside, "timed region") if inside else (rows, "whole run")
        return {"sm_mhz": statistics.median(r[1] for r in used), "sm_max_mhz": used[-1][2],
                "reasons": sorted({n for r in used for n in r[3]}), "samples": len(used),
                "window": where, "interval_ms": ClockSampler.INTERVAL_MS}

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        with open(self.path) as f:
            return self.parse(f, self.window)


def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i["num_threads"] for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def oracle_prefill_sample(heads: int = 8):
    """fp64 oracle on the first `heads` query heads (and their KV heads) of the
    prefill workload, full causal rows.  Returns (TFLOP/s, seconds, sample text)."""
    import oracle
    q, k, v, _ = make_prefill(PREFILL)
    g = PREFILL.Hq // PREFILL.Hkv
    hk = max(1, heads // g)
    qs = q[:, :heads].float().double().numpy()
    ks = k[:, :hk].float().double().numpy()
    vs = v[:, :hk].float().double().numpy()
    t0 = time.perf_counter()
    oracle.attention(qs, ks, vs, PREFILL.softmax_scale, True)
    dt = time.perf_counter() - t0
    flops = 4.0 * heads * PREFILL.Nq * PREFILL.Nk * PREFILL.D / 2
    return flops / dt / 1e12, dt, (f"{heads} of {PREFILL.Hq} query heads of "
                                   f"{PREFILL.name} (full causal rows), fp64")


def oracle_decode_sample(seqs: int = 8):
    import oracle
    q, kc, vc, table, lens = make_decode(DECODE)
    kcf, vcf = kc.float().numpy(), vc.float().numpy()
    t0 = time.perf_counter()
    oracle.decode_paged(q[:seqs].float().double().numpy(), kcf, vcf, table[:seqs].numpy(),
                        lens[:seqs].numpy(), DECODE.softmax_scale, DECODE.page_size)
    dt = time.perf_counter() - t0
    kv_bytes = int(lens[:seqs].sum()) * DECODE.Hkv * DECODE.D * 2 * 2
    return kv_bytes / dt / 1e9, dt, f"{seqs} of {DECODE.B} sequences of {DECODE.name}, fp64"


def oracle_ragged_sample(heads: int = 4):
    """fp64 ragged-batch oracle on the shortest sequence of the ragged workload,
    its first `heads` query heads.  Returns (TFLOP/s, seconds, sample text)."""
    import oracle
    q, k, v, cu_q, cu_k = make_varlen(RAGGED)
    nq = cu_q[1:] - cu_q[:-1]
    b = int(torch.argmin(nq))
    q0, q1, k0, k1 = (int(x) for x in (cu_q[b], cu_q[b + 1], cu_k[b], cu_k[b + 1]))
    g = RAGGED.Hq // RAGGED.Hkv
    hk = max(1, heads // g)
    qs = q[q0:q1, :heads].float().double().numpy()
    ks = k[k0:k1, :hk].float().double().numpy()
    vs = v[k0:k1, :hk].float().double().numpy()
    cu1 = np.array([0, q1 - q0])
    ck1 = np.array([0, k1 - k0])
    t0 = time.perf_counter()
    oracle.varlen_attention(qs, ks, vs, cu1, ck1, RAGGED.softmax_scale, RAGGED.causal)
    dt = time.perf_counter() - t0
    flops = varlen_flops(torch.tensor(cu1), torch.tensor(ck1), heads, RAGGED.D, RAGGED.causal)
    return flops / dt / 1e12, dt, (f"sequence {b} ({q1 - q0} tokens), {heads} of {RAGGED.Hq} "
                                   f"query heads of {RAGGED.name}, fp64")


def oracle_paged_sample(heads: int = 4):
    """fp64 paged-prefill oracle on the sequence with the fewest cached keys of the
    paged workload, its first `heads` query heads.  Returns (TFLOP/s, seconds, text)."""
    import oracle
    q, kc, vc, table, cu_q, lens = make_paged_prefill(PAGED)
    b = int(torch.argmin(lens))
    q0, q1 = int(cu_q[b]), int(cu_q[b + 1])
    g = PAGED.Hq // PAGED.Hkv
    hk = max(1, heads // g)
    qs = q[q0:q1, :heads].float().double().numpy()
    kcs = kc[:, :, :hk].float().numpy()
    vcs = vc[:, :, :hk].float().numpy()
    cu1 = np.array([0, q1 - q0])
    t0 = time.perf_counter()
    oracle.paged_prefill(qs, kcs, vcs, table[b:b + 1].numpy(), cu1, lens[b:b + 1].numpy(),
                         PAGED.softmax_scale, PAGED.causal, PAGED.page_size)
    dt = time.perf_counter() - t0
    ck1 = torch.tensor([0, int(lens[b])])
    flops = varlen_flops(torch.tensor(cu1), ck1, heads, PAGED.D, PAGED.causal)
    return flops / dt / 1e12, dt, (f"sequence {b} ({q1 - q0} queries, {int(lens[b])} keys), "
                                   f"{heads} of {PAGED.Hq} query heads of {PAGED.name}, fp64")


def widened_rows(fa, dev, stream, flush, warmup, steps, peaks, peak_src):
    """Ragged and paged prefill (rows added beyond the headline path), each timed
    like the headline kernels with its roofline fraction and an oracle sample.
    A failure here is reported in the row and does not touch the headline."""
    out = {}
    sp = stream.cuda_stream

    def timed(launch):
        ts = []
        for i in range(warmup + steps):
            flush(i & 0xff)
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            launch()
            b.record(stream)
            b.synchronize()
            if i >= warmup:
                ts.append(a.elapsed_time(b))
        return statistics.median(ts)

    def row(name, flops, ms, sample_fn):
        tf = flops / (ms * 1e-3) / 1e12
        otf, odt, sample = sample_fn()
        return {"workload": name, "value": tf, "unit": "TFLOP/s", "ms_per_launch": ms,
                "roofline": {"bound": "tensor", "achieved": tf, "peak": peaks["bf16_tflops"],
                             "unit": "TFLOP/s", "frac": tf / peaks["bf16_tflops"],
                             "peak_source": f"{peak_src} burst bf16"},
                "cpu_baseline": {"value": otf, "unit": "TFLOP/s", "cores": cpu_threads(),
                                 "kind": "oracle", "sample": sample, "seconds": odt}}

    try:
        c = RAGGED
        q_h, k_h, v_h, cq_h, ck_h = make_varlen(c)
        flops = varlen_flops(cq_h, ck_h, c.Hq, c.D, c.causal)
        max_q = int((cq_h[1:] - cq_h[:-1]).max())
        max_k = int((ck_h[1:] - ck_h[:-1]).max())
        q, k, v, cq, ck = (t.to(dev) for t in (q_h, k_h, v_h, cq_h, ck_h))
        o = torch.empty_like(q)
        lse = torch.empty((c.Hq, q.shape[0]), dtype=torch.float32, device=dev)
        ms = timed(lambda: fa.fa_fwd_varlen(q, k, v, o, lse, cq, ck, c.B, c.Hq, c.Hkv, max_q,
                                            max_k, q.shape[0], k.shape[0], c.D, c.softmax_scale,
                                            c.causal, stream=sp))
        if fa.device_status() != 0:
            raise RuntimeError(fa.last_error())
        out["ragged_prefill"] = row(c.name, flops, ms, oracle_ragged_sample)
        del q, k, v, o, lse
    except Exception as e:  # reported, never fatal for the headline line
        out["ragged_prefill"] = {"workload": RAGGED.name, "error": f"{type(e).__name__}: {e}"[:300]}
    try:
        c = PAGED
        q_h, kc_h, vc_h, t_h, cq_h, l_h = make_paged_prefill(c)
        ck_h = torch.zeros_like(cq_h)
        ck_h[1:] = torch.cumsum(l_h, 0)
        flops = varlen_flops(cq_h, ck_h, c.Hq, c.D, c.causal)
        max_q = int((cq_h[1:] - cq_h[:-1]).max())
        q, kc, vc, tab, cq, ln = (t.to(dev) for t in (q_h, kc_h, vc_h, t_h, cq_h, l_h))
        o = torch.empty_like(q)
        lse = torch.empty((c.Hq, q.shape[0]), dtype=torch.float32, device=dev)
        ms = timed(lambda: fa.fa_fwd_paged(q, kc, vc, tab, o, lse, cq, ln, c.B, c.Hq, c.Hkv, max_q,
                                           tab.shape[1], c.num_pages, q.shape[0], c.D,
                                           c.page_size, c.softmax_scale, c.causal, stream=sp))
        if fa.device_status() != 0:
            raise RuntimeError(fa.last_error())
        out["paged_prefill"] = row(c.name, flops, ms, oracle_paged_sample)
        del q, kc, vc, o, lse
    except Exception as e:  # reported, never fatal for the headline line
        out["paged_prefill"] = {"workload": PAGED.name, "error": f"{type(e).__name__}: {e}"[:300]}
    return out


def fp8_and_backward_rows(fa, dev, stream, flush, warmup, steps, peaks, peak_src):
    """The FP8 forward and its quantiser, and the backward, on the headline
    prefill workload (B1 Hq32 Hkv8 N8192 D128 causal), each with its roofline."""
    from exact_tiled_attention_40_b200.inputs import FP8_CASES, hadamard_signs, make_dout
    out = {}
    sp = stream.cuda_stream

    def timed(launch):
        ts = []
        for i in range(warmup + steps):
            flush(i & 0xff)
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            launch()
            b.record(stream)
            b.synchronize()
            if i >= warmup:
                ts.append(a.elapsed_time(b))
        if fa.device_status() != 0:
            raise RuntimeError(fa.last_error())
        return statistics.median(ts)

    f = FP8_CASES["fp8_gqa_b1_hq32_hkv8_n8192_d128_causal"]
    c = f.prefill
    try:
        q_h, k_h, v_h, gen = make_prefill(c)
        q, k, v = q_h.to(dev), k_h.to(dev), v_h.to(dev)
        signs = hadamard_signs(c.D, f.sign_seed).to(dev)
        q8, qs = fa.quantize_e4m3(q, 128, signs)
        k8, ks = fa.quantize_e4m3(k, 128, signs)
        v8, vs = fa.quantize_e4m3(v, 0)
        o = torch.empty(q.shape, dtype=torch.bfloat16, device=dev)
        lse = torch.empty((c.B, c.Hq, c.Nq), dtype=torch.float32, device=dev)

        def quant():
            fa.fa_quantize_e4m3(q, q8, qs, c.B * c.Hq, c.Nq, c.D, 128, signs, stream=sp)
            fa.fa_quantize_e4m3(k, k8, ks, c.B * c.Hkv, c.Nk, c.D, 128, signs, stream=sp)
            fa.fa_quantize_e4m3(v, v8, vs, c.B * c.Hkv, c.Nk, c.D, 0, None, stream=sp)
        ms = timed(quant)
        gbs = 3 * (q.numel() + k.numel() + v.numel()) / (ms * 1e-3) / 1e9
        out["quantize_e4m3"] = {"workload": f.name, "value": gbs, "unit": "GB/s",
                                "ms_per_launch": ms,
                                "roofline": {"bound": "hbm", "achieved": gbs,
                                             "peak": peaks["hbm_gbs"], "unit": "GB/s",
                                             "frac": gbs / peaks["hbm_gbs"],
                                             "peak_source": f"{peak_src} copy"}}
        ms = timed(lambda: fa.fa_fwd_fp8(q8, k8, v8, qs, ks, vs, o, lse, c.B, c.Hq, c.Hkv, c.Nq,
                                         c.Nk, c.D, c.softmax_scale, c.causal, stream=sp))
        tf = c.flops / (ms * 1e-3) / 1e12
        pk = 2 * peaks["bf16_tflops"]
        out["fp8_prefill"] = {"workload": f.name, "value": tf, "unit": "TFLOP/s",
                              "ms_per_launch": ms,
                              "roofline": {"bound": "tensor", "achieved": tf, "peak": pk,
                                           "unit": "TFLOP/s", "frac": tf / pk,
                                           "peak_source": f"{peak_src} burst bf16 x 2 "
                                                          "(nominal fp8 / bf16 ratio)"}}
        do = make_dout(c, gen).to(dev)
        ob, lb = fa.attention(q, k, v, c.softmax_scale, c.causal)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        delta = torch.empty((c.B, c.Hq, c.Nq), dtype=torch.float32, device=dev)
        ms = timed(lambda: fa.fa_bwd(q, k, v, ob, lb, do, dq, dk, dv, delta, c.B, c.Hq, c.Hkv,
                                     c.Nq, c.Nk, c.D, c.softmax_scale, c.causal, stream=sp))
        tf = 2.5 * c.flops / (ms * 1e-3) / 1e12
        out["backward"] = {"workload": c.name, "value": tf, "unit": "TFLOP/s",
                           "ms_per_launch": ms, "flops": "2.5 x the forward's",
                           "roofline": {"bound": "tensor", "achieved": tf,
                                        "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                                        "frac": tf / peaks["bf16_tflops"],
                                        "peak_source": f"{peak_src} burst bf16"}}
    except Exception as e:  # reported, never fatal for the headline line
        out["error"] = f"{type(e).__name__}: {e}"[:300]
    return out


def oracle_heads_sample(case, heads: int = 1):
    """fp64 oracle on the first `heads` query heads of batch entry 0 of a dense
    prefill workload (full rows).  Returns (TFLOP/s, seconds, sample text)."""
    import oracle
    q, k, v, _ = make_prefill(case)
    g = case.Hq // case.Hkv
    hk = max(1, -(-heads // g))
    qs = q[:1, :heads].float().double().numpy()
    ks = k[:1, :hk].float().double().numpy()
    vs = v[:1, :hk].float().double().numpy()
    t0 = time.perf_counter()
    oracle.attention(qs, ks, vs, case.softmax_scale, case.causal)
    dt = time.perf_counter() - t0
    flops = 4.0 * heads * case.Nq * case.Nk * case.D / (2 if case.causal else 1)
    return flops / dt / 1e12, dt, f"{heads} of {case.B * case.Hq} (sequence, head) pairs of {case.name}, fp64"


def oracle_rows_sample(case, rows: int = 8):
    """fp64 oracle on `rows` query rows of head 0 (the last rows, full causal
    prefixes) of a long workload.  Returns (TFLOP/s, seconds, sample text)."""
    import oracle
    q, k, v, _ = make_prefill(case)
    sel = [(0, 0, case.Nq - 1 - r) for r in range(rows)]
    kd = k[:, :1].float().double().numpy()
    vd = v[:, :1].float().double().numpy()
    qd = q[:, :1].float().double().numpy()
    t0 = time.perf_counter()
    oracle.attention_rows(qd, kd, vd, case.softmax_scale, case.causal, sel)
    dt = time.perf_counter() - t0
    flops = sum(4.0 * (i + 1) * case.D for _, _, i in sel)
    return flops / dt / 1e12, dt, f"{rows} query rows (full causal prefixes) of {case.name}, fp64"


def dense_prefill_rows(fa, dev, stream, flush, warmup, steps, peaks, peak_src):
    """The pages' other dense prefill workloads: (2, 8, 4096, 64) fp16 with and
    without the causal mask, and the 131072-token causal GQA case."""
    out = {}
    sp = stream.cuda_stream
    specs = [("mha_fp16", "mha_b2_h8_n4096_d64_fp16", oracle_heads_sample),
             ("mha_fp16_causal", "mha_b2_h8_n4096_d64_fp16_causal", oracle_heads_sample),
             ("long_context", "gqa_b1_hq32_hkv8_n131072_d128_causal", oracle_rows_sample)]
    for key, name, sample_fn in specs:
        c = PREFILL_CASES[name]
        try:
            q_h, k_h, v_h, _ = make_prefill(c)
            q, k, v = q_h.to(dev), k_h.to(dev), v_h.to(dev)
            del q_h, k_h, v_h
            o = torch.empty_like(q)
            lse = torch.empty((c.B, c.Hq, c.Nq), dtype=torch.float32, device=dev)
            long_case = c.Nq > 16384
            n_warm, n_steps = (3, 5) if long_case else (warmup, steps)
            ts = []
            for i in range(n_warm + n_steps):
                flush(i & 0xff)
                a = torch.cuda.Event(enable_timing=True)
                b = torch.cuda.Event(enable_timing=True)
                a.record(stream)
                fa.fa_fwd(q, k, v, o, lse, c.B, c.Hq, c.Hkv, c.Nq, c.Nk, c.D, c.softmax_scale,
                          c.causal, stream=sp)
                b.record(stream)
                b.synchronize()
                if i >= n_warm:
                    ts.append(a.elapsed_time(b))
            if fa.device_status() != 0:
                raise RuntimeError(fa.last_error())
            ms = statistics.median(ts)
            tf = c.flops / (ms * 1e-3) / 1e12
            otf, odt, sample = sample_fn(c)
            # a launch of a tenth of a second or more runs under the power cap:
            # the GEMM peak measured over seconds is its denominator
            sustained = ms >= 100.0
            peak = peaks["bf16_tflops_sustained" if sustained else "bf16_tflops"]
            kind = "sustained" if sustained else "burst"
            out[key] = {"workload": c.name, "dtype": c.dtype, "value": tf, "unit": "TFLOP/s",
                        "ms_per_launch": ms, "launches_timed": n_steps,
                        "roofline": {"bound": "tensor", "achieved": tf,
                                     "peak": peak, "unit": "TFLOP/s",
                                     "frac": tf / peak,
                                     "peak_source": f"{peak_src} {kind} bf16 (fp16 dense "
                                                    "tensor peak is the same)",
                                     "frac_of_burst": tf / peaks["bf16_tflops"],
                                     "frac_of_nominal_2250": tf / 2250.0},
                        "cpu_baseline": {"value": otf, "unit": "TFLOP/s",
                                         "cores": cpu_threads(), "kind": "oracle",
                                         "sample": sample, "seconds": odt}}
            del q, k, v, o, lse
            torch.cuda.empty_cache()
        except Exception as e:  # reported, never fatal for the headline line
            out[key] = {"workload": c.name, "error": f"{type(e).__name__}: {e}"[:300]}
    return out


def run_reference(args, world, rank):
    if rank != 0:
        return 0
    vals, dts = [], []
    for i in range(args.warmup + args.steps):
        tf, dt, sample = oracle_prefill_sample(heads=1)
        if i >= args.warmup:
            vals.append(tf)
            dts.append(dt)
    dec_gbs, dec_dt, dec_sample = oracle_decode_sample(seqs=2)
    value = statistics.median(vals)
    cores = cpu_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * statistics.mean(dts), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": PREFILL.name, "decode_workload": DECODE.name,
                   "l2": "oracle runs on the host"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "decode": {"value": dec_gbs, "unit": "GB/s", "sample": dec_sample},
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--headline-only", action="store_true",
                    help="skip the rows beyond the headline prefill and decode")
    args = ap.parse_args()
    world, rank, local = dist_env()
    if args.impl == "reference":
        return run_reference(args, world, rank)
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")

    from exact_tiled_attention_40_b200 import fa

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=dev)
        pg = torch.distributed.group.WORLD

    def barrier():
        if pg is not None:
            torch.distributed.barrier()
        torch.cuda.synchronize()

    # ---- inputs: each rank its own replica (seed offset by rank), resident in HBM
    pcase = dataclasses.replace(PREFILL, seed=PREFILL.seed + 1000 * rank)
    dcase = dataclasses.replace(DECODE, seed=DECODE.seed + 1000 * rank)
    q_h, k_h, v_h, _ = make_prefill(pcase)
    dq_h, kc_h, vc_h, table_h, lens_h = make_decode(dcase)
    q, k, v = q_h.to(dev), k_h.to(dev), v_h.to(dev)
    o = torch.empty_like(q)
    lse = torch.empty((pcase.B, pcase.Hq, pcase.Nq), dtype=torch.float32, device=dev)
    dq, kc, vc = dq_h.to(dev), kc_h.to(dev), vc_h.to(dev)
    table, lens = table_h.to(dev), lens_h.to(dev)
    do = torch.empty_like(dq)
    dlse = torch.empty((dcase.B, dcase.Hq), dtype=torch.float32, device=dev)
    flush = L2Flush(dev)
    stream = torch.cuda.current_stream(dev)
    sp = stream.cuda_stream
    sum_len = int(lens_h.sum())
    kv_bytes = sum_len * dcase.Hkv * dcase.D * 2 * 2
    dec_bytes = kv_bytes + dq.numel() * 2 * 2 + dlse.numel() * 4 + table_h.numel() * 4 \
        + lens_h.numel() * 4

    def prefill():
        fa.fa_fwd(q, k, v, o, lse, pcase.B, pcase.Hq, pcase.Hkv, pcase.Nq, pcase.Nk, pcase.D,
                  pcase.softmax_scale, pcase.causal, stream=sp)

    def decode():
        fa.fa_decode_paged(dq, kc, vc, table, lens, do, dcase.B, dcase.Hq, dcase.Hkv, dcase.D,
                           dcase.page_size, dcase.softmax_scale, table.shape[1], dcase.num_pages,
                           dlse, stream=sp)

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)]
          for _ in range(args.warmup + args.steps)]

    def step(i):
        flush(i & 0xff)
        ev[i][0].record(stream)
        prefill()
        ev[i][1].record(stream)
        flush((i + 1) & 0xff)
        ev[i][2].record(stream)
        decode()
        ev[i][3].record(stream)

    for i in range(args.warmup):
        step(i)
    barrier()
    sampler = ClockSampler(local)
    with sampler:
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        barrier()
        w0 = time.time()
        t0.record(stream)
        for i in range(args.warmup, args.warmup + args.steps):
            step(i)
        t1.record(stream)
        barrier()
        sampler.mark(w0, time.time())
    assert fa.device_status() == 0, fa.last_error()
    total_ms = t0.elapsed_time(t1)
    pre_ms = [ev[i][0].elapsed_time(ev[i][1]) for i in range(args.warmup, args.warmup + args.steps)]
    dec_ms = [ev[i][2].elapsed_time(ev[i][3]) for i in range(args.warmup, args.warmup + args.steps)]

    # the decode once more, outside the timed region, after a clean flush: the
    # write-only flush leaves dirty lines whose write-back lands inside each launch
    ev_c = [[torch.cuda.Event(enable_timing=True) for _ in range(2)]
            for _ in range(args.warmup + args.steps)]
    for i in range(args.warmup + args.steps):
        flush(i, clean=True)
        ev_c[i][0].record(stream)
        decode()
        ev_c[i][1].record(stream)
    torch.cuda.synchronize()
    dec_c_ms = [ev_c[i][0].elapsed_time(ev_c[i][1])
                for i in range(args.warmup, args.warmup + args.steps)]

    # ---- end to end through the C ABI with pinned host buffers
    qp, kp, vp = q_h.pin_memory(), k_h.pin_memory(), v_h.pin_memory()
    op = torch.empty(o.shape, dtype=o.dtype).pin_memory()
    lp = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()
    h2d = (qp.numel() + kp.numel() + vp.numel()) * 2
    d2h = op.numel() * 2 + lp.numel() * 4
    o_dev_ref = o.cpu()                      # the device-resident result of these inputs

    def e2e_loop(call):
        ts = []
        for i in range(args.warmup + args.steps):
            flush(i & 0xff)
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            call()
            b.record(stream)
            b.synchronize()
            if i >= args.warmup:
                ts.append(a.elapsed_time(b))
        return ts

    def serial():
        q.copy_(qp, non_blocking=True)
        k.copy_(kp, non_blocking=True)
        v.copy_(vp, non_blocking=True)
        prefill()
        op.copy_(o, non_blocking=True)
        lp.copy_(lse, non_blocking=True)

    def pipelined():
        fa.fa_fwd_host(qp, kp, vp, op, lp, q, k, v, o, lse, pcase.B, pcase.Hq, pcase.Hkv,
                       pcase.Nq, pcase.Nk, pcase.D, pcase.softmax_scale, pcase.causal, stream=sp)

    # fa_fwd_host overlaps the copies with the forward chunk by chunk; its output must
    # equal the device-resident result bit for bit, else the serial copies are timed
    e2e_mode = "fa_fwd_host (copies overlapped with the forward, chunk by chunk)"
    try:
        e2e_ms = e2e_loop(pipelined)
        if fa.device_status() != 0:
            raise RuntimeError(fa.last_error())
        if not torch.equal(op, o_dev_ref):
            raise RuntimeError("fa_fwd_host output differs from the device-resident output")
    except Exception as exc:  # reported in the line
        e2e_mode = f"serial copies around fa_fwd ({type(exc).__name__}: {exc})"[:300]
        e2e_ms = e2e_loop(serial)

    # ---- reduce over ranks (max time, summed work)
    sums = torch.tensor([sum(pre_ms), sum(dec_ms), total_ms, sum(e2e_ms)], dtype=torch.float64,
                        device=dev)
    if pg is not None:
        torch.distributed.all_reduce(sums, op=torch.distributed.ReduceOp.MAX)
    pre_max, dec_max, total_max, e2e_max = sums.tolist()
    K = args.steps
    value = world * K * pcase.flops / (pre_max * 1e-3) / 1e12
    dec_gbs = world * K * kv_bytes / (dec_max * 1e-3) / 1e9
    e2e_val = world * K * pcase.flops / (e2e_max * 1e-3) / 1e12

    peaks, peak_src = load_peaks()
    avg_pre_s = statistics.mean(pre_ms) * 1e-3
    avg_dec_s = statistics.mean(dec_ms) * 1e-3
    achieved = pcase.flops / avg_pre_s / 1e12
    dec_achieved = dec_bytes / avg_dec_s / 1e9
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": total_max / K, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": pcase.name, "decode_workload": dcase.name,
                   "B": pcase.B, "Hq": pcase.Hq, "Hkv": pcase.Hkv, "seq_len": pcase.Nq,
                   "head_dim": pcase.D, "causal": pcase.causal,
                   "decode_sum_len_per_rank": sum_len,
                   "l2": f"{FLUSH_BYTES >> 20} MiB buffer written before every launch",
                   "parallelism": f"replicas x{world} (weak scaling, no collective)"},
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"],
                     "unit": "TFLOP/s", "frac": achieved / peaks["bf16_tflops"],
                     "traffic": recorded_traffic("fa_fwd_kernel", "fa_fwd_sm100.cu"),
                     "kernel": "fa_fwd_kernel<128,bf16>", "peak_source": f"{peak_src} burst bf16",
                     "frac_of_nominal_2250": achieved / 2250.0},
        "decode": {"value": dec_gbs, "unit": "GB/s", "kv_bytes_per_step": kv_bytes,
                   "roofline": {"bound": "hbm", "achieved": dec_achieved, "peak": peaks["hbm_gbs"],
                                "unit": "GB/s", "frac": dec_achieved / peaks["hbm_gbs"],
                                "traffic": recorded_traffic("fa_decode_stream_kernel",
                                                            "fa_decode_sm100.cu"),
                                "kernel": "fa_decode_paged call: scan + stream<4> + merge",
                                "peak_source": f"{peak_src} copy bandwidth",
                                "frac_of_nominal_8000": dec_achieved / 8000.0},
                   "ms_per_launch": statistics.mean(dec_ms),
                   "after_clean_flush": {
                       "value": kv_bytes / (statistics.mean(dec_c_ms) * 1e-3) / 1e9,
                       "unit": "GB/s", "ms_per_launch": statistics.mean(dec_c_ms),
                       "frac_of_measured_copy": dec_bytes / (statistics.mean(dec_c_ms) * 1e-3)
                       / 1e9 / peaks["hbm_gbs"],
                       "l2": f"{FLUSH_BYTES >> 20} MiB written, then another "
                             f"{FLUSH_BYTES >> 20} MiB read: no input and no dirty line left"}},
        "prefill_ms_per_launch": statistics.mean(pre_ms),
        "e2e": {"value": e2e_val, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "mode": e2e_mode,
                "what": "prefill from pinned host "
                "q,k,v copied in and o,lse copied out inside the timed region"},
        # per step: fa_fwd_kernel, then fa_decode_paged's scan, stream and merge kernels
        "gpu_launches": 4 * K,
        "clocks": sampler.summary(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        tf, dt, sample = oracle_prefill_sample(heads=8)
        line["cpu_baseline"] = {"value": tf, "unit": "TFLOP/s", "cores": cpu_threads(),
                                "kind": "oracle", "sample": sample, "seconds": dt}
    if rank == 0 and world == 1 and not args.headline_only:
        # rows beyond the headline path, measured outside its timed region
        del q, k, v, o, lse, dq, kc, vc, table, lens, do, dlse
        torch.cuda.empty_cache()
        n = min(args.steps, 10)
        line["widened"] = widened_rows(fa, dev, stream, flush, args.warmup, n, peaks, peak_src)
        line["widened"].update(dense_prefill_rows(fa, dev, stream, flush, args.warmup, n, peaks,
                                                  peak_src))
        line["widened"].update(fp8_and_backward_rows(fa, dev, stream, flush, args.warmup, n,
                                                     peaks, peak_src))
    if rank == 0:
        print(json.dumps(line), flush=True)
    if pg is not None:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
