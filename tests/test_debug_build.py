"""The FA_DEBUG build of the library (every tensor-memory load, store and wait
checks first that its warp is converged, and flags a diverged warp in the
device error word instead of hanging on it).

CPU: the debug build compiles for sm_100a and exports exactly the release
library's entry points, all of them declared in include/fa.h.
GPU: the forward, backward and FP8 kernels of the debug build, loaded through
FA_LIBRARY in a fresh process, match the oracle and leave the error word clear
(no access found a diverged warp).
"""
import os
import subprocess
import sys

import pytest

from exact_tiled_attention_40_b200 import build, fa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def exported(path):
    out = subprocess.run(["nm", "-D", "--defined-only", path], check=True, capture_output=True,
                         text=True).stdout
    return sorted({line.split()[-1] for line in out.splitlines()
                   if line.split() and line.split()[-1].startswith("fa_")})


@pytest.fixture(scope="module")
def debug_lib():
    return build.build(debug=True)


def test_debug_build_exports_the_release_abi(debug_lib):
    release = build.build()
    assert exported(debug_lib) == exported(release)
    assert set(fa.header_symbols()) <= set(exported(debug_lib))


def test_debug_build_loads_and_validates_without_a_gpu(debug_lib):
    code = ("from exact_tiled_attention_40_b200 import fa; l = fa.lib(); "
            "assert fa.LIB_PATH.endswith('debug/libfa_sm100.so'); "
            "assert l.fa_version() == 100; "
            "rc = l.fa_fwd(None, None, None, None, None, 1, 2, 2, 8, 8, 96, 0.1, 0, None); "
            "assert rc == 2, rc")                              # head dim 96: FA_ERR_UNSUPPORTED
    env = dict(os.environ, FA_LIBRARY=debug_lib)
    subprocess.run([sys.executable, "-c", code], check=True, cwd=ROOT, env=env, timeout=120)


GPU_SCRIPT = r"""
import numpy as np, torch, oracle
from exact_tiled_attention_40_b200 import fa
from exact_tiled_attention_40_b200.inputs import PrefillCase, make_prefill, make_dout
assert fa.LIB_PATH.endswith("debug/libfa_sm100.so")
dev = torch.device("cuda", 0)
f64 = lambda t: t.float().double().numpy()
for case in (PrefillCase("dbg_causal", 1, 4, 2, 300, 300, 128, seed=41, causal=True),
             PrefillCase("dbg_plain", 2, 2, 1, 200, 333, 64, seed=42)):
    q, k, v, gen = make_prefill(case)
    o, lse = fa.attention(q.to(dev), k.to(dev), v.to(dev), case.softmax_scale, case.causal)
    torch.cuda.synchronize()
    assert fa.device_status() == 0, fa.last_error()
    O, L = oracle.attention(f64(q), f64(k), f64(v), case.softmax_scale, case.causal)
    assert np.abs(f64(o.cpu()) - O).max() <= 2e-2 and np.abs(lse.cpu().double().numpy() - L).max() <= 1e-3
    do = make_dout(case, gen)
    dq, dk, dv = fa.attention_backward(q.to(dev), k.to(dev), v.to(dev), o, lse, do.to(dev),
                                       case.softmax_scale, case.causal)
    torch.cuda.synchronize()
    assert fa.device_status() == 0, fa.last_error()
    ref = oracle.attention_backward(f64(q), f64(k), f64(v), f64(o.cpu()), lse.cpu().double().numpy(),
                                    f64(do), case.softmax_scale, case.causal)
    for got, want in zip((dq, dk, dv), ref):
        assert np.abs(f64(got.cpu()) - want).max() <= 0.1 * max(1.0, np.abs(want).max())
case = PrefillCase("dbg_fp8", 1, 4, 2, 260, 260, 128, seed=43, causal=True)
q, k, v, _ = make_prefill(case)
o8, l8 = fa.attention_fp8(q.to(dev), k.to(dev), v.to(dev), case.softmax_scale, True)
torch.cuda.synchronize()
assert fa.device_status() == 0, fa.last_error()
O, L = oracle.attention(f64(q), f64(k), f64(v), case.softmax_scale, True)
assert np.abs(f64(o8.cpu()) - O).max() <= 0.25
print("debug build: forward, backward and FP8 kernels clean")
"""


@pytest.mark.gpu
def test_debug_build_kernels_find_no_diverged_warp(cuda_device, debug_lib):
    env = dict(os.environ, FA_LIBRARY=debug_lib)
    r = subprocess.run([sys.executable, "-c", GPU_SCRIPT], cwd=ROOT, env=env, timeout=600,
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
