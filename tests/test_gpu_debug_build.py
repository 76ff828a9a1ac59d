"""The bounds-checked build (libwkv_debug.so, -DWKV_DEBUG) on the GPU.

Its kernels check the indices of their stores and workspace accesses; an index
outside its array would set a status bit (WKV_ERR_BOUNDS from
wkv_query_status) and skip the access instead of faulting. Here every kernel
of the library runs small ragged cases under it, in a child process that loads
the debug library: every call must report a clean status word and agree with
the float64 oracle. This is the stand-in for a memory checker on this machine.
"""
import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r'''
import numpy as np, torch, sys
sys.path.insert(0, "tests")
import wkv_recurrence_b200 as W
from wkv_recurrence_b200 import _abi, inputs as I
from oracle import oracle as O, v6_oracle as V
from parity_util import assert_out, assert_state, dev_f32, host
assert _abi.LIB_PATH.endswith("libwkv_debug.so"), _abi.LIB_PATH
checked = 0
for kernel in (1, 2, 3, 4, 5):
    for (B, T, C) in ((2, 517, 200), (3, 1000, 96), (1, 65, 36)):
        k, v, w, u, st = I.random_case(B, T, C, seed=T + kernel, k_spike=30.0, state=True)
        opts = {"kernel": kernel}
        ws = W.make_workspace(B, T, C, options=opts)
        for ext in (None, "wt", "r"):
            if ext == "wt" and kernel in (2, 4):
                continue
            wt = np.exp(np.random.default_rng(T).normal(-1, 1, k.shape)).astype(np.float32) if ext == "wt" else None
            r = np.random.default_rng(T + 1).normal(0, 1, k.shape).astype(np.float32) if ext == "r" else None
            out, so = W.forward(dev_f32(k), dev_f32(v), dev_f32(w), dev_f32(u), tuple(dev_f32(s) for s in st),
                                workspace=ws, options=opts, w_t=None if wt is None else dev_f32(wt),
                                r=None if r is None else dev_f32(r))
            code = W.query_status(ws)
            assert code == 0, (kernel, B, T, C, ext, code)
            ref, rst = O.recurrence_forward(k, v, w, u, st, w_t=wt, r=r)
            sc, sst = O.abs_scale_forward(k, v, w, u, st, w_t=wt, r=r)
            assert_out(host(out), ref, sc, 1e-5)
            assert_state(tuple(host(x) for x in so), rst, sst[0], 1e-5)
            checked += 1
# backward
k, v, w, u, st = I.random_case(2, 300, 96, seed=5, k_spike=20.0, state=True)
g = np.random.default_rng(5).normal(size=k.shape).astype(np.float32)
ws = torch.empty(W.api._abi.lib().wkv_backward_workspace_size(2, 300, 96), dtype=torch.uint8, device="cuda")
ws[:256].zero_()
dk, dv, dw, du, ds = W.backward(dev_f32(k), dev_f32(v), dev_f32(w), dev_f32(u), dev_f32(g),
                                tuple(dev_f32(s) for s in st), workspace=ws)
assert W.query_status(ws) == 0
ref, sc = O.recurrence_backward(k, v, w, u, g, st)
assert np.all(np.abs(host(dk) - ref["dk"]) <= 1e-5 * sc["dk"] + 1e-30)
checked += 1
# v6
g6 = np.random.default_rng(6)
r6, k6, v6 = (g6.normal(0, 1, (2, 70, 3, 64)).astype(np.float32) for _ in range(3))
w6 = np.exp(-np.exp(g6.normal(-1, 1, (2, 70, 3, 64)))).astype(np.float32)
ws6 = torch.zeros(256, dtype=torch.uint8, device="cuda")
y, _ = W.v6_forward(dev_f32(r6), dev_f32(w6), dev_f32(k6), dev_f32(v6), workspace=ws6)
assert W.query_status(ws6) == 0
yr, _ = V.recurrence(r6, w6, k6, v6)
ys, _ = V.abs_scale(r6, w6, k6, v6)
assert_out(host(y), yr, ys, 1e-5)
checked += 1
print("checked", checked)
'''


def test_bounds_checked_build_reports_clean_status_and_matches_oracle():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from wkv_recurrence_b200 import build
    build.build(debug=True)
    env = dict(os.environ, WKV_LIBRARY="debug", PYTHONPATH=ROOT)
    r = subprocess.run([sys.executable, "-c", CHILD], cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
    assert "checked" in r.stdout
