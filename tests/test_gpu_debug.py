"""The debug build (libmoe_debug.so, -DMOE_DEBUG) on the GPU: on valid inputs its results match
the oracle like the release build's and its bounds checks stay silent; on a slot table that
points outside the token rows, or group offsets past the rows, its checks record device error 3
and skip the access. Runs in a child process that loads only the debug library."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r'''
import sys
import numpy as np, torch
sys.path.insert(0, ROOT)
from expert_dispatch_gate_b200 import _lib as L, layer as M, workloads as W
from tests.test_gpu_parity import SMALL, compare_layer, small_inputs
lib = L.lib()
assert L.LIB_PATH.endswith("libmoe_debug.so"), L.LIB_PATH
assert lib.moe_debug_checks() == 1  # the planted cases below rely on the checks
# valid inputs: silent checks, oracle parity
for name in ("tiny", "e8_two_token_blocks", "e256_k8", "e96_partial_tiles", "h192_i320"):
    wl, cpu, dev = small_inputs(name)
    res = M.layer_forward(dev["x"], dev["w_router"], dev["w_gate"], dev["w_up"], dev["w_down"],
                          wl.k, wl.capacity_factor, logit_bias=dev["logit_bias"])
    torch.cuda.synchronize()
    assert res["ws"].check() == L.MOE_OK, name
    compare_layer(wl, cpu, dev, res)
# a slot table that names a token row past T: the row copy records error 3 and skips it
wl, cpu, dev = small_inputs("e256_k8")
al = M.align(M.route(dev["x"], dev["w_router"], wl.k)[0], wl.E, wl.capacity_factor,
             H=wl.H, I=wl.I)
bad = al["sorted_ids"].clone()
bad[3] = wl.T * wl.k + 40
shape = M.shape_of(wl.T, wl.H, wl.E, wl.k, wl.I, wl.capacity_factor, wl.dtype)
ws = M.Workspace(shape, "cuda")
y = torch.empty((wl.T * wl.k, wl.H), dtype=dev["x"].dtype, device="cuda")
L.moe_grouped_ffn(shape, dev["x"], bad, al["offsets"], dev["w_gate"], dev["w_up"],
                  dev["w_down"], y, ws.buf, ws.nbytes)
try:
    ws.check()
    raise SystemExit("no error recorded for a bad slot table")
except L.MoeError as e:
    assert e.status == L.MOE_ERR_DEVICE and "device error 3" in str(e), str(e)
# group offsets past the rows: the expert GEMMs record error 3 and run no tile
off = al["offsets"].clone()
off[-1] = wl.T * wl.k * 4
L.moe_grouped_ffn(shape, dev["x"], al["sorted_ids"], off, dev["w_gate"], dev["w_up"],
                  dev["w_down"], y, ws.buf, ws.nbytes)
try:
    ws.check()
    raise SystemExit("no error recorded for bad group offsets")
except L.MoeError as e:
    assert e.status == L.MOE_ERR_DEVICE and "device error 3" in str(e), str(e)
# the context stays usable
assert ws.check() == L.MOE_OK
print("debug build ok")
'''


def test_debug_build_checks():
    from expert_dispatch_gate_b200 import build as B
    lib = B.build(debug=True)
    assert os.path.exists(lib)
    env = dict(os.environ, MOE_DEBUG_LIB="1")
    r = subprocess.run([sys.executable, "-c", f"ROOT = {ROOT!r}\n" + CHILD], env=env, cwd=ROOT,
                       capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
    assert "debug build ok" in r.stdout
