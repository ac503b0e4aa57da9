"""The debug build on the GPU: libmaglev_debug.so (MAGLEV_DEBUG=1) runs a ragged
bf16 forward + backward of the injected layer and a decode step with mixed
positions in a child process; every result must match the oracle and no
in-kernel index check may fire (device status MAGLEV_OK). Any check that did
fire would record MAGLEV_ERR_BOUNDS instead of touching memory out of range."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r'''
import os, sys
sys.path.insert(0, os.path.join(ROOT, "tests")); sys.path.insert(0, ROOT)
import numpy as np, torch
import sliding_window_recurrent_b200 as mg
assert mg.LIB_PATH.endswith("libmaglev_debug.so"), mg.LIB_PATH
import oracle, synth
from helpers import assert_close, dev, host
from sliding_window_recurrent_b200.layer import InjectedSWALayer, DecodeLayerState

wl = dict(synth.WORKLOADS["layer_bf16"]); wl.update(B=2, T=300, H=2, d=256)
B, T, H, hd, d, W = wl["B"], wl["T"], wl["H"], wl["hd"], wl["d"], 100
x = synth.layer_inputs(wl, 77)
L = InjectedSWALayer(B, T, H, hd, d, W, dtype="bf16")
g = dev(x["gates"])
L.forward(dev(x["q"]), dev(x["k"]), dev(x["v"]), g, dev(x["m_shift"]), dev(x["w_mk"]), dev(x["w_mv"]))
L.backward(dev(x["k"]), dev(x["v"]), dev(x["dout"]), g, dev(x["m_shift"]), dev(x["w_mk"]), dev(x["w_mv"]))
torch.cuda.synchronize()
Rk, Rv = oracle.mem_project(x["m_shift"].f64, x["w_mk"].f64, x["w_mv"].f64)
f = oracle.inject_swa_forward(x["q"].f64, x["k"].f64, x["v"].f64, Rk, Rv, x["gates"].astype(np.float64), W)
bw = oracle.inject_swa_backward(x["q"].f64, x["k"].f64, x["v"].f64, Rk, Rv, x["gates"].astype(np.float64),
                                x["dout"].f64, W)
assert_close(host(L.out), f["out"], "bf16", "out")
for name in ("dq", "dk", "dv"):
    assert_close(host(getattr(L, name)), bw[name], "bf16", name)

Bd, Hd, D = 8, 2, 256
desc_pos = [-1, 0, 5, 98, 99, 100, 250, 4607]
xd = synth.decode_inputs(78, Bd, Hd, hd, D, W, desc_pos)
S = DecodeLayerState(Bd, Hd, hd, D, W, dtype="bf16")
pos = torch.tensor(desc_pos, dtype=torch.int64, device="cuda")
kr, vr = dev(xd["k_ring"]), dev(xd["v_ring"])
S.mem_project(pos, dev(xd["m_prev"]), dev(xd["w_mk"]), dev(xd["w_mv"]))
o = S.step(pos, dev(xd["q"]), dev(xd["k"]), dev(xd["v"]), dev(xd["gates"]), kr, vr)
torch.cuda.synchronize()
ok = [b for b in range(Bd) if desc_pos[b] >= 0]  # a negative position has an empty window: zero output
sub = lambda t: t.f64[ok]
pk = np.array(desc_pos)[ok]
krec, vrec = oracle.decode_mem_project(pk, sub(xd["m_prev"]), xd["w_mk"].f64, xd["w_mv"].f64, Hd)
od, _, _ = oracle.decode_step(pk, sub(xd["q"]), sub(xd["k"]), sub(xd["v"]), krec, vrec,
                              xd["gates"].astype(np.float64), sub(xd["k_ring"]), sub(xd["v_ring"]))
got = host(o)
assert_close(got[ok], od, "bf16", "decode out")
assert np.all(got[[b for b in range(Bd) if desc_pos[b] < 0]] == 0)
code = mg.maglev_device_status()
assert code == mg.MAGLEV_OK, code
print("DEBUG-BUILD-OK")
'''


def test_debug_build_runs_clean_and_matches_the_oracle():
    from sliding_window_recurrent_b200 import build as _build
    _build.build(quiet=True, debug=True)
    env = dict(os.environ, MAGLEV_DEBUG="1")
    r = subprocess.run([sys.executable, "-c", f"ROOT = {ROOT!r}\n" + CHILD], env=env, capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0 and "DEBUG-BUILD-OK" in r.stdout, r.stdout[-3000:] + r.stderr[-3000:]
