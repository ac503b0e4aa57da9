"""The bounded-wait failure path, exercised without faulting the GPU.

Every wait of the tensor-core kernels on an mbarrier gives up after
desc.spin_limit microseconds of GPU time: the waiting role raises its CTA's
abort flag and records MAGLEV_ERR_TIMEOUT in the device status word; every
role then stops issuing work, drains the copies and MMAs it has in flight,
frees its tensor memory and returns. Here the forward of the full d20 layer
runs with a 1 microsecond limit, far below the latency of its first TMA loads,
so waits expire in every CTA; the call must return promptly with the status
word set, and the next normal call must be correct.
"""
import time

import numpy as np
import pytest

import oracle
import synth
from helpers import assert_close, dev, host

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from sliding_window_recurrent_b200 import build as _build
    _build.build(quiet=True)
    import sliding_window_recurrent_b200 as mg
    from sliding_window_recurrent_b200.layer import InjectedSWALayer


def _layer(wl, spin_limit):
    return InjectedSWALayer(wl["B"], wl["T"], wl["H"], wl["hd"], wl["d"], wl["W"], dtype="bf16",
                            spin_limit=spin_limit)


def test_expired_waits_set_the_status_and_the_context_recovers():
    assert mg.maglev_device_status() == mg.MAGLEV_OK
    wl = dict(synth.WORKLOADS["layer_bf16"])
    x = synth.layer_inputs(wl, 3)
    args = [dev(x[n]) for n in ("q", "k", "v", "gates", "m_shift", "w_mk", "w_mv")]
    L = _layer(wl, spin_limit=1)
    t0 = time.perf_counter()
    L.forward(*args)
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert mg.maglev_device_status() == mg.MAGLEV_ERR_TIMEOUT
    assert elapsed < 20.0, elapsed           # each drain is itself bounded (2 s)
    assert mg.maglev_device_status() == mg.MAGLEV_OK  # reading the word cleared it

    # the context is intact: a normal call on a small case matches the oracle
    small = dict(wl, B=1, T=300, H=2, d=256, W=100)
    xs = synth.layer_inputs(small, 4)
    L2 = _layer(small, spin_limit=0)
    L2.forward(*[dev(xs[n]) for n in ("q", "k", "v", "gates", "m_shift", "w_mk", "w_mv")])
    torch.cuda.synchronize()
    Rk, Rv = oracle.mem_project(xs["m_shift"].f64, xs["w_mk"].f64, xs["w_mv"].f64)
    f = oracle.inject_swa_forward(xs["q"].f64, xs["k"].f64, xs["v"].f64, Rk, Rv, xs["gates"].astype(np.float64),
                                  small["W"])
    assert_close(host(L2.out), f["out"], "bf16", "out after recovery")
    assert mg.maglev_device_status() == mg.MAGLEV_OK
