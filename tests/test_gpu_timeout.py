"""The bounded-wait failure path, exercised without faulting the GPU.

Every wait of the tensor-core kernels on an mbarrier gives up after
desc.spin_limit microseconds of GPU time: the waiting role raises its CTA's
abort flag and records MAGLEV_ERR_TIMEOUT in the device status word; every
role then stops issuing work, drains the copies and MMAs it has in flight,
frees its tensor memory and returns. maglev_wait_selftest runs that path to
expiry on a wait that nothing completes; the full forward then runs with a 1
microsecond limit; after each, the next normal call must be correct.
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


def _check_small_forward():
    """A normal call on a small case matches the oracle: the context is intact."""
    wl = dict(synth.WORKLOADS["layer_bf16"], B=1, T=300, H=2, d=256, W=100)
    xs = synth.layer_inputs(wl, 4)
    L2 = _layer(wl, spin_limit=0)
    L2.forward(*[dev(xs[n]) for n in ("q", "k", "v", "gates", "m_shift", "w_mk", "w_mv")])
    torch.cuda.synchronize()
    Rk, Rv = oracle.mem_project(xs["m_shift"].f64, xs["w_mk"].f64, xs["w_mv"].f64)
    f = oracle.inject_swa_forward(xs["q"].f64, xs["k"].f64, xs["v"].f64, Rk, Rv, xs["gates"].astype(np.float64),
                                  wl["W"])
    assert_close(host(L2.out), f["out"], "bf16", "out after recovery")
    assert mg.maglev_device_status() == mg.MAGLEV_OK


def test_expired_wait_sets_the_status_and_the_context_recovers():
    """A wait on an mbarrier that nothing completes, with a bulk copy in
    flight and tensor memory held (maglev_wait_selftest): it must give up after
    its limit, record MAGLEV_ERR_TIMEOUT, drain, free and return."""
    assert mg.maglev_device_status() == mg.MAGLEV_OK
    src = torch.arange(1024, dtype=torch.float32, device="cuda")
    for limit_us in (1, 2000):
        t0 = time.perf_counter()
        mg.maglev_wait_selftest(src, 4096, limit_us)
        torch.cuda.synchronize()
        elapsed = time.perf_counter() - t0
        assert mg.maglev_device_status() == mg.MAGLEV_ERR_TIMEOUT, limit_us
        assert elapsed < 5.0, elapsed
        assert mg.maglev_device_status() == mg.MAGLEV_OK  # reading the word cleared it
    _check_small_forward()


def test_short_limit_on_the_full_forward_returns():
    """The full d20 layer forward with a 1 microsecond bound on every wait: each
    wait that outlives it aborts its CTA (whether one does depends on timing, so
    the status may read either way); the call must return promptly and the
    next normal call must be correct."""
    assert mg.maglev_device_status() == mg.MAGLEV_OK
    wl = dict(synth.WORKLOADS["layer_bf16"])
    x = synth.layer_inputs(wl, 3)
    args = [dev(x[n]) for n in ("q", "k", "v", "gates", "m_shift", "w_mk", "w_mv")]
    L = _layer(wl, spin_limit=1)
    t0 = time.perf_counter()
    L.forward(*args)
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert mg.maglev_device_status() in (mg.MAGLEV_OK, mg.MAGLEV_ERR_TIMEOUT)
    assert elapsed < 20.0, elapsed           # each drain is itself bounded (2 s)
    _check_small_forward()
