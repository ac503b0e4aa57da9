"""The scratch-free consistency loss (maglev_consistency_loss_noalloc).

Some callers cannot allocate device memory -- a plugin or custom-op interface
that passes only its input and output tensors, or a latency-critical loop in
which cudaMalloc (which may synchronise the device) is not allowed. For them
the library keeps the loss's partial sums in a file-scope device array. This
test calls that entry point through the C ABI and checks it against the
workspace-taking maglev_consistency_loss and against the CPU oracle on the
same inputs, for two calls in a row (a large problem, then a smaller one, so
stale partials from the first call would show), and checks that oversize
inputs are refused.

It lives in its own file, collected last, and passes both alone in a fresh
process and after the rest of the suite.
"""
import numpy as np
import pytest

import oracle
import synth
from helpers import TOL, assert_close, dev, host

torch = pytest.importorskip("torch")

if torch.cuda.is_available():
    from sliding_window_recurrent_b200 import build as _build
    _build.build(quiet=True)
    import sliding_window_recurrent_b200 as mg


def _reference(m, t, rows, d, code, lam, accumulate, dm0):
    td = m.dtype
    loss = torch.zeros((), device="cuda")
    dm = dm0.clone()
    dmt = torch.empty(rows, d, dtype=td, device="cuda")
    ws = torch.empty(mg.maglev_consistency_workspace_bytes(rows, d), dtype=torch.uint8, device="cuda")
    mg.maglev_consistency_loss(m, t, rows, d, code, lam, 0.0, loss, dm, dmt, accumulate, ws)
    return loss, dm, dmt


def _noalloc(m, t, rows, d, code, lam, accumulate, dm0):
    loss = torch.full((), -1.0, device="cuda")
    dm = dm0.clone()
    dmt = torch.empty(rows, d, dtype=m.dtype, device="cuda")
    mg.maglev_consistency_loss_noalloc(m, t, rows, d, code, lam, 0.0, loss, dm, dmt, accumulate)
    return loss, dm, dmt


@pytest.mark.gpu
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_noalloc_matches_workspace_entry_point_twice(dtype):
    code = mg.MAGLEV_BF16 if dtype == "bf16" else mg.MAGLEV_F32
    lam = 0.1
    for call, (rows, d, accumulate) in enumerate([(8192, 1280, 1), (37, 96, 0)]):
        m = dev(synth.normal(31 + call, 1, (rows, d), dtype=dtype))
        t = dev(synth.normal(31 + call, 2, (rows, d), dtype=dtype))
        dm0 = dev(synth.normal(31 + call, 3, (rows, d), dtype=dtype))
        ref = _reference(m, t, rows, d, code, lam, accumulate, dm0)
        got = _noalloc(m, t, rows, d, code, lam, accumulate, dm0)
        torch.cuda.synchronize()
        r_loss, g_loss = float(ref[0].item()), float(got[0].item())
        assert abs(g_loss - r_loss) <= 1e-5 * abs(r_loss), (call, g_loss, r_loss)
        assert_close(host(got[1]), host(ref[1]), dtype, f"dm call {call}")
        assert_close(host(got[2]), host(ref[2]), dtype, f"dm_target call {call}")
        # and directly against the CPU oracle of the loss
        o_loss, o_dm, o_dmt = oracle.consistency_loss(host(m), host(t), lam)
        if accumulate:
            o_dm = o_dm + host(dm0)
        assert abs(g_loss - o_loss) <= 1e-5 * abs(o_loss), (call, g_loss, o_loss)
        assert_close(host(got[1]), o_dm, dtype, f"dm vs oracle, call {call}")
        assert_close(host(got[2]), o_dmt, dtype, f"dm_target vs oracle, call {call}")
    assert TOL[dtype] > 0


@pytest.mark.gpu
def test_noalloc_rejects_oversize_inputs():
    loss = torch.zeros((), device="cuda")
    fake = 1 << 20  # never dereferenced: the size check fails first
    with pytest.raises(mg.MaglevError) as e:
        mg.maglev_consistency_loss_noalloc(fake, fake, 65536, 1025, mg.MAGLEV_BF16, 0.1, 0.0,
                                           loss, None, None, 0)
    assert e.value.status == mg.MAGLEV_ERR_UNSUPPORTED
    assert "67108864" in str(e.value)
    np.testing.assert_equal(float(loss.item()), 0.0)
