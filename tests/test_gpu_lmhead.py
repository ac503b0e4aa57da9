"""GPU parity of the softcapped LM head with cross-entropy (maglev_lm_head_ce)
against the CPU fp64 oracle, through the C ABI.

paper.rainbus.top, 方法步骤详情: the memory state m_t feeds the LM head
p(x_{t+1} | x_<=t) = softmax(15 tanh(U m_t / 15)), and the loss averages the
per-token cross-entropy over the positions in I. The pages give no vocabulary
size; 65,536 (2^16) stands in for the d20 model's. U is drawn with std
4/sqrt(d), so that raw logits reach the cap's bend (|z| ~ 4 sigma ~ 16).
"""
import numpy as np
import pytest

import oracle
import synth
from helpers import TOL, assert_close, dev, host

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from sliding_window_recurrent_b200 import build as _build
    _build.build(quiet=True)
    import sliding_window_recurrent_b200 as mg


def _inputs(seed, N, d, V):
    m = synth.normal(seed, synth.TID["h0"], (N, d))
    U = synth.normal(seed, synth.TID["w_qkv"], (V, d), std=4.0 / np.sqrt(d))
    y = (synth.uniform(seed, synth.TID["pos"], (N,), 0.0, 1.0) * V).astype(np.int64)
    return m, U, np.minimum(y, V - 1)


def _gpu(m, U, y, N, d, V):
    loss = torch.zeros((), device="cuda")
    lse = torch.empty(N, device="cuda")
    dm = torch.empty(N, d, dtype=torch.bfloat16, device="cuda")
    dU = torch.empty(V, d, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(mg.maglev_lm_head_workspace_bytes(N, d, V), dtype=torch.uint8, device="cuda")
    mg.maglev_lm_head_ce(N, d, V, mg.MAGLEV_BF16, 15.0, 0.0, dev(m), dev(U), torch.from_numpy(y).cuda(), loss, lse,
                         dm, dU, ws)
    torch.cuda.synchronize()
    return float(loss.item()), host(lse), host(dm), host(dU)


def _oracle_blocks(m, U, y, rows_per_block=256):
    """The oracle over row blocks: the loss and dU are sums over rows, lse and dm
    are per row, so the blocks (each with the whole batch's 1/N) compose."""
    N = m.shape[0]
    loss, lse, dm, dU = 0.0, [], [], 0.0
    for a in range(0, N, rows_per_block):
        b = min(N, a + rows_per_block)
        l, e, g, h = oracle.lm_head_ce(m[a:b], U, y[a:b], inv_count=1.0 / N)
        loss += l
        lse.append(e)
        dm.append(g)
        dU = dU + h
    return loss, np.concatenate(lse), np.concatenate(dm), dU


@pytest.mark.parametrize("N,d,V", [(300, 200, 4000), (1, 64, 8), (129, 1280, 2056)])
def test_lm_head_ragged(N, d, V):
    """Ragged row tiles, a K extent that is not a multiple of 64 and a vocabulary
    that is not a multiple of the 256-column tile."""
    m, U, y = _inputs(5, N, d, V)
    g = _gpu(m, U, y, N, d, V)
    r = oracle.lm_head_ce(m.f64, U.f64, y)
    assert abs(g[0] - r[0]) <= 1e-3 * abs(r[0]), (g[0], r[0])
    assert_close(g[1], r[1], "bf16", "lse")
    assert_close(g[2], r[2], "bf16", "dm")
    assert_close(g[3], r[3], "bf16", "dU")


def test_lm_head_full_size():
    """N = B*T = 8192 tokens of the d20 layer, d = 1280, V = 65,536."""
    N, d, V = 8192, 1280, 65536
    m, U, y = _inputs(6, N, d, V)
    g = _gpu(m, U, y, N, d, V)
    r = _oracle_blocks(m.f64, U.f64, y)
    assert abs(g[0] - r[0]) <= 1e-3 * abs(r[0]), (g[0], r[0])
    assert_close(g[1], r[1], "bf16", "lse", "elementwise")
    assert_close(g[2], r[2], "bf16", "dm")
    assert_close(g[3], r[3], "bf16", "dU")


def test_lm_head_uniform_when_weights_vanish():
    """U = 0: every capped logit is 0, so LSE = log V and the loss is log V
    exactly as in the oracle's closed form; dm = 0."""
    N, d, V = 256, 128, 1024
    m, _, y = _inputs(7, N, d, V)
    U0 = synth.Tensor(np.zeros((V, d), np.uint16), "bf16")
    loss, lse, dm, _ = _gpu(m, U0, y, N, d, V)
    np.testing.assert_allclose(lse, np.log(V), rtol=1e-6)
    assert abs(loss - np.log(V)) <= 1e-5 * np.log(V)
    assert np.all(dm == 0)
