"""Parity of the prefiller + decoder stack (Q -> memory -> P -> loss) with the oracle.

The stack runs every layer through the C ABI (sliding_window_recurrent_b200.stack)
and is compared, tensor by tensor, with oracle.stack_forward_backward on the
same seeded inputs. The combined upstream gradient of each last layer is held
in the activation type on the GPU; the oracle is told to round it the same way.
"""
import numpy as np
import pytest

import oracle
import synth
from tests.helpers import TOL, assert_close, dev, host

pytestmark = pytest.mark.gpu


def _bf16(x):
    return synth.bf16_bits_to_f64(synth.round_to_bf16_bits(np.asarray(x, dtype=np.float32)))


def _zero_last_dout(x):
    """Zero the upstream gradient of each stack's last layer, so that the
    memory's gradient (the consistency loss through RMSNorm, plus the shifted
    projection gradient on Q's side) is all that drives those layers."""
    for key in ("q_layers", "p_layers"):
        L = x[key][-1]
        L["dout"] = synth.Tensor(np.zeros_like(L["dout"].bits), L["dout"].dtype)


def _run(wl, seed, q_windows, p_windows, zero_last_dout=False, per_layer_wrec=False, shared_kv_gates=False):
    import torch
    from sliding_window_recurrent_b200.stack import PrefillerDecoderStack

    x = synth.stack_inputs(wl, seed, q_windows, p_windows, per_layer_wrec, shared_kv_gates)
    if zero_last_dout:
        _zero_last_dout(x)
    B, T, H, hd = wl["B"], wl["T"], wl["H"], wl["hd"]
    S = PrefillerDecoderStack(B, T, H, hd, q_windows, p_windows, lam=wl["lam"], dtype=wl["dtype"],
                              per_layer_wrec=per_layer_wrec, shared_kv_gates=shared_kv_gates)
    qi = [(dev(L["q"]), dev(L["k"]), dev(L["v"])) for L in x["q_layers"]]
    pi = [(dev(L["q"]), dev(L["k"]), dev(L["v"]), dev(L["gates"])) for L in x["p_layers"]]
    qd = [dev(L["dout"]) for L in x["q_layers"]]
    pd = [dev(L["dout"]) for L in x["p_layers"]]
    if per_layer_wrec:
        wk = torch.stack([dev(L["w_mk"]) for L in x["p_layers"]])
        wv = torch.stack([dev(L["w_mv"]) for L in x["p_layers"]])
    else:
        wk, wv = dev(x["w_mk"]), dev(x["w_mv"])
    S.step(qi, pi, qd, pd, wk, wv)
    torch.cuda.synchronize()

    f64 = lambda L, keys: {k: (L[k].f64 if isinstance(L[k], synth.Tensor) else L[k]) for k in keys}
    ql = [dict(f64(L, ("q", "k", "v", "dout")), window=L["window"]) for L in x["q_layers"]]
    pkeys = ("q", "k", "v", "dout") + (("w_mk", "w_mv") if per_layer_wrec else ())
    pl = [dict(f64(L, pkeys), gates=L["gates"].astype(np.float64), window=L["window"]) for L in x["p_layers"]]
    store = _bf16 if wl["dtype"] == "bf16" else None
    w = (None, None) if per_layer_wrec else (x["w_mk"].f64, x["w_mv"].f64)
    ref = oracle.stack_forward_backward(ql, pl, w[0], w[1], wl["lam"], store=store)
    return S, ref


def _check_all(S, ref, dt):
    B, T, H, hd = S.B, S.T, S.H, S.hd
    for i, L in enumerate(S.q):
        assert_close(host(L.out), ref["q_out"][i], dt, f"Q{i} out")
        for g in ("dq", "dk", "dv"):
            assert_close(host(getattr(L, g)), ref["q_grads"][i][g], dt, f"Q{i} {g}")
    for i, L in enumerate(S.p):
        assert_close(host(L.out), ref["p_out"][i], dt, f"P{i} out")
        for g in ("dq", "dk", "dv"):
            assert_close(host(getattr(L, g)), ref["p_grads"][i][g], dt, f"P{i} {g}")
        assert_close(host(L.dgate), ref["p_grads"][i]["dgate"], dt, f"P{i} dgate", "scaled",
                     ref["p_grads"][i]["dgate_scale"])
    assert_close(host(S.m_prime), ref["m_prime"], dt, "m'")
    assert_close(host(S.m_shift), ref["m_shift"], dt, "m_shift")
    assert np.all(host(S.m_shift)[:, 0] == 0), "row 0 of the shifted memory is m'_0 = 0"
    assert_close(host(S.m), ref["m"], dt, "m")
    assert abs(float(S.loss.item()) - ref["loss"]) <= TOL[dt] * abs(ref["loss"]), (float(S.loss.item()), ref["loss"])
    assert_close(host(S.dm_shift), ref["dm_shift"], dt, "dm_shift")
    if S.per_layer_wrec:
        for i, g in enumerate(ref["p_grads"]):
            for n in ("dR_k", "dR_v"):
                assert_close(host(getattr(S, n)[i]), g[n].reshape(B, T, -1), dt, f"P{i} {n}")
            for n in ("dw_mk", "dw_mv"):
                assert_close(host(getattr(S, n)[i]), g[n], dt, f"P{i} {n}")
    else:
        assert_close(host(S.dR_k), ref["dR_k"], dt, "dR_k")
        assert_close(host(S.dR_v), ref["dR_v"], dt, "dR_v")
        assert_close(host(S.dw_mk), ref["dw_mk"], dt, "dW_mk")
        assert_close(host(S.dw_mv), ref["dw_mv"], dt, "dW_mv")


@pytest.mark.parametrize("T", [200, 129])
def test_stack_bf16_small(T):
    """SLSL prefiller (window 64 and full causal) and a 3-layer injected decoder,
    ragged T, two heads of 128 (the tensor-core path)."""
    wl = dict(B=2, T=T, H=2, hd=128, dtype="bf16", lam=0.1)
    S, ref = _run(wl, 1234, [64, T, 64, T], [64, 64, 64])
    _check_all(S, ref, "bf16")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_stack_loss_gradient_drives_last_layers(dtype):
    """Each stack's last layer gets no upstream gradient of its own: P's last
    layer is driven by the consistency loss alone (through RMSNorm), Q's last
    layer by the loss's m' term plus the shifted projection gradient. With
    lambda = 10 and |I| = B*T = 300 the gradients of P's last layer are ~1e-2
    of the other layers' (bf16 keeps their full relative precision), so a
    wrong memory-state backward shows in that layer's dq, dk, dv and gate
    gradients."""
    hd = 128 if dtype == "bf16" else 64
    wl = dict(B=2, T=150, H=2, hd=hd, dtype=dtype, lam=10.0)
    S, ref = _run(wl, 1237, [48, 150], [48, 48, 48], zero_last_dout=True)
    g = ref["p_grads"][-1]
    assert 0 < np.abs(g["dq"]).max() < 0.1, "P's last layer sees only the small loss gradient"
    _check_all(S, ref, dtype)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("per_layer_wrec,shared_kv_gates", [(True, False), (False, True), (True, True)])
def test_stack_variants(dtype, per_layer_wrec, shared_kv_gates):
    """The decoder with one W^rec per layer (dm_shift summed over the layers'
    projections in one fp32 accumulation) and/or gates shared by K and V."""
    hd = 128 if dtype == "bf16" else 64
    wl = dict(B=2, T=170, H=2, hd=hd, dtype=dtype, lam=0.5)
    S, ref = _run(wl, 1239, [64, 170], [64, 64, 64], per_layer_wrec=per_layer_wrec,
                  shared_kv_gates=shared_kv_gates)
    _check_all(S, ref, dtype)


def test_stack_f32_small():
    """The same stack on the fp32 path (CUDA cores), head dim 64."""
    wl = dict(B=1, T=150, H=2, hd=64, dtype="f32", lam=1.0)
    S, ref = _run(wl, 1235, [32, 150], [32, 32])
    _check_all(S, ref, "f32")


def _slice_b0(L):
    out = {}
    for k, v in L.items():
        if isinstance(v, synth.Tensor):
            out[k] = v.f64[:1]
        elif k == "gates":
            out[k] = v.astype(np.float64)
        else:
            out[k] = v
    return out


def test_stack_full_size_batch_row_0():
    """Every launch at the benchmark's shape (B=8, T=2048, 10 heads of 128,
    windows 512 and full 2048): a 2-layer SL prefiller and a 2-layer decoder.
    Batch row 0 of every output and gradient is compared with the oracle run
    on that row alone, with the loss's |I| of the whole batch."""
    import torch
    from sliding_window_recurrent_b200.stack import PrefillerDecoderStack

    wl = dict(synth.WORKLOADS["stack20_bf16"])
    B, T, H, hd = wl["B"], wl["T"], wl["H"], wl["hd"]
    q_windows, p_windows = [512, T], [512, 512]
    x = synth.stack_inputs(wl, 1234, q_windows, p_windows)
    S = PrefillerDecoderStack(B, T, H, hd, q_windows, p_windows, lam=wl["lam"])
    qi = [(dev(L["q"]), dev(L["k"]), dev(L["v"])) for L in x["q_layers"]]
    pi = [(dev(L["q"]), dev(L["k"]), dev(L["v"]), dev(L["gates"])) for L in x["p_layers"]]
    qd = [dev(L["dout"]) for L in x["q_layers"]]
    pd = [dev(L["dout"]) for L in x["p_layers"]]
    S.step(qi, pi, qd, pd, dev(x["w_mk"]), dev(x["w_mv"]))
    torch.cuda.synchronize()

    ref = oracle.stack_forward_backward([_slice_b0(L) for L in x["q_layers"]],
                                        [_slice_b0(L) for L in x["p_layers"]],
                                        x["w_mk"].f64, x["w_mv"].f64, wl["lam"], store=_bf16,
                                        inv_count=1.0 / (B * T))
    h0 = lambda t: host(t[:1])
    for i, L in enumerate(S.q):
        assert_close(h0(L.out), ref["q_out"][i], "bf16", f"Q{i} out")
        for g in ("dq", "dk", "dv"):
            assert_close(h0(getattr(L, g)), ref["q_grads"][i][g], "bf16", f"Q{i} {g}")
    for i, L in enumerate(S.p):
        assert_close(h0(L.out), ref["p_out"][i], "bf16", f"P{i} out")
        for g in ("dq", "dk", "dv"):
            assert_close(h0(getattr(L, g)), ref["p_grads"][i][g], "bf16", f"P{i} {g}")
    assert_close(h0(S.m_prime), ref["m_prime"], "bf16", "m'")
    assert_close(h0(S.m), ref["m"], "bf16", "m")
    assert_close(h0(S.dm_shift), ref["dm_shift"], "bf16", "dm_shift")
    assert_close(h0(S.dR_k), ref["dR_k"], "bf16", "dR_k")
    assert_close(h0(S.dR_v), ref["dR_v"], "bf16", "dR_v")


def test_stack_twenty_decoder_layers():
    """The decoder depth of the benchmark: 20 injected layers (W = 512) sharing
    one projection, so dL/dR is a sum of 20 layers' shares, kept in fp32 and
    rounded once; an SL prefiller (W = 512, full 2048). One batch row of the
    full shape (T = 2048, 10 heads of 128): every P layer, dR, dm_shift, dW."""
    wl = dict(B=1, T=2048, H=10, hd=128, dtype="bf16", lam=0.1)
    S, ref = _run(wl, 1238, [512, 2048], [512] * 20)
    _check_all(S, ref, "bf16")
