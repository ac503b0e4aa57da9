"""GPU parity of libmaglev against the CPU fp64 oracle, through the C ABI.

Tolerance: 1e-4 for fp32 storage, 2e-2 for bf16 storage with fp32
accumulation, on the normwise error max|gpu - ref| / max|ref| of each tensor;
LSE row by row in the log domain (an absolute error below 1, a relative one
above); each gate-gradient entry against the RMS size of the products it sums
(a sum of B*T*hd terms can cancel far below its rounding-error scale), within
helpers.GATE_TOL (derived there from an emulation of the bf16 operands). The
full-size layer test also reports the element-wise error max|gpu - ref| /
max(|ref|, rms(ref)); it is not gated, because the bf16 operands of the
attention (q_rot, k_bar and P rounded to bf16) move individual scores by ~1e-2
and the worst of 2e7 outputs by ~0.1 of the RMS (values in the design notes).
Index work (window membership, ring slots, untouched ring entries) is compared
bit-exactly.
"""
import numpy as np
import pytest

import oracle
import synth
from helpers import TOL, assert_close, dev, elementwise, host, normwise

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from sliding_window_recurrent_b200 import build as _build
    _build.build(quiet=True)
    import sliding_window_recurrent_b200 as mg
    from sliding_window_recurrent_b200.layer import DecodeLayerState, InjectedSWALayer


def wl_of(name, **over):
    wl = dict(synth.WORKLOADS[name])
    wl.update(over)
    return wl


def run_gpu(wl, x, inject=True, lam=None, bwd=True, pos0=0, fused=False):
    B, T, H, hd, d, W = wl["B"], wl["T"], wl["H"], wl["hd"], wl["d"], wl["W"]
    D = H * hd
    L = InjectedSWALayer(B, T, H, hd, d, W, dtype=wl["dtype"], inject=inject, pos0=pos0,
                         rope_base=wl["rope_base"], eps=wl["eps"])
    q, k, v = dev(x["q"]), dev(x["k"]), dev(x["v"])
    gates = dev(x["gates"]) if inject else None
    m = dev(x["m_shift"]) if inject else None
    wk = dev(x["w_mk"]) if inject else None
    wv = dev(x["w_mv"]) if inject else None
    L.forward(q, k, v, gates, m, wk, wv)
    res = {"out": host(L.out), "lse": host(L.lse)}
    if inject:
        res["R_k"], res["R_v"] = host(L.R_k), host(L.R_v)
    if bwd:
        dout = dev(x["dout"]).clone()
        if lam is not None and fused:  # the loss together with the backward's first pass
            L.consistency_prepare_bwd(dev(x["target"]), lam, dout)
            res["loss"] = float(L.loss.item())
        elif lam is not None:
            L.consistency(L.out.view(B * T, D), dev(x["target"]).view(B * T, D), lam,
                          dm=dout.view(B * T, D), accumulate_dm=True)
            res["loss"] = float(L.loss.item())
        L.backward(k, v, dout, gates, m, wk, wv, prepared=fused and lam is not None)
        res["dout_total"] = host(dout)
        res["loss_bits"] = L.loss.clone()
        for n in ("dq", "dk", "dv"):
            res[n] = host(getattr(L, n))
        if inject:
            for n in ("dR_k", "dR_v", "dgate", "dm_shift", "dw_mk", "dw_mv"):
                res[n] = host(getattr(L, n))
    torch.cuda.synchronize()
    return res


def run_oracle(wl, x, inject=True, lam=None, bwd=True, pos0=0):
    B, T, H, hd, W = wl["B"], wl["T"], wl["H"], wl["hd"], wl["W"]
    D = H * hd
    q, k, v = x["q"].f64, x["k"].f64, x["v"].f64
    gates = x["gates"].astype(np.float64)
    Rk = Rv = None
    if inject:
        Rk, Rv = oracle.mem_project(x["m_shift"].f64, x["w_mk"].f64, x["w_mv"].f64)
    f = oracle.inject_swa_forward(q, k, v, Rk, Rv, gates, W, pos0, wl["rope_base"], wl["eps"], inject)
    res = {"out": f["out"], "lse": f["lse"], "R_k": Rk, "R_v": Rv}
    if bwd:
        dout = x["dout"].f64
        if lam is not None:
            loss, dm, _ = oracle.consistency_loss(f["out"].reshape(B * T, D), x["target"].f64.reshape(B * T, D), lam)
            res["loss"] = loss
            dout = dout + dm.reshape(dout.shape)
            if wl["dtype"] == "bf16":
                # the bf16 path consumes the total upstream gradient as a bf16
                # tensor (the MMA operand type): apply that rounding here too
                dout = synth.bf16_bits_to_f64(synth.round_to_bf16_bits(dout.astype(np.float32)))
        g = oracle.inject_swa_backward(q, k, v, Rk, Rv, gates, dout, W, pos0, wl["rope_base"], wl["eps"], inject)
        res.update(dq=g["dq"], dk=g["dk"], dv=g["dv"])
        if inject:
            dms, dWk, dWv = oracle.mem_project_backward(x["m_shift"].f64, x["w_mk"].f64, x["w_mv"].f64,
                                                        g["dR_k"], g["dR_v"])
            res.update(dR_k=g["dR_k"], dR_v=g["dR_v"], dgate=g["dgate"], dgate_scale=g["dgate_scale"], dm_shift=dms,
                       dw_mk=dWk, dw_mv=dWv)
    return res


# LSE [B,H,T] is judged row by row in the log domain (floor 1); each gate
# gradient entry against the RMS size of the B*T*hd products it sums (its
# rounding-error scale, dgate_scale); every other tensor normwise.
def compare(gpu, ref, dtype, names, report_elementwise=False):
    errs = {}
    for n in names:
        if n == "lse":
            errs[n] = assert_close(gpu[n], ref[n], dtype, n, "log")
        elif n == "dgate":
            errs[n] = assert_close(gpu[n], ref[n], dtype, n, "scaled", ref["dgate_scale"])
        else:
            errs[n] = assert_close(gpu[n], ref[n], dtype, n)
            if report_elementwise:  # reported, not gated: see the module docstring
                errs[n + ":elementwise"] = elementwise(gpu[n], ref[n])
    return errs


FWD = ["out", "lse", "R_k", "R_v"]
BWD = ["dq", "dk", "dv", "dR_k", "dR_v", "dgate", "dm_shift", "dw_mk", "dw_mv"]


# --------------------------------------------------------------------------- layer parity
def test_tiny_f32_forward_backward_with_loss():
    wl = wl_of("tiny_f32")
    x = synth.layer_inputs(wl, 1234)
    g = run_gpu(wl, x, lam=wl["lam"])
    r = run_oracle(wl, x, lam=wl["lam"])
    compare(g, r, "f32", FWD + BWD)
    assert abs(g["loss"] - r["loss"]) <= 1e-4 * abs(r["loss"])


@pytest.mark.parametrize("seed", [1235, 1236])
def test_tiny_f32_other_seeds(seed):
    wl = wl_of("tiny_f32")
    x = synth.layer_inputs(wl, seed)
    compare(run_gpu(wl, x, lam=1.0), run_oracle(wl, x, lam=1.0), "f32", FWD + BWD)


@pytest.mark.parametrize("hd,T,W,pos0", [(128, 300, 100, 0), (64, 333, 47, 5), (128, 129, 1, 0),
                                         (64, 200, 512, 0), (128, 1, 8, 2)])
def test_bf16_ragged_shapes(hd, T, W, pos0):
    wl = wl_of("layer_bf16", B=2, T=T, H=3, hd=hd, d=160, W=W, target="independent")
    x = synth.layer_inputs(wl, 77)
    compare(run_gpu(wl, x, lam=0.1, pos0=pos0), run_oracle(wl, x, lam=0.1, pos0=pos0), "bf16", FWD + BWD)


def test_f32_no_injection_full_causal():
    wl = wl_of("tiny_f32", T=200, W=4096)
    x = synth.layer_inputs(wl, 5, inject=False)
    compare(run_gpu(wl, x, inject=False), run_oracle(wl, x, inject=False), "f32",
            ["out", "lse", "dq", "dk", "dv"])


def test_layer_bf16_full_size():
    """B=4, T=2048, d=1280, 10 heads x 128, W=512: forward + backward + loss."""
    wl = wl_of("layer_bf16")
    x = synth.layer_inputs(wl, 1234)
    g = run_gpu(wl, x, lam=wl["lam"])
    r = run_oracle(wl, x, lam=wl["lam"])
    errs = compare(g, r, "bf16", FWD + BWD, report_elementwise=True)
    print("full-size layer errors:", {k: f"{v:.2e}" for k, v in errs.items()})
    assert abs(g["loss"] - r["loss"]) <= 2e-2 * abs(r["loss"])


@pytest.mark.parametrize("name,over", [("tiny_f32", {}), ("layer_bf16", dict(B=2, T=300, H=3, hd=128, d=160, W=100)),
                                       ("layer_bf16", dict(B=2, T=333, H=3, hd=64, d=160, W=47)), ("layer_bf16", {})])
def test_loss_prepare_bwd_fused(name, over):
    """maglev_consistency_loss_prepare_bwd, then the backward told it ran:
    every output within tolerance of the oracle, and against the separate loss
    and backward calls the same loss bit for bit and the same updated dO."""
    wl = wl_of(name, **over)
    if name == "layer_bf16" and over:
        wl["target"] = "independent"
    x = synth.layer_inputs(wl, 4321)
    lam = 0.1 if wl["dtype"] == "bf16" else 1.0
    g = run_gpu(wl, x, lam=lam, fused=True)
    r = run_oracle(wl, x, lam=lam)
    compare(g, r, wl["dtype"], FWD + BWD)
    tol = 2e-2 if wl["dtype"] == "bf16" else 1e-4
    assert abs(g["loss"] - r["loss"]) <= tol * abs(r["loss"])
    p = run_gpu(wl, x, lam=lam)
    assert torch.equal(g["loss_bits"], p["loss_bits"])
    assert np.array_equal(g["dout_total"], p["dout_total"])
    for n in BWD:  # only the order of Delta's fp32 sums differs between the two paths
        assert normwise(g[n], p[n]) <= tol, n


# --------------------------------------------------------------------------- bit-exact probes
def test_mask_probe_bit_exact():
    """q = 0 => uniform weights over the window; v_j = e_{j mod hd} with W <= hd:
    the nonzero set of o_i is exactly {j mod hd : i-W+1 <= j <= i}."""
    T, H, hd, W = 256, 1, 64, 64
    L = InjectedSWALayer(1, T, H, hd, 8, W, dtype="f32", inject=False)
    q = torch.zeros(1, T, H, hd, device="cuda")
    k = torch.randn(1, T, H, hd, device="cuda")
    v = torch.zeros(1, T, H, hd, device="cuda")
    v[0, torch.arange(T), 0, torch.arange(T) % hd] = 1.0
    L.forward(q, k, v)
    o = host(L.out)[0, :, 0]
    for i in range(T):
        want = {j % hd for j in range(max(0, i - W + 1), i + 1)}
        got = set(np.nonzero(o[i])[0].tolist())
        assert got == want, i
        n = min(i + 1, W)
        np.testing.assert_allclose(o[i][list(want)], 1.0 / n, rtol=1e-6)


def test_gate_off_bitwise_equals_plain_swa():
    wl = wl_of("layer_bf16", B=1, T=400, H=2, hd=128, d=96, W=64)
    x = synth.layer_inputs(wl, 3)
    x["gates"] = np.array([[0.0, 0.0], [-np.inf, -np.inf], [0.0, 0.0], [-np.inf, -np.inf]], np.float32)
    a = run_gpu(wl, x, inject=True, bwd=False)
    b = run_gpu(wl, x, inject=False, bwd=False)
    np.testing.assert_array_equal(a["out"], b["out"])
    np.testing.assert_array_equal(a["lse"], b["lse"])


def test_window_perturbation_bitwise():
    wl = wl_of("layer_bf16", B=1, T=320, H=2, hd=64, d=64, W=40)
    x = synth.layer_inputs(wl, 11)
    base = run_gpu(wl, x, bwd=False)["out"]
    i = 250
    x2 = dict(x)
    kb = x["k"].bits.copy()
    vb = x["v"].bits.copy()
    kb[0, : i - 40 + 1] = synth.round_to_bf16_bits(np.full(kb[0, : i - 40 + 1].shape, 3.0, np.float32))
    vb[0, : i - 40 + 1] = synth.round_to_bf16_bits(np.full(vb[0, : i - 40 + 1].shape, -2.0, np.float32))
    x2["k"] = synth.Tensor(kb, "bf16")
    x2["v"] = synth.Tensor(vb, "bf16")
    pert = run_gpu(wl, x2, bwd=False)["out"]
    np.testing.assert_array_equal(pert[0, i], base[0, i])
    assert np.abs(pert[0, i - 40] - base[0, i - 40]).max() > 0


@pytest.mark.parametrize("dtype,hd,n_layers", [("f32", 64, 3), ("bf16", 128, 4)])
def test_accumulated_memory_gradient_over_layers(dtype, hd, n_layers):
    """dR_mode FIRST / ADD / LAST sums dL/dR over layers that share W^rec in
    fp32 and rounds the total once; mode FIRST and ADD leave dR_k/dR_v alone."""
    wl = wl_of("layer_bf16", B=1, T=256, H=2, hd=hd, d=64, W=32, dtype=dtype)
    xs = [synth.layer_inputs(wl, 40, layer=l) for l in range(n_layers)]
    B, T, H, d, W = 1, 256, 2, 64, 32
    td = torch.bfloat16 if dtype == "bf16" else torch.float32
    m, wk, wv = dev(xs[0]["m_shift"]), dev(xs[0]["w_mk"]), dev(xs[0]["w_mv"])
    dRk = torch.full((B, T, H * hd), 7.0, dtype=td, device="cuda")
    dRv = torch.full((B, T, H * hd), 7.0, dtype=td, device="cuda")
    acc = (torch.empty(B, T, H * hd, device="cuda"), torch.empty(B, T, H * hd, device="cuda"))
    want_k = 0
    want_v = 0
    Rk, Rv = oracle.mem_project(xs[0]["m_shift"].f64, xs[0]["w_mk"].f64, xs[0]["w_mv"].f64)
    modes = [mg.MAGLEV_DR_FIRST] + [mg.MAGLEV_DR_ADD] * (n_layers - 2) + [mg.MAGLEV_DR_LAST]
    for l, (x, mode) in enumerate(zip(xs, modes)):
        L = InjectedSWALayer(B, T, H, hd, d, W, dtype=dtype)
        q, k, v, gt = dev(x["q"]), dev(x["k"]), dev(x["v"]), dev(x["gates"])
        L.forward(q, k, v, gt, m, wk, wv)
        L.dR_k, L.dR_v = dRk, dRv
        L.backward(k, v, dev(x["dout"]), gt, dR_mode=mode, dR_acc=acc)
        if mode != mg.MAGLEV_DR_LAST:
            torch.cuda.synchronize()
            assert torch.all(dRk == 7.0) and torch.all(dRv == 7.0), "running sums stay in dR_acc"
        g = oracle.inject_swa_backward(x["q"].f64, x["k"].f64, x["v"].f64, Rk, Rv,
                                       x["gates"].astype(np.float64), x["dout"].f64, W)
        want_k = want_k + g["dR_k"]
        want_v = want_v + g["dR_v"]
    torch.cuda.synchronize()
    assert_close(host(dRk), want_k, dtype, "dR_k sum")
    assert_close(host(dRv), want_v, dtype, "dR_v sum")


# --------------------------------------------------------------------------- projection backward alone
@pytest.mark.parametrize("which", ["both", "dm", "dw"])
def test_mem_project_bwd_outputs(which):
    """maglev_mem_project_bwd on its own: dm_shift and dW together (one launch
    that deals the tiles of both over the SM pairs) and each alone (a launch of
    its own), with ragged rows (B*T = 600, K of dW not a multiple of the K block)
    and ragged columns (d = 384, half a pair tile past 256)."""
    B, T, H, hd, d = 2, 300, 2, 128, 384
    D = H * hd
    seed = 77
    m = synth.normal(seed, 901, (B, T, d))
    wk = synth.normal(seed, 902, (D, d), std=d ** -0.5)
    wv = synth.normal(seed, 903, (D, d), std=d ** -0.5)
    dRk = synth.normal(seed, 904, (B, T, D))
    dRv = synth.normal(seed, 905, (B, T, D))
    L = InjectedSWALayer(B, T, H, hd, d, 64, dtype="bf16")
    dm = torch.full((B, T, d), float("nan"), dtype=torch.bfloat16, device="cuda") if which != "dw" else None
    dwk = torch.full((D, d), float("nan"), dtype=torch.bfloat16, device="cuda") if which != "dm" else None
    dwv = torch.full((D, d), float("nan"), dtype=torch.bfloat16, device="cuda") if which != "dm" else None
    mg.maglev_mem_project_bwd(L.desc, dev(m), dev(wk), dev(wv), dev(dRk), dev(dRv), dm, dwk, dwv)
    torch.cuda.synchronize()
    ref_dm, ref_dwk, ref_dwv = oracle.mem_project_backward(m.f64, wk.f64, wv.f64, dRk.f64, dRv.f64)
    if dm is not None:
        assert_close(host(dm), ref_dm, "bf16", "dm_shift")
    if dwk is not None:
        assert_close(host(dwk), ref_dwk, "bf16", "dw_mk")
        assert_close(host(dwv), ref_dwv, "bf16", "dw_mv")
    assert mg.maglev_device_status() == 0


# --------------------------------------------------------------------------- projection in the call
LAYER_OUTPUTS = ("out", "lse", "R_k", "R_v", "dq", "dk", "dv", "dR_k", "dR_v", "dgate", "dm_shift", "dw_mk",
                 "dw_mv")


def test_projection_in_call_matches_separate_calls_bitwise():
    """The shared projection run inside the forward and backward calls (m_shift
    given) against maglev_mem_project / maglev_mem_project_bwd called on their
    own around calls without it: every output agrees bit for bit, eagerly on a
    non-default caller stream and replayed from a CUDA graph captured from the
    same calls. dq is reproducible here because W < 128: each query row takes
    the contributions of at most two 128-key tiles, and two fp32 adds into the
    zeroed accumulator give the same sum in either order."""
    wl = wl_of("layer_bf16", B=2, T=300, H=3, hd=128, d=160, W=100, target="independent")
    x = synth.layer_inputs(wl, 99)
    B, T, H, hd, d, W = (wl[n] for n in ("B", "T", "H", "hd", "d", "W"))
    q, k, v, gates = dev(x["q"]), dev(x["k"]), dev(x["v"]), dev(x["gates"])
    m, wk, wv, dout = dev(x["m_shift"]), dev(x["w_mk"]), dev(x["w_mv"]), dev(x["dout"])

    def layer():
        return InjectedSWALayer(B, T, H, hd, d, W, dtype="bf16", rope_base=wl["rope_base"], eps=wl["eps"])

    sep = layer()
    mg.maglev_mem_project(sep.desc, m, wk, wv, sep.R_k, sep.R_v)
    sep.forward(q, k, v, gates)
    sep.backward(k, v, dout, gates)
    mg.maglev_mem_project_bwd(sep.desc, m, wk, wv, sep.dR_k, sep.dR_v, sep.dm_shift, sep.dw_mk, sep.dw_mv)
    torch.cuda.synchronize()

    eager = layer()
    st = torch.cuda.Stream()
    st.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(st):
        eager.forward(q, k, v, gates, m, wk, wv, stream=st)
        eager.backward(k, v, dout, gates, m, wk, wv, stream=st)
    st.synchronize()
    for n in LAYER_OUTPUTS:
        assert torch.equal(getattr(eager, n), getattr(sep, n)), n

    graphed = layer()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        graphed.forward(q, k, v, gates, m, wk, wv)
        graphed.backward(k, v, dout, gates, m, wk, wv)
    g.replay()
    torch.cuda.synchronize()
    for n in LAYER_OUTPUTS:
        assert torch.equal(getattr(graphed, n), getattr(sep, n)), n
    del g
    assert mg.maglev_device_status() == 0


# --------------------------------------------------------------------------- consistency loss
@pytest.mark.parametrize("dtype,rows,d", [("f32", 256, 128), ("bf16", 8192, 1280), ("bf16", 3, 17)])
def test_consistency_loss(dtype, rows, d):
    m = synth.normal(9, 1, (rows, d), dtype=dtype)
    t = synth.normal(9, 2, (rows, d), dtype=dtype)
    lam = 0.1
    ref_loss, ref_dm, ref_dmt = oracle.consistency_loss(m.f64, t.f64, lam)
    td = torch.bfloat16 if dtype == "bf16" else torch.float32
    dm = torch.empty(rows, d, dtype=td, device="cuda")
    dmt = torch.empty_like(dm)
    loss = torch.zeros((), device="cuda")
    ws = torch.empty(mg.maglev_consistency_workspace_bytes(rows, d), dtype=torch.uint8, device="cuda")
    code = mg.MAGLEV_BF16 if dtype == "bf16" else mg.MAGLEV_F32
    mg.maglev_consistency_loss(dev(m), dev(t), rows, d, code, lam, 0.0, loss, dm, dmt, 0, ws)
    l1 = loss.item()
    mg.maglev_consistency_loss(dev(m), dev(t), rows, d, code, lam, 0.0, loss, dm, dmt, 0, ws)
    assert loss.item() == l1                          # fixed reduction order
    assert abs(l1 - ref_loss) <= 1e-5 * abs(ref_loss)
    assert_close(host(dm), ref_dm, dtype, "dm")
    assert_close(host(dmt), ref_dmt, dtype, "dm_target")


# --------------------------------------------------------------------------- decode
def decode_case(B, H, hd, d, W, pos, dtype, seed=21, inject=True):
    x = synth.decode_inputs(seed, B, H, hd, d, W, pos, dtype=dtype)
    S = DecodeLayerState(B, H, hd, d, W, dtype=dtype, inject=inject)
    pos_t = torch.from_numpy(x["pos"]).cuda()
    kr, vr = dev(x["k_ring"]), dev(x["v_ring"])
    S.mem_project(pos_t, dev(x["m_prev"]), dev(x["w_mk"]), dev(x["w_mv"]))
    S.step(pos_t, dev(x["q"]), dev(x["k"]), dev(x["v"]), dev(x["gates"]), kr, vr)
    torch.cuda.synchronize()
    H_ = H
    krec, vrec = oracle.decode_mem_project(x["pos"], x["m_prev"].f64, x["w_mk"].f64, x["w_mv"].f64, H_)
    out, kr2, vr2 = oracle.decode_step(x["pos"], x["q"].f64, x["k"].f64, x["v"].f64, krec, vrec,
                                       x["gates"].astype(np.float64), x["k_ring"].f64, x["v_ring"].f64,
                                       inject=inject)
    return x, S, host(kr), host(vr), (krec, vrec, out, kr2, vr2)


@pytest.mark.parametrize("dtype,hd,W,pos", [
    ("f32", 64, 64, [0, 5, 63, 64, 200, 6400]),
    ("bf16", 128, 512, [0, 1, 510, 511, 512, 4607]),
    ("bf16", 64, 33, [32, 33, 7, 100, 0, 1000]),
])
def test_decode_step_parity(dtype, hd, W, pos):
    B, H, d = len(pos), 2, 96
    x, S, kr, vr, (krec, vrec, out, kr2, vr2) = decode_case(B, H, hd, d, W, pos, dtype)
    assert_close(host(S.krec), krec, dtype, "krec_rot")
    assert_close(host(S.vrec), vrec, dtype, "vrec")
    assert_close(host(S.out), out, dtype, "out")
    for b, p in enumerate(pos):
        s = p % W
        keep = [j for j in range(W) if j != s]
        np.testing.assert_array_equal(kr[b][:, keep], x["k_ring"].f64[b][:, keep])
        np.testing.assert_array_equal(vr[b][:, keep], x["v_ring"].f64[b][:, keep])
        assert normwise(kr[b][:, s], kr2[b][:, s]) <= TOL[dtype]
        assert normwise(vr[b][:, s], vr2[b][:, s]) <= TOL[dtype]


def test_decode_full_shape():
    """64 sequences x 10 heads x 128, 512-entry ring, positions 512 and 4607."""
    pos = [512] * 32 + [4607] * 32
    x, S, kr, vr, (krec, vrec, out, kr2, vr2) = decode_case(64, 10, 128, 1280, 512, pos, "bf16")
    assert_close(host(S.out), out, "bf16", "out")
    assert_close(host(S.krec), krec, "bf16", "krec_rot")


def test_decode_full_shape_mixed_positions():
    """640 (sequence, head) pairs, so each persistent CTA walks several pairs in a
    row, with positions that change from pair to pair: negative (no write, zero
    output), partial rings (p < W-1), p = W-1, wrapped rings. Every slot of both
    rings is checked: the new entry against the oracle, all others bit-exact."""
    B, H, hd, d, W = 64, 10, 128, 1280, 512
    cycle = [-1, 0, 1, 37, 255, 510, 511, 512, 1000, 4607, -5, 2047, 300]
    pos = [cycle[b % len(cycle)] for b in range(B)]
    x = synth.decode_inputs(23, B, H, hd, d, W, pos, dtype="bf16")
    S = DecodeLayerState(B, H, hd, d, W, dtype="bf16")
    pos_t = torch.from_numpy(x["pos"]).cuda()
    kr, vr = dev(x["k_ring"]), dev(x["v_ring"])
    S.mem_project(pos_t, dev(x["m_prev"]), dev(x["w_mk"]), dev(x["w_mv"]))
    S.step(pos_t, dev(x["q"]), dev(x["k"]), dev(x["v"]), dev(x["gates"]), kr, vr)
    torch.cuda.synchronize()
    kr, vr, out = host(kr), host(vr), host(S.out)
    ok = [b for b in range(B) if pos[b] >= 0]
    bad = [b for b in range(B) if pos[b] < 0]
    sub = lambda t: t.f64[ok]
    krec, vrec = oracle.decode_mem_project(x["pos"][ok], sub(x["m_prev"]), x["w_mk"].f64, x["w_mv"].f64, H)
    o_ref, kr2, vr2 = oracle.decode_step(x["pos"][ok], sub(x["q"]), sub(x["k"]), sub(x["v"]), krec, vrec,
                                         x["gates"].astype(np.float64), sub(x["k_ring"]), sub(x["v_ring"]))
    assert_close(out[ok], o_ref, "bf16", "out")
    assert np.all(out[bad] == 0), "a negative position writes zeros to out"
    for b in bad:  # ring untouched
        np.testing.assert_array_equal(kr[b], x["k_ring"].f64[b])
        np.testing.assert_array_equal(vr[b], x["v_ring"].f64[b])
    for i, b in enumerate(ok):
        s_ = pos[b] % W
        keep = [j for j in range(W) if j != s_]
        np.testing.assert_array_equal(kr[b][:, keep], x["k_ring"].f64[b][:, keep])
        np.testing.assert_array_equal(vr[b][:, keep], x["v_ring"].f64[b][:, keep])
        assert normwise(kr[b][:, s_], kr2[i][:, s_]) <= TOL["bf16"], (b, pos[b])
        assert normwise(vr[b][:, s_], vr2[i][:, s_]) <= TOL["bf16"], (b, pos[b])


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_decode_matches_training_row(dtype):
    """Ring filled with the forward's mixed entries (in the ring's storage
    type): decode at p equals forward row p -- recurrence equals teacher
    forcing when the ring holds what the training pass mixed."""
    wl = wl_of("layer_bf16", B=1, T=700, H=2, hd=128, d=128, W=512, dtype=dtype)
    x = synth.layer_inputs(wl, 8)
    B, T, H, hd, W = 1, 700, 2, 128, 512
    Rk, Rv = oracle.mem_project(x["m_shift"].f64, x["w_mk"].f64, x["w_mv"].f64)
    f = oracle.inject_swa_forward(x["q"].f64, x["k"].f64, x["v"].f64, Rk, Rv,
                                  x["gates"].astype(np.float64), W)
    for p in (0, 300, 511, 699):
        kr = np.zeros((1, H, W, hd), np.float32)
        vr = np.zeros((1, H, W, hd), np.float32)
        for j in range(max(0, p - W + 1), p):
            kr[0, :, j % W] = f["k_bar"][0, j]
            vr[0, :, j % W] = f["v_bar"][0, j]
        kr_t = synth.Tensor.from_float(kr, dtype)
        vr_t = synth.Tensor.from_float(vr, dtype)
        S = DecodeLayerState(1, H, hd, 128, W, dtype=dtype)
        pos_t = torch.tensor([p], dtype=torch.int64, device="cuda")
        row = lambda t: synth.Tensor(np.ascontiguousarray(t.bits[:, p]), t.dtype)
        S.mem_project(pos_t, dev(row(x["m_shift"])), dev(x["w_mk"]), dev(x["w_mv"]))
        o = S.step(pos_t, dev(row(x["q"])), dev(row(x["k"])), dev(row(x["v"])),
                   dev(x["gates"]), dev(kr_t), dev(vr_t))
        assert_close(host(o)[0], f["out"][0, p], dtype, f"decode row {p}")


def test_device_status_clean():
    assert mg.maglev_device_status() == 0
