"""Pins of the CPU oracle against things other than itself.

The pages ("Maglev: Sliding Recurrent Memory", paper.rainbus.top, 方法步骤详情)
print no worked numeric example, so the oracle is pinned by:
  * library routines for the special cases the method reduces to (torch CPU
    scaled_dot_product_attention and rms_norm in float64, complex rotation),
  * closed forms and invariants the pages fix (gate neutral at 0, window of W
    keys with self included, relative-position RoPE, gate-off = plain SWA),
  * brute force over explicit window lists on tiny shapes,
  * central finite differences and torch autograd for every gradient,
  * the decode <-> teacher-forcing identity (recurrence equals the training form
    when fed the same memory).
Each pin is chosen so that a dropped term, a wrong sign/index, a transposed
operand or an off-by-one window fails at least one test.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
import synth

RNG = np.random.default_rng(7)


def rand(*shape):
    return RNG.standard_normal(shape)


# ---------------------------------------------------------------- test-side helpers
def rotate_complex(x, pos, base):
    """Independent RoPE: (x_c + i x_{c+hd/2}) * exp(i pos base^(-2c/hd))."""
    hd = x.shape[-1]
    z = x[..., : hd // 2] + 1j * x[..., hd // 2:]
    freqs = np.power(float(base), -np.arange(0, hd, 2, dtype=np.float64) / hd)
    w = np.exp(1j * np.multiply.outer(np.asarray(pos, dtype=np.float64), freqs))
    r = z * w
    return np.concatenate([r.real, r.imag], axis=-1)


def sdpa(q, k, v, mask=None, causal=False):
    """torch CPU float64 attention over [T, hd] operands of one head."""
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a))[None, None]
    m = None if mask is None else torch.from_numpy(mask)[None, None]
    o = F.scaled_dot_product_attention(t(q), t(k), t(v), attn_mask=m, is_causal=causal)
    return o[0, 0].numpy()


def band(T, W):
    i = np.arange(T)[:, None]
    j = np.arange(T)[None, :]
    return (j <= i) & (i - j < W)


def layer(B=2, T=24, H=2, hd=8, d=12):
    D = H * hd
    return dict(q=rand(B, T, H, hd), k=rand(B, T, H, hd), v=rand(B, T, H, hd),
                m=rand(B, T, d), wk=rand(D, d) / np.sqrt(d), wv=rand(D, d) / np.sqrt(d),
                a=RNG.uniform(-2, 2, (4, H)), dout=rand(B, T, H, hd))


# ---------------------------------------------------------------- gate / rope / rmsnorm
def test_gate_neutral_and_limits():
    # g = 2 sigmoid(a): exactly 1 at a = 0 (neutral value), 0 at -inf, 2 at +inf.
    assert oracle.gate(np.array([0.0]))[0] == 1.0
    assert oracle.gate(np.array([-np.inf]))[0] == 0.0
    assert oracle.gate(np.array([np.inf]))[0] == 2.0
    assert oracle.gate_slope(np.array([-np.inf]))[0] == 0.0
    assert oracle.gate_slope(np.array([0.0]))[0] == 0.5
    a = np.linspace(-30, 30, 101)
    np.testing.assert_allclose(oracle.gate(a), 1.0 + np.tanh(a / 2.0), rtol=1e-14, atol=1e-15)


def test_rope_matches_complex_rotation():
    x = rand(5, 7, 16)
    pos = RNG.integers(0, 5000, size=(5, 7))
    for base in (10000.0, 500.0):
        np.testing.assert_allclose(oracle.rope(x, pos, base), rotate_complex(x, pos, base), atol=1e-12)
        np.testing.assert_allclose(oracle.rope(x, pos, base, inverse=True),
                                   rotate_complex(x, -pos, base), atol=1e-12)


def test_rope_closed_form_and_invariants():
    hd = 8
    e0 = np.zeros(hd)
    e0[0] = 1.0
    p = 3.0
    y = oracle.rope(e0, np.array(p), 10000.0)       # theta_0 = 1
    assert abs(y[0] - math.cos(p)) < 1e-15 and abs(y[hd // 2] - math.sin(p)) < 1e-15
    assert np.all(np.delete(y, [0, hd // 2]) == 0)
    x = rand(11, hd)
    pos = np.arange(11)
    r = oracle.rope(x, pos, 10000.0)
    np.testing.assert_allclose(np.linalg.norm(r, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-13)
    np.testing.assert_allclose(oracle.rope(r, pos, 10000.0, inverse=True), x, atol=1e-13)
    # relative position: <R(i) a, R(j) b> depends on i - j only
    a, b = rand(hd), rand(hd)
    s1 = oracle.rope(a, np.array(40), 1e4) @ oracle.rope(b, np.array(13), 1e4)
    s2 = oracle.rope(a, np.array(1040), 1e4) @ oracle.rope(b, np.array(1013), 1e4)
    assert abs(s1 - s2) < 1e-11


def test_rmsnorm_matches_torch_and_closed_form():
    x = rand(6, 4, 32)
    ref = F.rms_norm(torch.from_numpy(x), (32,), eps=1e-6).numpy()
    np.testing.assert_allclose(oracle.rmsnorm(x, 1e-6), ref, rtol=1e-13)
    c = 0.37
    y = oracle.rmsnorm(np.full(16, c), 1e-6)
    np.testing.assert_allclose(y, c / math.sqrt(c * c + 1e-6), rtol=1e-15)


def test_rmsnorm_backward_matches_autograd():
    x = rand(3, 5, 16)
    dy = rand(3, 5, 16)
    xt = torch.from_numpy(x).requires_grad_(True)
    F.rms_norm(xt, (16,), eps=1e-3).backward(torch.from_numpy(dy))
    np.testing.assert_allclose(oracle.rmsnorm_backward(x, dy, 1e-3), xt.grad.numpy(), rtol=1e-12, atol=1e-13)


# ---------------------------------------------------------------- attention forward
def test_full_window_no_injection_equals_causal_sdpa():
    L = layer(B=1, T=30, H=2, hd=8)
    f = oracle.inject_swa_forward(L["q"], L["k"], L["v"], None, None, None, window=30, inject=False)
    pos = np.arange(30)
    for h in range(2):
        qr = rotate_complex(L["q"][0, :, h], pos, 1e4)
        kr = rotate_complex(L["k"][0, :, h], pos, 1e4)
        np.testing.assert_allclose(f["out"][0, :, h], sdpa(qr, kr, L["v"][0, :, h], causal=True), atol=1e-12)
        # W > T is the same as W = T
    g = oracle.inject_swa_forward(L["q"], L["k"], L["v"], None, None, None, window=1000, inject=False)
    np.testing.assert_array_equal(g["out"], f["out"])


def test_lse_matches_torch_logsumexp():
    L = layer(B=1, T=20, H=1, hd=8)
    W = 6
    f = oracle.inject_swa_forward(L["q"], L["k"], L["v"], None, None, None, window=W, inject=False)
    pos = np.arange(20)
    qr = rotate_complex(L["q"][0, :, 0], pos, 1e4)
    kr = rotate_complex(L["k"][0, :, 0], pos, 1e4)
    s = torch.from_numpy(qr @ kr.T / math.sqrt(8)).masked_fill(~torch.from_numpy(band(20, W)), -math.inf)
    np.testing.assert_allclose(f["lse"][0, 0], torch.logsumexp(s, dim=1).numpy(), rtol=1e-13)


@pytest.mark.parametrize("W", [1, 3, 7, 24])
def test_gate_off_is_plain_swa(W):
    # a_rec = -inf, a_loc = 0  =>  g_rec = 0, g_loc = 1: Maglev "generalizes
    # sliding-window attention" (gptget abstract); result = band-masked SDPA.
    L = layer(B=2, T=24, H=2, hd=8)
    a = np.array([[0.0, 0.0], [-np.inf, -np.inf], [0.0, 0.0], [-np.inf, -np.inf]])
    Rk, Rv = oracle.mem_project(L["m"], L["wk"], L["wv"])
    f = oracle.inject_swa_forward(L["q"], L["k"], L["v"], Rk, Rv, a, window=W)
    plain = oracle.inject_swa_forward(L["q"], L["k"], L["v"], None, None, None, window=W, inject=False)
    np.testing.assert_array_equal(f["out"], plain["out"])
    pos = np.arange(24)
    for b in range(2):
        for h in range(2):
            qr = rotate_complex(L["q"][b, :, h], pos, 1e4)
            kr = rotate_complex(L["k"][b, :, h], pos, 1e4)
            ref = sdpa(qr, kr, L["v"][b, :, h], mask=band(24, W))
            np.testing.assert_allclose(f["out"][b, :, h], ref, atol=1e-12)


def test_memory_only_entries_match_library_composition():
    # a_loc = -inf, a_rec = 0: keys = RoPE(RMSNorm_head(m W_mk^T)), values = m W_mv^T.
    B, T, H, hd, d, W = 1, 20, 2, 8, 12, 5
    L = layer(B, T, H, hd, d)
    a = np.array([[-np.inf] * H, [0.0] * H, [-np.inf] * H, [0.0] * H])
    Rk, Rv = oracle.mem_project(L["m"], L["wk"], L["wv"])
    f = oracle.inject_swa_forward(L["q"], L["k"], L["v"], Rk, Rv, a, window=W, pos0=17)
    m = torch.from_numpy(L["m"][0])
    rk = (m @ torch.from_numpy(L["wk"]).T).reshape(T, H, hd)
    rv = (m @ torch.from_numpy(L["wv"]).T).reshape(T, H, hd)
    nk = F.rms_norm(rk, (hd,), eps=1e-6).numpy()
    pos = 17 + np.arange(T)
    for h in range(H):
        qr = rotate_complex(L["q"][0, :, h], pos, 1e4)
        kr = rotate_complex(nk[:, h], pos, 1e4)
        ref = sdpa(qr, kr, rv[:, h].numpy(), mask=band(T, W))
        np.testing.assert_allclose(f["out"][0, :, h], ref, atol=1e-12)


def test_general_gates_match_library_composition():
    B, T, H, hd, d, W = 1, 18, 3, 8, 10, 4
    L = layer(B, T, H, hd, d)
    Rk, Rv = oracle.mem_project(L["m"], L["wk"], L["wv"])
    f = oracle.inject_swa_forward(L["q"], L["k"], L["v"], Rk, Rv, L["a"], window=W)
    g = 2.0 * torch.sigmoid(torch.from_numpy(L["a"])).numpy()
    nk = F.rms_norm(torch.from_numpy(Rk.reshape(T, H, hd)), (hd,), eps=1e-6).numpy()
    pos = np.arange(T)
    for h in range(H):
        qr = rotate_complex(L["q"][0, :, h], pos, 1e4)
        kb = g[0, h] * rotate_complex(L["k"][0, :, h], pos, 1e4) + g[1, h] * rotate_complex(nk[:, h], pos, 1e4)
        vb = g[2, h] * L["v"][0, :, h] + g[3, h] * Rv.reshape(T, H, hd)[:, h]
        np.testing.assert_allclose(f["out"][0, :, h], sdpa(qr, kb, vb, mask=band(T, W)), atol=1e-12)


def test_window_perturbation_boundary():
    # o_i ignores keys older than i-W+1 and depends on key i-W+1 (W keys, self included).
    B, T, H, hd, d, W = 1, 40, 1, 8, 8, 9
    L = layer(B, T, H, hd, d)
    Rk, Rv = oracle.mem_project(L["m"], L["wk"], L["wv"])
    base = oracle.inject_swa_forward(L["q"], L["k"], L["v"], Rk, Rv, L["a"], W)["out"]
    i = 30
    for j, changes in [(i - W, False), (i - W - 5, False), (i - W + 1, True), (i, True)]:
        k2, v2 = L["k"].copy(), L["v"].copy()
        k2[0, j] += 3.0
        v2[0, j] += 3.0
        o2 = oracle.inject_swa_forward(L["q"], k2, v2, Rk, Rv, L["a"], W)["out"]
        if changes:
            assert np.abs(o2[0, i] - base[0, i]).max() > 1e-6
        else:
            np.testing.assert_array_equal(o2[0, i], base[0, i])


def test_constant_values_give_constant_output():
    # Rows of P sum to 1: with v_bar = c everywhere the output is c.
    B, T, H, hd, d, W = 2, 16, 2, 8, 8, 5
    L = layer(B, T, H, hd, d)
    Rk, _ = oracle.mem_project(L["m"], L["wk"], L["wv"])
    v = np.full((B, T, H, hd), 0.75)
    Rv = np.full((B, T, H * hd), -1.25)
    f = oracle.inject_swa_forward(L["q"], L["k"], v, Rk, Rv, L["a"], W)
    g = oracle.gate(L["a"])
    want = g[2] * 0.75 + g[3] * (-1.25)
    np.testing.assert_allclose(f["out"], np.broadcast_to(want[None, None, :, None], f["out"].shape), atol=1e-13)


def test_position_offset_invariance():
    B, T, H, hd, d, W = 1, 20, 2, 8, 8, 6
    L = layer(B, T, H, hd, d)
    Rk, Rv = oracle.mem_project(L["m"], L["wk"], L["wv"])
    o0 = oracle.inject_swa_forward(L["q"], L["k"], L["v"], Rk, Rv, L["a"], W, pos0=0)["out"]
    o1 = oracle.inject_swa_forward(L["q"], L["k"], L["v"], Rk, Rv, L["a"], W, pos0=1234)["out"]
    np.testing.assert_allclose(o0, o1, atol=1e-10)


def _brute_force(q, k, v, Rk, Rv, a, W, base, eps):
    """Scalar loops with an explicit window list per position (tiny shapes only)."""
    B, T, H, hd = q.shape
    half = hd // 2
    g = [[2.0 / (1.0 + math.exp(-x)) if x != -math.inf else 0.0 for x in row] for row in a]

    def rot(x, p):
        y = [0.0] * hd
        for c in range(half):
            th = p * base ** (-2.0 * c / hd)
            y[c] = x[c] * math.cos(th) - x[c + half] * math.sin(th)
            y[c + half] = x[c] * math.sin(th) + x[c + half] * math.cos(th)
        return y

    out = np.zeros_like(q)
    for b in range(B):
        for h in range(H):
            kb, vb, qr = [], [], []
            for t in range(T):
                r = [Rk[b, t, h * hd + c] for c in range(hd)]
                ms = sum(x * x for x in r) / hd
                n = [x / math.sqrt(ms + eps) for x in r]
                kl, kr = rot(list(k[b, t, h]), t), rot(n, t)
                kb.append([g[0][h] * kl[c] + g[1][h] * kr[c] for c in range(hd)])
                vb.append([g[2][h] * v[b, t, h, c] + g[3][h] * Rv[b, t, h * hd + c] for c in range(hd)])
                qr.append(rot(list(q[b, t, h]), t))
            for i in range(T):
                keys = [j for j in range(T) if i - W + 1 <= j <= i]
                s = [sum(qr[i][c] * kb[j][c] for c in range(hd)) / math.sqrt(hd) for j in keys]
                mx = max(s)
                e = [math.exp(x - mx) for x in s]
                z = sum(e)
                for c in range(hd):
                    out[b, i, h, c] = sum(e[n] * vb[j][c] for n, j in enumerate(keys)) / z
    return out


@pytest.mark.parametrize("W", [1, 3, 16])
def test_brute_force_tiny(W):
    B, T, H, hd, d = 1, 16, 1, 4, 6
    L = layer(B, T, H, hd, d)
    Rk, Rv = oracle.mem_project(L["m"], L["wk"], L["wv"])
    f = oracle.inject_swa_forward(L["q"], L["k"], L["v"], Rk, Rv, L["a"], W)
    bf = _brute_force(L["q"], L["k"], L["v"], Rk, Rv, L["a"], W, 1e4, 1e-6)
    np.testing.assert_allclose(f["out"], bf, atol=1e-13)


# ---------------------------------------------------------------- backward
def _total_loss(L, Rk, Rv, a, W, target, lam):
    f = oracle.inject_swa_forward(L["q"], L["k"], L["v"], Rk, Rv, a, W)
    B, T, H, hd = f["out"].shape
    loss, _, _ = oracle.consistency_loss(f["out"].reshape(B * T, H * hd), target, lam)
    return np.sum(f["out"] * L["dout"]) + loss


def test_backward_central_differences():
    B, T, H, hd, d, W = 1, 10, 2, 4, 6, 4
    L = layer(B, T, H, hd, d)
    target = rand(B * T, H * hd)
    lam = 0.3
    Rk, Rv = oracle.mem_project(L["m"], L["wk"], L["wv"])
    f = oracle.inject_swa_forward(L["q"], L["k"], L["v"], Rk, Rv, L["a"], W)
    _, dm, _ = oracle.consistency_loss(f["out"].reshape(B * T, H * hd), target, lam)
    dout = L["dout"] + dm.reshape(B, T, H, hd)
    g = oracle.inject_swa_backward(L["q"], L["k"], L["v"], Rk, Rv, L["a"], dout, W)
    dms, dWk, dWv = oracle.mem_project_backward(L["m"], L["wk"], L["wv"], g["dR_k"], g["dR_v"])
    grads = {"q": g["dq"], "k": g["dk"], "v": g["dv"], "a": g["dgate"], "m": dms, "wk": dWk, "wv": dWv}
    h = 1e-6
    for name, grad in grads.items():
        for idx in [tuple(RNG.integers(0, s) for s in grad.shape) for _ in range(6)]:
            def loss_at(delta):
                L2 = {kk: (vv.copy() if isinstance(vv, np.ndarray) else vv) for kk, vv in L.items()}
                L2[name][idx] += delta
                rk, rv = oracle.mem_project(L2["m"], L2["wk"], L2["wv"])
                return _total_loss(L2, rk, rv, L2["a"], W, target, lam)
            fd = (loss_at(h) - loss_at(-h)) / (2 * h)
            assert abs(fd - grad[idx]) <= 1e-6 * max(1.0, abs(fd)), (name, idx, fd, grad[idx])


def test_backward_matches_torch_autograd():
    B, T, H, hd, d, W = 2, 14, 2, 8, 10, 5
    L = layer(B, T, H, hd, d)
    Rk, Rv = oracle.mem_project(L["m"], L["wk"], L["wv"])
    g = oracle.inject_swa_backward(L["q"], L["k"], L["v"], Rk, Rv, L["a"], L["dout"], W, pos0=3)
    T_ = lambda x: torch.from_numpy(np.ascontiguousarray(x)).requires_grad_(True)
    q, k, v, rk, rv, a = T_(L["q"]), T_(L["k"]), T_(L["v"]), T_(Rk), T_(Rv), T_(L["a"])
    pos = torch.arange(T, dtype=torch.float64) + 3
    freqs = 1e4 ** (-torch.arange(0, hd, 2, dtype=torch.float64) / hd)
    ang = pos[:, None] * freqs[None, :]                    # [T, hd/2]

    def rot(x):                                            # x [B,T,H,hd]
        z = torch.complex(x[..., : hd // 2], x[..., hd // 2:])
        w = torch.polar(torch.ones_like(ang), ang)[None, :, None, :]
        r = z * w
        return torch.cat([r.real, r.imag], dim=-1)

    gt = 2 * torch.sigmoid(a)
    krec = rot(F.rms_norm(rk.reshape(B, T, H, hd), (hd,), eps=1e-6))
    kb = gt[0][None, None, :, None] * rot(k) + gt[1][None, None, :, None] * krec
    vb = gt[2][None, None, :, None] * v + gt[3][None, None, :, None] * rv.reshape(B, T, H, hd)
    o = F.scaled_dot_product_attention(rot(q).transpose(1, 2), kb.transpose(1, 2), vb.transpose(1, 2),
                                       attn_mask=torch.from_numpy(band(T, W)))
    o.transpose(1, 2).backward(torch.from_numpy(L["dout"]))
    for name, tg in [("dq", q), ("dk", k), ("dv", v), ("dR_k", rk), ("dR_v", rv), ("dgate", a)]:
        np.testing.assert_allclose(g[name], tg.grad.numpy(), rtol=1e-10, atol=1e-11, err_msg=name)


def test_mem_project_backward_matches_autograd():
    m, wk, wv = rand(2, 5, 6), rand(8, 6), rand(8, 6)
    dk, dv = rand(2, 5, 8), rand(2, 5, 8)
    tm, tk, tv = (torch.from_numpy(x).requires_grad_(True) for x in (m, wk, wv))
    ((tm @ tk.T) * torch.from_numpy(dk)).sum().add(((tm @ tv.T) * torch.from_numpy(dv)).sum()).backward()
    dm, dWk, dWv = oracle.mem_project_backward(m, wk, wv, dk, dv)
    np.testing.assert_allclose(dm, tm.grad.numpy(), rtol=1e-12)
    np.testing.assert_allclose(dWk, tk.grad.numpy(), rtol=1e-12)
    np.testing.assert_allclose(dWv, tv.grad.numpy(), rtol=1e-12)


# ---------------------------------------------------------------- stack (Q -> memory -> P -> loss)
def _stack(B=1, T=7, H=1, hd=4, nq=2, np_=2, variant="shared"):
    """variant: "shared" (one W^rec, four gates), "per_layer" (each P layer its
    own W^rec), "kv_gates" (one W^rec, [2, H] gates shared by K and V)."""
    D = H * hd
    ng = 2 if variant == "kv_gates" else 4
    ql = [dict(q=rand(B, T, H, hd), k=rand(B, T, H, hd), v=rand(B, T, H, hd), dout=rand(B, T, H, hd),
               window=3 if i % 2 == 0 else T) for i in range(nq)]
    pl = [dict(q=rand(B, T, H, hd), k=rand(B, T, H, hd), v=rand(B, T, H, hd), dout=rand(B, T, H, hd),
               gates=RNG.uniform(-2, 2, (ng, H)), window=3) for _ in range(np_)]
    if variant == "per_layer":
        for L in pl:
            L["w_mk"], L["w_mv"] = rand(D, D) / np.sqrt(D), rand(D, D) / np.sqrt(D)
        return ql, pl, None, None
    return ql, pl, rand(D, D) / np.sqrt(D), rand(D, D) / np.sqrt(D)


def _stack_objective(ql, pl, wk, wv, lam):
    r = oracle.stack_forward_backward(ql, pl, wk, wv, lam)
    j = r["loss"]
    for L, o in zip(ql, r["q_out"]):
        j += np.sum(o * L["dout"])
    for L, o in zip(pl, r["p_out"]):
        j += np.sum(o * L["dout"])
    return j


def test_shift_memory_and_state():
    m = rand(2, 5, 3)
    s = oracle.shift_memory(m)
    assert np.all(s[:, 0] == 0) and np.array_equal(s[:, 1:], m[:, :-1])
    o = rand(2, 5, 6)
    ref = F.rms_norm(torch.from_numpy(o), (6,), eps=1e-6).numpy()
    np.testing.assert_allclose(oracle.memory_state(o), ref, rtol=1e-13)


@pytest.mark.parametrize("variant", ["shared", "per_layer", "kv_gates"])
def test_stack_central_differences(variant):
    """Every gradient of the stack objective, including the path from P's loss
    and injection back through the shift into Q's last layer; for one shared
    W^rec, a W^rec per decoder layer, and gates shared by K and V."""
    ql, pl, wk, wv = _stack(np_=3 if variant == "per_layer" else 2, variant=variant)
    lam = 0.7
    r = oracle.stack_forward_backward(ql, pl, wk, wv, lam)
    cases = []
    for li in range(len(ql)):
        for key in ("q", "k", "v"):
            cases.append((("q", li, key), r["q_grads"][li]["d" + key]))
    for li in range(len(pl)):
        for key in ("q", "k", "v"):
            cases.append((("p", li, key), r["p_grads"][li]["d" + key]))
        cases.append((("p", li, "gates"), r["p_grads"][li]["dgate"]))
        if variant == "per_layer":
            cases += [(("p", li, "w_mk"), r["p_grads"][li]["dw_mk"]), (("p", li, "w_mv"), r["p_grads"][li]["dw_mv"])]
    if variant != "per_layer":
        cases += [(("w", 0, "wk"), r["dw_mk"]), (("w", 0, "wv"), r["dw_mv"])]
    h = 1e-6
    for (side, li, key), grad in cases:
        for idx in [tuple(RNG.integers(0, s) for s in grad.shape) for _ in range(3)]:
            def j_at(delta):
                ql2 = [{k: (v.copy() if isinstance(v, np.ndarray) else v) for k, v in L.items()} for L in ql]
                pl2 = [{k: (v.copy() if isinstance(v, np.ndarray) else v) for k, v in L.items()} for L in pl]
                wk2 = wk.copy() if wk is not None else None
                wv2 = wv.copy() if wv is not None else None
                if side == "q":
                    ql2[li][key][idx] += delta
                elif side == "p":
                    pl2[li][key][idx] += delta
                else:
                    (wk2 if key == "wk" else wv2)[idx] += delta
                return _stack_objective(ql2, pl2, wk2, wv2, lam)
            fd = (j_at(h) - j_at(-h)) / (2 * h)
            assert abs(fd - grad[idx]) <= 1e-6 * max(1.0, abs(fd)), (side, li, key, idx, fd, grad[idx])


def test_shared_kv_gates_equal_four_equal_gates():
    """The shared K/V form is the four-gate form with the value's logits set
    equal to the key's; its gradient is the sum of the two shares."""
    B, T, H, hd, W = 1, 9, 2, 4, 3
    q, k, v, dout = (rand(B, T, H, hd) for _ in range(4))
    Rk, Rv = rand(B, T, H * hd), rand(B, T, H * hd)
    g2 = RNG.uniform(-2, 2, (2, H))
    g4 = np.concatenate([g2, g2])
    f2 = oracle.inject_swa_forward(q, k, v, Rk, Rv, g2, W)
    f4 = oracle.inject_swa_forward(q, k, v, Rk, Rv, g4, W)
    assert np.array_equal(f2["out"], f4["out"])
    d2 = oracle.inject_swa_backward(q, k, v, Rk, Rv, g2, dout, W)["dgate"]
    d4 = oracle.inject_swa_backward(q, k, v, Rk, Rv, g4, dout, W)["dgate"]
    assert d2.shape == (2, H)
    np.testing.assert_allclose(d2, d4[:2] + d4[2:], rtol=1e-14)


def test_per_layer_projection_with_equal_weights_equals_shared():
    """Giving every decoder layer the same W^rec reproduces the shared form:
    the per-layer dW^l sum to the shared dW."""
    ql, pl, wk, wv = _stack(np_=3)
    r = oracle.stack_forward_backward(ql, pl, wk, wv, 0.3)
    pl2 = [dict(L, w_mk=wk, w_mv=wv) for L in pl]
    r2 = oracle.stack_forward_backward(ql, pl2, None, None, 0.3)
    np.testing.assert_allclose(r2["loss"], r["loss"], rtol=1e-14)
    np.testing.assert_allclose(sum(g["dw_mk"] for g in r2["p_grads"]), r["dw_mk"], rtol=1e-10, atol=1e-13)
    np.testing.assert_allclose(r2["dm_shift"], r["dm_shift"], rtol=1e-10, atol=1e-13)


def test_stack_gates_off_decouples_memory():
    """With both recurrent gates shut (a = -inf) P ignores the memory: P's
    outputs are plain SWA, the projection gets no gradient, and Q's last layer
    sees only its own dout plus the loss's target term."""
    ql, pl, wk, wv = _stack(T=9)
    for L in pl:
        L["gates"][1] = -np.inf
        L["gates"][3] = -np.inf
        L["gates"][0] = 0.0
        L["gates"][2] = 0.0
    r = oracle.stack_forward_backward(ql, pl, wk, wv, 0.5)
    for L, o in zip(pl, r["p_out"]):
        plain = oracle.inject_swa_forward(L["q"], L["k"], L["v"], None, None, None, L["window"], inject=False)
        assert np.array_equal(o, plain["out"])
    assert np.all(r["dw_mk"] == 0) and np.all(r["dw_mv"] == 0) and np.all(r["dm_shift"] == 0)
    B, T, H, hd = ql[-1]["q"].shape
    oq = r["q_out"][-1].reshape(B, T, H * hd)
    _, _, dmp = oracle.consistency_loss(r["m"].reshape(B * T, -1), r["m_prime"].reshape(B * T, -1), 0.5)
    want = ql[-1]["dout"] + oracle.rmsnorm_backward(oq, dmp.reshape(B, T, -1), 1e-6).reshape(B, T, H, hd)
    np.testing.assert_allclose(r["q_grads"][-1]["dout"], want, rtol=1e-13, atol=1e-13)


# ---------------------------------------------------------------- consistency loss
def test_consistency_loss_closed_forms():
    rows, d = 7, 64
    m = rand(rows, d)
    loss, dm, dmt = oracle.consistency_loss(m, m.copy(), 0.1)
    assert loss == 0.0 and np.all(dm == 0)
    c, lam = 0.5, 0.1
    loss, dm, dmt = oracle.consistency_loss(m + c, m, lam)
    # per row ||c 1||^2 / sqrt(d) = c^2 sqrt(d); averaged over rows (|I| = rows)
    assert abs(loss - lam * c * c * math.sqrt(d)) < 1e-13
    np.testing.assert_allclose(dm, 2 * lam * c / (rows * math.sqrt(d)), rtol=1e-13)
    np.testing.assert_array_equal(dmt, -dm)
    loss2, _, _ = oracle.consistency_loss(m + c, m, lam, inv_count=1.0)
    assert abs(loss2 - rows * loss) < 1e-12


# ---------------------------------------------------------------- decode
def test_decode_equals_teacher_forced_row():
    # Recurrence = training form when fed the same memory (rainbus 研究动机 interface):
    # ring filled with the forward's mixed entries for p-W+1..p-1, then one decode
    # step at p reproduces the forward's row p.
    B, T, H, hd, d, W = 1, 40, 2, 8, 12, 8
    L = layer(B, T, H, hd, d)
    Rk, Rv = oracle.mem_project(L["m"], L["wk"], L["wv"])
    f = oracle.inject_swa_forward(L["q"], L["k"], L["v"], Rk, Rv, L["a"], W)
    for p in (0, 3, W - 1, W, W + 5, 2 * W + 1, T - 1):
        kr = rand(B, H, W, hd)     # garbage in dead / stale slots
        vr = rand(B, H, W, hd)
        for j in range(max(0, p - W + 1), p):
            kr[0, :, j % W] = f["k_bar"][0, j]
            vr[0, :, j % W] = f["v_bar"][0, j]
        krec, vrec = oracle.decode_mem_project(np.array([p]), L["m"][:, p], L["wk"], L["wv"], H)
        out, kr2, vr2 = oracle.decode_step(np.array([p]), L["q"][:, p], L["k"][:, p], L["v"][:, p],
                                           krec, vrec, L["a"], kr, vr)
        np.testing.assert_allclose(out[0], f["out"][0, p], atol=1e-12)
        np.testing.assert_allclose(kr2[0, :, p % W], f["k_bar"][0, p], atol=1e-12)


def test_decode_ring_update_touches_one_slot():
    B, H, W, hd, d = 3, 2, 8, 4, 6
    pos = np.array([5, 8, 21])
    kr, vr = rand(B, H, W, hd), rand(B, H, W, hd)
    q, k, v = rand(B, H, hd), rand(B, H, hd), rand(B, H, hd)
    krec, vrec = rand(B, H, hd), rand(B, H, hd)
    out, kr2, vr2 = oracle.decode_step(pos, q, k, v, krec, vrec, RNG.uniform(-2, 2, (4, H)), kr, vr)
    for b in range(B):
        s = pos[b] % W
        keep = [x for x in range(W) if x != s]
        np.testing.assert_array_equal(kr2[b][:, keep], kr[b][:, keep])
        np.testing.assert_array_equal(vr2[b][:, keep], vr[b][:, keep])
        assert np.abs(kr2[b][:, s] - kr[b][:, s]).max() > 0


def test_decode_prefix_ignores_dead_slots():
    # p < W-1: only slots 0..p are live; the rest must not matter.
    B, H, W, hd = 1, 1, 8, 4
    pos = np.array([2])
    kr, vr = rand(B, H, W, hd), rand(B, H, W, hd)
    args = (rand(B, H, hd), rand(B, H, hd), rand(B, H, hd), rand(B, H, hd), rand(B, H, hd), np.zeros((4, H)))
    o1, _, _ = oracle.decode_step(pos, *args, kr, vr)
    kr[:, :, 3:] += 5.0
    vr[:, :, 3:] -= 5.0
    o2, _, _ = oracle.decode_step(pos, *args, kr, vr)
    np.testing.assert_array_equal(o1, o2)


def test_synth_inputs_are_seeded_and_sliceable():
    wl = synth.WORKLOADS["tiny_f32"]
    a = synth.layer_inputs(wl, 1234)
    b = synth.layer_inputs(wl, 1234)
    c = synth.layer_inputs(wl, 1235)
    np.testing.assert_array_equal(a["q"].bits, b["q"].bits)
    assert not np.array_equal(a["q"].bits, c["q"].bits)
    assert np.all(a["mtraj"].f64[:, 0] == 0)          # m'_0 = 0
    np.testing.assert_array_equal(a["m_shift"].f64[:, 1:], a["mtraj"].f64[:, 1:-1])
    x = np.array([1.0, 1.00390625, 1.005859375, -3.14159], dtype=np.float32)
    bits = synth.round_to_bf16_bits(x)
    np.testing.assert_array_equal(synth.bf16_bits_to_f64(bits), [1.0, 1.0, 1.0078125, -3.140625])


# ---------------------------------------------------------------- LM head, softcapped CE
def test_lm_head_zero_weights_give_log_vocab():
    """U = 0: every logit is 0, the softmax is uniform and each token's CE is
    log V exactly; dm is 0 and dU = -(1/N) sum_t (onehot - 1/V) m_t^T."""
    N, d, V = 5, 8, 11
    m = rand(N, d)
    y = RNG.integers(0, V, N)
    loss, lse, dm, dU = oracle.lm_head_ce(m, np.zeros((V, d)), y)
    np.testing.assert_allclose(loss, np.log(V), rtol=1e-15)
    np.testing.assert_allclose(lse, np.log(V), rtol=1e-15)
    assert np.all(dm == 0)
    oh = np.zeros((N, V))
    oh[np.arange(N), y] = 1.0
    np.testing.assert_allclose(dU, ((1.0 / V - oh) / N).T @ m, rtol=1e-13, atol=1e-15)


def test_lm_head_softcap_limits():
    """The cap bounds every logit: a huge raw logit saturates at +15 (its
    probability then e^15 / (e^15 + (V-1) e^c_other)), and the cap's slope is
    1 at 0 and vanishes in saturation."""
    d, V = 4, 3
    m = np.array([[1.0, 0, 0, 0]])
    U = np.zeros((V, d))
    U[0, 0] = 1e6                                     # z = (1e6, 0, 0)
    loss, lse, _, dU = oracle.lm_head_ce(m, U, np.array([1]))
    np.testing.assert_allclose(lse[0], np.log(np.exp(15.0) + 2.0), rtol=1e-14)
    np.testing.assert_allclose(loss, lse[0] - 0.0, rtol=1e-14)
    assert abs(dU[0, 0]) < 1e-300                     # tanh' = 0 in saturation
    # small logits: softcap(z) = z to third order, so the CE matches the plain one
    U2 = rand(V, d) * 1e-3
    l_cap = oracle.lm_head_ce(m, U2, np.array([2]))[0]
    z = (m @ U2.T)[0]
    l_plain = np.log(np.sum(np.exp(z))) - z[2]
    assert abs(l_cap - l_plain) < 1e-9


def test_lm_head_matches_torch_cross_entropy_and_autograd():
    """Loss against torch's cross_entropy of the softcapped logits, gradients
    against autograd through matmul, tanh and cross_entropy (fp64)."""
    N, d, V = 6, 10, 17
    m, U = rand(N, d), rand(V, d)
    y = RNG.integers(0, V, N)
    loss, lse, dm, dU = oracle.lm_head_ce(m, U, y, inv_count=1.0 / 4)
    tm = torch.from_numpy(m).requires_grad_(True)
    tU = torch.from_numpy(U).requires_grad_(True)
    c = 15.0 * torch.tanh((tm @ tU.T) / 15.0)
    tl = F.cross_entropy(c, torch.from_numpy(y), reduction="sum") / 4
    tl.backward()
    np.testing.assert_allclose(loss, tl.item(), rtol=1e-13)
    np.testing.assert_allclose(lse, torch.logsumexp(c, 1).detach().numpy(), rtol=1e-13)
    np.testing.assert_allclose(dm, tm.grad.numpy(), rtol=1e-11, atol=1e-14)
    np.testing.assert_allclose(dU, tU.grad.numpy(), rtol=1e-11, atol=1e-14)


def test_lm_head_central_differences():
    N, d, V = 4, 6, 9
    m, U = rand(N, d) * 3, rand(V, d) * 3               # large enough for the cap to bend
    y = RNG.integers(0, V, N)
    _, _, dm, dU = oracle.lm_head_ce(m, U, y)
    h = 1e-6
    for arr, grad in ((m, dm), (U, dU)):
        for _ in range(6):
            idx = tuple(RNG.integers(0, s) for s in arr.shape)
            a0 = arr[idx]
            arr[idx] = a0 + h
            lp = oracle.lm_head_ce(m, U, y)[0]
            arr[idx] = a0 - h
            lm = oracle.lm_head_ce(m, U, y)[0]
            arr[idx] = a0
            fd = (lp - lm) / (2 * h)
            assert abs(fd - grad[idx]) <= 1e-7 * max(1.0, abs(fd)), (idx, fd, grad[idx])


def test_gate_gradient_scale_bounds_the_sum():
    """dgate_scale is the RMS size sqrt(sum t^2) of the B*T*hd products t each
    gate gradient sums (times the gate's slope): by Cauchy-Schwarz
    |dgate| <= sqrt(B*T*hd) * dgate_scale, with equality when all products are
    equal; with the shared K/V form the two shares' scales add in quadrature."""
    B, T, H, hd, W = 1, 9, 2, 4, 3
    q, k, v, dout = (rand(B, T, H, hd) for _ in range(4))
    Rk, Rv = rand(B, T, H * hd), rand(B, T, H * hd)
    g4 = RNG.uniform(-2, 2, (4, H))
    r = oracle.inject_swa_backward(q, k, v, Rk, Rv, g4, dout, W)
    assert np.all(np.abs(r["dgate"]) <= np.sqrt(B * T * hd) * r["dgate_scale"] * (1 + 1e-12))
    assert np.all(r["dgate_scale"] > 0)
    r2 = oracle.inject_swa_backward(q, k, v, Rk, Rv, g4[:2], dout, W)
    r4 = oracle.inject_swa_backward(q, k, v, Rk, Rv, np.concatenate([g4[:2], g4[:2]]), dout, W)
    np.testing.assert_allclose(r2["dgate_scale"], np.sqrt(r4["dgate_scale"][:2] ** 2 + r4["dgate_scale"][2:] ** 2),
                               rtol=1e-13)
