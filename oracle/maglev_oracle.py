"""Plain float64 CPU oracle of Maglev's injected sliding-window attention.

TEST INFRASTRUCTURE ONLY. Only tests/, __graft_entry__.smoke() and bench.py's
cpu_baseline / reference legs may import or run this module. The CUDA path
never calls it, and it shares no code with the CUDA path.

Source: "Maglev: Sliding Recurrent Memory" (arXiv 2608.02870), as summarised on
  [rainbus]  paper.rainbus.top/paper/2608.02870 -- sections 前置知识 (SWA, KV
             cache, RoPE), 研究动机 (the interface p(x_{t+1}, m_t | x_{t-W+1:t},
             M_{t-1})), 核心方法 and 方法步骤详情 (every formula used here);
  [gist]     gist.science/nl/paper/2608.02870 -- section Inferentiemechanisme
             (injection through learned projections and gating, no extra cache).

What the method computes (rainbus, 方法步骤详情): at position t of decoder layer l
the shifted memory m'_{t-1} (m'_0 = 0) passes through projections shared across
layers, k_rec = RMSNorm(W_k^rec m'_{t-1}) and v_rec = W_v^rec m'_{t-1}; both the
local key and k_rec are RoPE-rotated (前置知识 / 方法步骤详情: rotate both keys
before mixing); a per-layer gate g = 2*sigmoid(a) (neutral 1 at a = 0) mixes them
into the position's own K/V entry, k_bar = g_loc*k + g_rec*k_rec (v_bar likewise);
the layer attends over the most recent W mixed entries. The loss adds
lambda*||m_t - m'_t||^2 / sqrt(d), averaged over the positions in I.

Readings where the pages leave a step open (each is listed in the design notes):
  * gates: four per-head scalar logits per layer [4, H] = (k_loc, k_rec, v_loc,
    v_rec), each g = 2*sigmoid(a); a = -inf gives g = 0 exactly;
  * RMSNorm of k_rec: per head over hd channels, no weight, eps added to the
    mean square; the local q/k get no norm;
  * RoPE: half-split pairs (c, c + hd/2), theta_c = base^(-2c/hd), angle p*theta_c
    at the entry's absolute position p;
  * window: keys j in [i-W+1, i] (W keys, self included); scale 1/sqrt(hd);
  * decode: write the new entry to ring slot p mod W, then attend over the
    min(p+1, W) live slots.

Every array is float64; inputs arrive as the exact float64 values of the
bf16/f32 arrays the GPU gets. Nothing here is blocked, fused or reordered
beyond the definitions.
"""
from __future__ import annotations

import numpy as np


# --------------------------------------------------------------------------
# Elementary pieces
# --------------------------------------------------------------------------
def sigmoid(a):
    """Logistic function, finite for a = +-inf (sigmoid(-inf) = 0)."""
    a = np.asarray(a, dtype=np.float64)
    out = np.empty_like(a)
    pos = a >= 0
    out[pos] = 1.0 / (1.0 + np.exp(-a[pos]))
    e = np.exp(a[~pos])
    out[~pos] = e / (1.0 + e)
    return out


def gate(a):
    """g = 2*sigmoid(a): neutral value 1 at a = 0 (rainbus, 方法步骤详情)."""
    return 2.0 * sigmoid(a)


def gate_slope(a):
    """dg/da = 2*sigmoid(a)*(1 - sigmoid(a)); 0 at a = +-inf."""
    s = sigmoid(a)
    return 2.0 * s * (1.0 - s)


def gate_rows(gate_logits):
    """The four per-head gate logits (k_loc, k_rec, v_loc, v_rec) as a [4, H]
    array. rainbus, 方法步骤详情, gives the key's gates and says the value is
    mixed "likewise"; a [2, H] argument is the reading in which the value reuses
    the key's two gates (shared K/V gates: rows loc, rec)."""
    a = np.asarray(gate_logits, dtype=np.float64)
    return np.concatenate([a, a]) if a.shape[0] == 2 else a


def fold_gate_grads(dgate4, gate_logits):
    """Gradient of the logits as given: [4, H] as is, or for shared K/V gates
    [2, H] the sum of the key's and the value's share of each gate."""
    return dgate4[:2] + dgate4[2:] if np.asarray(gate_logits).shape[0] == 2 else dgate4


def rope_angles(pos, hd: int, base: float):
    """angle[..., c] = pos * base^(-2c/hd), c = 0..hd/2-1 (rainbus, 前置知识: RoPE)."""
    c = np.arange(hd // 2, dtype=np.float64)
    inv_freq = base ** (-2.0 * c / hd)
    return np.asarray(pos, dtype=np.float64)[..., None] * inv_freq


def rope(x, pos, base: float, inverse: bool = False):
    """Rotate pairs (x_c, x_{c+hd/2}) of x[..., hd] by the angle at position pos.

    pos broadcasts against x.shape[:-1]. inverse=True applies the transpose
    (rotation by the negative angle), used by the backward pass.
    """
    hd = x.shape[-1]
    ang = rope_angles(pos, hd, base)
    cos, sin = np.cos(ang), np.sin(ang)
    if inverse:
        sin = -sin
    x1, x2 = x[..., : hd // 2], x[..., hd // 2:]
    return np.concatenate([x1 * cos - x2 * sin, x1 * sin + x2 * cos], axis=-1)


def rmsnorm(x, eps: float):
    """x / sqrt(mean(x^2) + eps) over the last axis, no weight."""
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)


def rmsnorm_backward(x, dy, eps: float):
    """Gradient of rmsnorm(x) w.r.t. x, given dy: (dy - y * mean(y*dy)) / r."""
    r = np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    y = x / r
    return (dy - y * np.mean(y * dy, axis=-1, keepdims=True)) / r


def window_mask(T: int, window: int, offset: int = 0):
    """mask[i, j] = True iff key j is in query i's window: i-W+1 <= j <= i.

    (rainbus, 前置知识: each position attends to the most recent W tokens;
    研究动机: the window x_{t-W+1:t} holds W tokens, the current one included.)
    """
    i = np.arange(T)[:, None] + offset
    j = np.arange(T)[None, :] + offset
    return (j <= i) & (j >= i - window + 1)


# --------------------------------------------------------------------------
# a1: memory projection (shared across layers: no layer index on W^rec)
# --------------------------------------------------------------------------
def mem_project(m_shift, w_mk, w_mv):
    """R_k = m_shift W_mk^T, R_v = m_shift W_mv^T. m_shift [..., d], W [D, d]."""
    return m_shift @ w_mk.T, m_shift @ w_mv.T


def mem_project_backward(m_shift, w_mk, w_mv, dR_k, dR_v):
    """dm_shift = dR_k W_mk + dR_v W_mv; dW = dR^T m_shift summed over rows."""
    d = m_shift.shape[-1]
    D = w_mk.shape[0]
    m2 = m_shift.reshape(-1, d)
    dk2 = dR_k.reshape(-1, D)
    dv2 = dR_v.reshape(-1, D)
    dm = dk2 @ w_mk + dv2 @ w_mv
    return dm.reshape(m_shift.shape), dk2.T @ m2, dv2.T @ m2


# --------------------------------------------------------------------------
# a2-a5: injection + sliding-window attention, forward
# --------------------------------------------------------------------------
def inject_swa_forward(q, k, v, R_k, R_v, gate_logits, window: int, pos0: int = 0,
                       rope_base: float = 10000.0, eps: float = 1e-6, inject: bool = True):
    """Forward of one decoder layer's attention with recurrent K/V injection.

    q, k, v: [B, T, H, hd] pre-RoPE local projections.
    R_k, R_v: [B, T, H*hd] projected shifted memory (row t uses m'_{t-1}).
    gate_logits: [4, H] = (k_loc, k_rec, v_loc, v_rec), or [2, H] = (loc, rec)
    shared by the key and the value (see gate_rows).
    Returns a dict with out [B,T,H,hd], lse [B,H,T] and the intermediates.
    """
    B, T, H, hd = q.shape
    pos = pos0 + np.arange(T)                                 # absolute positions
    posb = np.broadcast_to(pos[None, :, None], (B, T, H))
    q_rot = rope(q, posb, rope_base)
    k_loc = rope(k, posb, rope_base)
    res = {"q_rot": q_rot, "k_loc": k_loc}
    if inject:
        g = gate(gate_rows(gate_logits))                      # [4, H]
        Rk = R_k.reshape(B, T, H, hd)
        Rv = R_v.reshape(B, T, H, hd)
        n = rmsnorm(Rk, eps)                                  # per head, hd channels
        k_rec = rope(n, posb, rope_base)                      # rotate before mixing
        k_bar = g[0][None, None, :, None] * k_loc + g[1][None, None, :, None] * k_rec
        v_bar = g[2][None, None, :, None] * v + g[3][None, None, :, None] * Rv
        res.update(k_rec=k_rec, n=n, g=g)
    else:
        k_bar, v_bar = k_loc, v
    out = np.empty_like(q)
    lse = np.empty((B, H, T))
    for b in range(B):
        for h in range(H):
            P, lse[b, h] = attention_probs(q_rot[b, :, h], k_bar[b, :, h], window)
            out[b, :, h] = P @ v_bar[b, :, h]
    res.update(out=out, lse=lse, k_bar=k_bar, v_bar=v_bar)
    return res


def attention_probs(q_rot, k_bar, window: int):
    """P = softmax(q_rot k_bar^T / sqrt(hd) restricted to the window), and its
    log-sum-exp per row. q_rot, k_bar: [T, hd] of one (batch, head)."""
    T, hd = q_rot.shape
    S = (q_rot @ k_bar.T) / np.sqrt(hd)
    S = np.where(window_mask(T, window), S, -np.inf)
    mx = S.max(axis=1, keepdims=True)          # finite: the diagonal is always in the window
    E = np.exp(S - mx)
    Z = E.sum(axis=1, keepdims=True)
    return E / Z, (mx + np.log(Z))[:, 0]


# --------------------------------------------------------------------------
# a6: backward (chain rule of the forward above, derived by hand)
# --------------------------------------------------------------------------
def inject_swa_backward(q, k, v, R_k, R_v, gate_logits, dout, window: int, pos0: int = 0,
                        rope_base: float = 10000.0, eps: float = 1e-6, inject: bool = True):
    """Gradients of <out, dout> w.r.t. q, k, v, R_k, R_v and the gate logits."""
    B, T, H, hd = q.shape
    f = inject_swa_forward(q, k, v, R_k, R_v, gate_logits, window, pos0, rope_base, eps, inject)
    scale = 1.0 / np.sqrt(hd)
    dq_rot = np.empty_like(q)
    dk_bar = np.empty_like(q)
    dv_bar = np.empty_like(q)
    for b in range(B):
        for h in range(H):
            P, _ = attention_probs(f["q_rot"][b, :, h], f["k_bar"][b, :, h], window)
            dO = dout[b, :, h]
            dv_bar[b, :, h] = P.T @ dO                       # dV = P^T dO
            dP = dO @ f["v_bar"][b, :, h].T                  # dP = dO V^T
            dS = P * (dP - np.sum(P * dP, axis=1, keepdims=True))
            dq_rot[b, :, h] = (dS @ f["k_bar"][b, :, h]) * scale
            dk_bar[b, :, h] = (dS.T @ f["q_rot"][b, :, h]) * scale
    pos = pos0 + np.arange(T)
    posb = np.broadcast_to(pos[None, :, None], (B, T, H))
    dq = rope(dq_rot, posb, rope_base, inverse=True)
    out = {"dq": dq, "dq_rot": dq_rot, "dk_bar": dk_bar, "dv_bar": dv_bar, "fwd": f}
    if inject:
        g = f["g"]
        gk_l, gk_r, gv_l, gv_r = (g[i][None, None, :, None] for i in range(4))
        out["dk"] = gk_l * rope(dk_bar, posb, rope_base, inverse=True)
        out["dv"] = gv_l * dv_bar
        dn = rope(gk_r * dk_bar, posb, rope_base, inverse=True)
        Rk = R_k.reshape(B, T, H, hd)
        out["dR_k"] = rmsnorm_backward(Rk, dn, eps).reshape(B, T, H * hd)
        out["dR_v"] = (gv_r * dv_bar).reshape(B, T, H * hd)
        terms = [dk_bar * f["k_loc"], dk_bar * f["k_rec"], dv_bar * v, dv_bar * R_v.reshape(B, T, H, hd)]
        dg = np.stack([np.sum(t, axis=(0, 1, 3)) for t in terms])
        slope = gate_slope(gate_rows(gate_logits))
        out["dgate"] = fold_gate_grads(dg * slope, gate_logits)
        # Scale of each gate gradient's rounding error: each is a sum of B*T*hd
        # products, whose rounding error grows with the RMS size of the summands
        # (sqrt of the sum of their squares), not with the sum itself, which can
        # cancel. Test infrastructure: not a quantity of the method.
        sc2 = np.stack([np.sum(t * t, axis=(0, 1, 3)) for t in terms]) * slope ** 2
        out["dgate_scale"] = np.sqrt(fold_gate_grads(sc2, gate_logits))
    else:
        out["dk"] = rope(dk_bar, posb, rope_base, inverse=True)
        out["dv"] = dv_bar
    return out


# --------------------------------------------------------------------------
# a7: consistency loss
# --------------------------------------------------------------------------
def consistency_loss(m, m_target, lam: float, inv_count: float | None = None):
    """L = lam/|I| * sum_t ||m_t - m'_t||^2 / sqrt(d)  (rainbus, 方法步骤详情).

    m, m_target: [rows, d]; inv_count = 1/|I| (default 1/rows).
    Returns (L, dL/dm, dL/dm_target).
    """
    rows, d = m.shape
    if inv_count is None:
        inv_count = 1.0 / rows
    diff = m - m_target
    loss = lam * inv_count * np.sum(diff * diff) / np.sqrt(d)
    dm = 2.0 * lam * inv_count * diff / np.sqrt(d)
    return loss, dm, -dm


# --------------------------------------------------------------------------
# LM head with softcapped logits and cross-entropy
# --------------------------------------------------------------------------
def lm_head_ce(m, U, targets, softcap: float = 15.0, inv_count: float | None = None):
    """Per-token next-token loss of the memory state (rainbus, 方法步骤详情):
    p(x_{t+1} | x_<=t) = softmax(c_t), c_t = softcap * tanh(U m_t / softcap)
    with softcap = 15, and the loss (1/|I|) sum_t CE_t with
    CE_t = -log p(targets_t) = logsumexp(c_t) - c_t[targets_t].

    m [N, d], U [V, d], targets [N] int. inv_count = 1/|I| (default 1/N).
    Returns (loss, lse [N], dm [N, d], dU [V, d]): by the chain rule,
    dL/dc_t = inv_count (softmax(c_t) - onehot(targets_t)) and
    dc/dz = 1 - tanh(z / softcap)^2 for the raw logits z = U m_t.
    """
    N = m.shape[0]
    if inv_count is None:
        inv_count = 1.0 / N
    z = m @ U.T                                        # [N, V] raw logits
    t = np.tanh(z / softcap)
    c = softcap * t
    mx = c.max(axis=1, keepdims=True)
    lse = (mx + np.log(np.sum(np.exp(c - mx), axis=1, keepdims=True)))[:, 0]
    rows = np.arange(N)
    ce = lse - c[rows, targets]
    loss = inv_count * np.sum(ce)
    dc = np.exp(c - lse[:, None])                      # softmax(c_t)
    dc[rows, targets] -= 1.0
    dc *= inv_count
    dz = dc * (1.0 - t * t)
    return loss, lse, dz @ U, dz.T @ m


# --------------------------------------------------------------------------
# stack: prefiller Q and decoder P around one shared memory
# --------------------------------------------------------------------------
def memory_state(o, eps: float = 1e-6):
    """m_t = RMSNorm(o_t) over the d channels of each row (rainbus, 方法步骤详情:
    the memory is the stack's final state after RMSNorm; no weight). o [B,T,d]."""
    return rmsnorm(o, eps)


def shift_memory(m):
    """The memory read at position t is m_{t-1}; row 0 reads m_0 = 0
    (rainbus, 方法步骤详情). m [B,T,d] -> [B,T,d]."""
    out = np.zeros_like(m)
    out[:, 1:] = m[:, :-1]
    return out


def stack_forward_backward(q_layers, p_layers, w_mk, w_mv, lam: float, rope_base: float = 10000.0,
                           eps: float = 1e-6, store=None, inv_count: float | None = None):
    """One training step of a prefiller Q and a decoder P that share a memory.

    Q's layers (no injection; dicts with q, k, v, dout, window) run first;
    m' = RMSNorm(O of Q's last layer) is its memory, and P reads the shifted
    memory m_shift = shift(m') through one projection shared by every layer
    (rainbus, 方法步骤详情: 共享投影, rows t read m'_{t-1}). P's layers (dicts with
    q, k, v, gates, dout, window) run injected; m = RMSNorm(O of P's last
    layer) meets m' in the consistency loss. The objective is
        J = sum over all layers <O_l, dout_l> + L_cons(m, m').
    Every layer has d = H * hd channels. Returns the forward values and the
    gradients of J (chain rule through the functions above).
    `store` (optional) maps the combined upstream gradient of each last layer
    (its dout plus the memory's gradient) to the values kept in storage, for
    comparison with an implementation that keeps it in a narrower type.
    `inv_count` is the loss's 1/|I| (default 1/(B*T)); batch rows are
    independent apart from |I| and the sums over rows (loss, dW, gate grads),
    so a slice of rows with the full batch's |I| reproduces those rows.
    Per-layer memory projection (rainbus, 未来方向: 逐层记忆投影): when every P
    layer dict carries its own w_mk, w_mv, layer l reads R^l = m_shift W^l^T,
    the shifted memory's gradient is the sum of every layer's dR^l W^l, and
    each layer's dW^l is returned in its p_grads entry (w_mk, w_mv unused).
    """
    store = store if store is not None else (lambda x: x)
    B, T, H, hd = q_layers[-1]["q"].shape
    D = H * hd
    per_layer = all("w_mk" in L for L in p_layers)
    qf = [inject_swa_forward(L["q"], L["k"], L["v"], None, None, None, L["window"], 0, rope_base, eps,
                             inject=False) for L in q_layers]
    oq = qf[-1]["out"].reshape(B, T, D)
    m_prime = memory_state(oq, eps)
    m_shift = shift_memory(m_prime)
    if per_layer:
        Rs = [mem_project(m_shift, L["w_mk"], L["w_mv"]) for L in p_layers]
    else:
        Rs = [mem_project(m_shift, w_mk, w_mv)] * len(p_layers)
    R_k, R_v = Rs[0]
    pf = [inject_swa_forward(L["q"], L["k"], L["v"], Rs[i][0], Rs[i][1], L["gates"], L["window"], 0, rope_base,
                             eps) for i, L in enumerate(p_layers)]
    op = pf[-1]["out"].reshape(B, T, D)
    m = memory_state(op, eps)
    loss, dm, dm_prime = consistency_loss(m.reshape(B * T, D), m_prime.reshape(B * T, D), lam, inv_count)
    dm = dm.reshape(B, T, D)
    dm_prime = dm_prime.reshape(B, T, D)

    # P: the last layer also receives the loss through RMSNorm
    p_grads = []
    dR_k = np.zeros_like(R_k)
    dR_v = np.zeros_like(R_v)
    dm_shift = np.zeros_like(m_shift)
    for i, L in enumerate(p_layers):
        dout = L["dout"]
        if i == len(p_layers) - 1:
            dout = store(dout + rmsnorm_backward(op, dm, eps).reshape(B, T, H, hd))
        g = inject_swa_backward(L["q"], L["k"], L["v"], Rs[i][0], Rs[i][1], L["gates"], dout, L["window"], 0,
                                rope_base, eps)
        grads = {"dq": g["dq"], "dk": g["dk"], "dv": g["dv"], "dgate": g["dgate"], "dgate_scale": g["dgate_scale"],
                 "dout": dout}
        if per_layer:
            dms, dwk, dwv = mem_project_backward(m_shift, L["w_mk"], L["w_mv"], g["dR_k"], g["dR_v"])
            dm_shift += dms
            grads.update(dR_k=g["dR_k"], dR_v=g["dR_v"], dw_mk=dwk, dw_mv=dwv)
        else:
            dR_k += g["dR_k"]
            dR_v += g["dR_v"]
        p_grads.append(grads)
    if per_layer:
        dw_mk = dw_mv = None
    else:
        dm_shift, dw_mk, dw_mv = mem_project_backward(m_shift, w_mk, w_mv, dR_k, dR_v)
    # m_shift[t] = m'[t-1]: its gradient lands one row earlier
    dm_prime = dm_prime.copy()
    dm_prime[:, :-1] += dm_shift[:, 1:]
    q_grads = []
    for i, L in enumerate(q_layers):
        dout = L["dout"]
        if i == len(q_layers) - 1:
            dout = store(dout + rmsnorm_backward(oq, dm_prime, eps).reshape(B, T, H, hd))
        g = inject_swa_backward(L["q"], L["k"], L["v"], None, None, None, dout, L["window"], 0, rope_base, eps,
                                inject=False)
        q_grads.append({"dq": g["dq"], "dk": g["dk"], "dv": g["dv"], "dout": dout})
    return {"loss": loss, "q_out": [f["out"] for f in qf], "p_out": [f["out"] for f in pf],
            "m": m, "m_prime": m_prime, "m_shift": m_shift, "R_k": R_k, "R_v": R_v,
            "q_grads": q_grads, "p_grads": p_grads, "dR_k": dR_k, "dR_v": dR_v,
            "dm_shift": dm_shift, "dw_mk": dw_mk, "dw_mv": dw_mv}


# --------------------------------------------------------------------------
# a8: recurrent decode step over a rolling W-entry ring
# --------------------------------------------------------------------------
def decode_mem_project(pos, m_prev, w_mk, w_mv, H: int, rope_base: float = 10000.0, eps: float = 1e-6):
    """k_rec = RoPE_p(RMSNorm_head(W_mk m_{p-1})), v_rec = W_mv m_{p-1}. m_prev [B, d]."""
    B = m_prev.shape[0]
    D = w_mk.shape[0]
    hd = D // H
    Rk = (m_prev @ w_mk.T).reshape(B, H, hd)
    Rv = (m_prev @ w_mv.T).reshape(B, H, hd)
    posb = np.broadcast_to(np.asarray(pos)[:, None], (B, H))
    return rope(rmsnorm(Rk, eps), posb, rope_base), Rv


def decode_step(pos, q, k, v, krec_rot, vrec, gate_logits, k_ring, v_ring,
                rope_base: float = 10000.0, inject: bool = True):
    """One recurrent step at absolute positions pos[B] (rainbus, 方法步骤详情 and
    研究动机: m_t = P(x_{t-W+1:t}, M_{t-1}); gist, Inferentiemechanisme: the state
    rides in the K/V cache, whose size is that of plain SWA).

    q, k, v [B, H, hd] pre-RoPE; krec_rot, vrec [B, H, hd]; rings [B, H, W, hd]
    hold post-RoPE, post-mix entries. The new entry is written to slot p mod W,
    then q attends over the live slots (positions max(0, p-W+1)..p).
    Returns (out [B,H,hd], k_ring', v_ring'); the inputs are not modified.
    """
    B, H, W, hd = k_ring.shape
    pos = np.asarray(pos, dtype=np.int64)
    posb = np.broadcast_to(pos[:, None], (B, H))
    q_rot = rope(q, posb, rope_base)
    k_loc = rope(k, posb, rope_base)
    if inject:
        g = gate(gate_rows(gate_logits))
        k_new = g[0][None, :, None] * k_loc + g[1][None, :, None] * krec_rot
        v_new = g[2][None, :, None] * v + g[3][None, :, None] * vrec
    else:
        k_new, v_new = k_loc, v
    kr = k_ring.copy()
    vr = v_ring.copy()
    out = np.empty_like(q)
    scale = 1.0 / np.sqrt(hd)
    for b in range(B):
        p = int(pos[b])
        slot = p % W
        kr[b, :, slot] = k_new[b]
        vr[b, :, slot] = v_new[b]
        live = np.arange(W) if p >= W - 1 else np.arange(p + 1)
        for h in range(H):
            s = (kr[b, h, live] @ q_rot[b, h]) * scale
            e = np.exp(s - s.max())
            out[b, h] = (e / e.sum()) @ vr[b, h, live]
    return out, kr, vr
