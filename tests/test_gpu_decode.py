"""Multi-step recurrent decode on the GPU against the oracle, through the C ABI.

One token step of an L-layer decoder: maglev_decode_mem_project(m_{p-1}) once
(W^rec is shared by the layers), then maglev_decode_step per layer over that
layer's own rolling ring; the step's memory m_p is RMSNorm of the last layer's
output (maglev_memory_state) and is fed back into the next step
(paper.rainbus.top, 研究动机: m_t = P(x_{t-W+1:t}, M_{t-1}); 方法步骤详情: m is the
final state after RMSNorm). Each step's per-layer q, k, v are seeded stand-ins
for the model's projections of its residual stream.

Shapes are the benchmark's: 64 sequences, 10 heads of 128, d = 1280, 512-entry
rings pre-filled with seeded N(0,1) entries; two layers (every layer runs the
same kernel on its own ring).
"""
import numpy as np
import pytest

import oracle
import synth
from helpers import TOL, assert_close, dev, host, normwise

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from sliding_window_recurrent_b200 import build as _build
    _build.build(quiet=True)
    import sliding_window_recurrent_b200 as mg

B, H, HD, D, W, L = 64, 10, 128, 1280, 512, 2
EPS = 1e-6


def _desc():
    return mg.DecodeDesc(B=B, H=H, hd=HD, d_mem=D, window=W, rope_base=10000.0, rms_eps=EPS, inject=1,
                         dtype=mg.MAGLEV_BF16, spin_limit=0)


class GpuDecoder:
    """Device state of an L-layer decode: rings, memory, and step buffers."""

    def __init__(self, seed, m0):
        self.desc = _desc()
        x0 = synth.decode_inputs(seed, B, H, HD, D, W, [0] * B)
        self.wk, self.wv = dev(x0["w_mk"]), dev(x0["w_mv"])
        self.gates = [synth.uniform(seed, synth.TID["gates"] + 64 * l, (4, H), -2.0, 2.0) for l in range(L)]
        self.gates_d = [dev(g) for g in self.gates]
        self.rings = []
        for l in range(L):
            xl = synth.decode_inputs(seed, B, H, HD, D, W, [0] * B, layer=l)
            self.rings.append((dev(xl["k_ring"]), dev(xl["v_ring"])))
        self.m = m0.clone()
        self.krec = torch.empty(B, H, HD, dtype=torch.bfloat16, device="cuda")
        self.vrec = torch.empty_like(self.krec)
        self.out = [torch.empty_like(self.krec) for _ in range(L)]
        self.rstd = torch.empty(B, dtype=torch.float32, device="cuda")
        self.ws = torch.zeros(max(16, mg.maglev_decode_workspace_bytes(self.desc)), dtype=torch.uint8, device="cuda")

    def step(self, pos_t, qkv):
        mg.maglev_decode_mem_project(self.desc, pos_t, self.m, self.wk, self.wv, self.krec, self.vrec)
        for l in range(L):
            q, k, v = qkv[l]
            kr, vr = self.rings[l]
            mg.maglev_decode_step(self.desc, pos_t, q, k, v, self.krec, self.vrec, self.gates_d[l], kr, vr,
                                  self.out[l], self.ws)
        mg.maglev_memory_state(B, 1, D, EPS, mg.MAGLEV_BF16, self.out[L - 1], self.m, None, self.rstd)


def oracle_step(pos, m, qkv, gates, rings, w_mk, w_mv):
    """One token step of the same decoder in fp64: returns (outs, rings', m_p)."""
    krec, vrec = oracle.decode_mem_project(pos, m, w_mk, w_mv, H, eps=EPS)
    outs, new = [], []
    for l in range(L):
        q, k, v = qkv[l]
        o, kr, vr = oracle.decode_step(pos, q, k, v, krec, vrec, gates[l].astype(np.float64), *rings[l])
        outs.append(o)
        new.append((kr, vr))
    m_p = oracle.memory_state(outs[-1].reshape(B, 1, D), EPS)[:, 0]
    return outs, new, m_p


def _host_qkv(seed, l, s):
    sub = (l << 20) | s
    return tuple(synth.normal(seed, synth.TID[n], (B, H, HD), sub=sub) for n in ("q", "k", "v"))


def _bf16(x):
    return synth.bf16_bits_to_f64(synth.round_to_bf16_bits(np.asarray(x, dtype=np.float32)))


def test_decode_trajectory_16_steps():
    """16 steps with the ring carried and m fed back, from positions 505 (first
    lap: slots 505..511 then 0..8, crossing p = 511 -> 512) and 1017 (second
    lap, same slots). Every step's output of every layer is compared with the
    oracle run over the same 16 steps on its own memory; at the end the written
    slots of both rings are compared within tolerance and every other slot
    bit-exactly with the pre-filled ring. What the GPU keeps from one step to
    the next is stored in bf16 (the memory m_p and the new ring entries), and
    the oracle's trajectory stores the same values rounded the same way, so that
    the storage rounding is not compounded over the 16 steps on one side only."""
    seed = 41
    x0 = synth.decode_inputs(seed, B, H, HD, D, W, [0] * B)
    m0 = synth.normal(seed, synth.TID["m_prev"], (B, D), sub=1 << 30)
    G = GpuDecoder(seed, dev(m0))
    p0 = np.array([505 + 512 * (b % 2) for b in range(B)], dtype=np.int64)
    rings0 = [(host(kr), host(vr)) for kr, vr in G.rings]
    rings = [(a.copy(), b.copy()) for a, b in rings0]
    m = m0.f64
    wk, wv = x0["w_mk"].f64, x0["w_mv"].f64
    for s in range(16):
        pos = p0 + s
        qkv_h = [_host_qkv(seed, l, s) for l in range(L)]
        G.step(torch.from_numpy(pos).cuda(), [tuple(dev(t) for t in qkv_h[l]) for l in range(L)])
        outs, rings, m = oracle_step(pos, m, [tuple(t.f64 for t in qkv_h[l]) for l in range(L)], G.gates,
                                     rings, wk, wv)
        m = _bf16(m)
        for kr, vr in rings:  # the written slots, as the ring stores them
            for b in range(B):
                slot = int(pos[b] % W)
                kr[b, :, slot] = _bf16(kr[b, :, slot])
                vr[b, :, slot] = _bf16(vr[b, :, slot])
        for l in range(L):
            assert_close(host(G.out[l]), outs[l], "bf16", f"step {s} layer {l} out")
        assert_close(host(G.m), m, "bf16", f"step {s} memory")
    written = [sorted({int((p + s) % W) for s in range(16)}) for p in p0]
    for l in range(L):
        for r, name in ((0, "k"), (1, "v")):
            got = host(G.rings[l][r])
            for b in range(B):
                keep = np.setdiff1d(np.arange(W), written[b])
                np.testing.assert_array_equal(got[b][:, keep], rings0[l][r][b][:, keep])
                err = normwise(got[b][:, written[b]], rings[l][r][b][:, written[b]])
                assert err <= TOL["bf16"], (l, name, b, err)


def test_decode_teacher_forced_checkpoints():
    """4096 steps from the pre-filled ring (positions 0..511, m_511 = 0), as in
    the benchmark's decode run; at steps 0, 511, 512, 2047 and 4095 the GPU's
    own rings and memory are handed to the oracle for one step, whose output and
    written slot must match the GPU's step, with every other slot unchanged."""
    seed = 43
    x0 = synth.decode_inputs(seed, B, H, HD, D, W, [0] * B)
    G = GpuDecoder(seed, torch.zeros(B, D, dtype=torch.bfloat16, device="cuda"))
    wk, wv = x0["w_mk"].f64, x0["w_mv"].f64
    gen = torch.Generator(device="cuda")
    gen.manual_seed(seed)
    checks = {0, 511, 512, 2047, 4095}
    for s in range(4096):
        p = 512 + s
        pos_t = torch.full((B,), p, dtype=torch.int64, device="cuda")
        qkv = [tuple(torch.randn(B, H, HD, generator=gen, device="cuda").to(torch.bfloat16) for _ in range(3))
               for _ in range(L)]
        if s not in checks:
            G.step(pos_t, qkv)
            continue
        before = [(host(kr), host(vr)) for kr, vr in G.rings]
        m_before = host(G.m)
        G.step(pos_t, qkv)
        pos = np.full(B, p, dtype=np.int64)
        outs, after, _ = oracle_step(pos, m_before, [tuple(host(t) for t in qkv[l]) for l in range(L)],
                                     G.gates, before, wk, wv)
        slot = p % W
        keep = [j for j in range(W) if j != slot]
        for l in range(L):
            assert_close(host(G.out[l]), outs[l], "bf16", f"step {s} layer {l} out")
            for r in range(2):
                got = host(G.rings[l][r])
                np.testing.assert_array_equal(got[:, :, keep], before[l][r][:, :, keep])
                assert_close(got[:, :, slot], after[l][r][:, :, slot], "bf16", f"step {s} layer {l} slot")
        del before, after


@pytest.mark.parametrize("T", [700, 300])
def test_prefill_from_prompt_then_decode(T):
    """Training-form forward over a T-token prompt, maglev_decode_prefill into
    fresh rings, then one decode step at position T: its output must equal row
    T of the oracle's (T+1)-row forward (recurrence = teacher forcing). T = 700
    fills the whole ring (positions 188..699, slot 188 then takes position 700);
    T = 300 fills slots 0..299 and must leave the others untouched."""
    from sliding_window_recurrent_b200.layer import DecodeLayerState, InjectedSWALayer

    Bq, Hq = 2, 10
    wl = dict(synth.WORKLOADS["layer_bf16"])
    wl.update(B=Bq, T=T + 1, H=Hq)
    x = synth.layer_inputs(wl, 51)
    rows = lambda t, a, b: synth.Tensor(np.ascontiguousarray(t.bits[:, a:b]), t.dtype)
    Lyr = InjectedSWALayer(Bq, T, Hq, HD, D, W, dtype="bf16")
    Lyr.forward(dev(rows(x["q"], 0, T)), dev(rows(x["k"], 0, T)), dev(rows(x["v"], 0, T)), dev(x["gates"]),
                dev(rows(x["m_shift"], 0, T)), dev(x["w_mk"]), dev(x["w_mv"]))
    fill = 9.0
    kr = torch.full((Bq, Hq, W, HD), fill, dtype=torch.bfloat16, device="cuda")
    vr = torch.full_like(kr, fill)
    mg.maglev_decode_prefill(Lyr.desc, Lyr.saved, kr, vr)
    torch.cuda.synchronize()

    Rk, Rv = oracle.mem_project(x["m_shift"].f64, x["w_mk"].f64, x["w_mv"].f64)
    f = oracle.inject_swa_forward(x["q"].f64, x["k"].f64, x["v"].f64, Rk, Rv, x["gates"].astype(np.float64), W)
    live = list(range(max(0, T - W), T))
    slots = [j % W for j in live]
    got_k, got_v = host(kr), host(vr)
    assert_close(got_k[:, :, slots], f["k_bar"][:, live].transpose(0, 2, 1, 3), "bf16", "prefilled k")
    assert_close(got_v[:, :, slots], f["v_bar"][:, live].transpose(0, 2, 1, 3), "bf16", "prefilled v")
    dead = sorted(set(range(W)) - set(slots))
    assert np.all(got_k[:, :, dead] == fill) and np.all(got_v[:, :, dead] == fill)

    S = DecodeLayerState(Bq, Hq, HD, D, W, dtype="bf16")
    pos_t = torch.full((Bq,), T, dtype=torch.int64, device="cuda")
    S.mem_project(pos_t, dev(rows(x["m_shift"], T, T + 1)).view(Bq, D), dev(x["w_mk"]), dev(x["w_mv"]))
    o = S.step(pos_t, *(dev(rows(x[n], T, T + 1)).view(Bq, Hq, HD) for n in ("q", "k", "v")), dev(x["gates"]),
               kr, vr)
    torch.cuda.synchronize()
    assert_close(host(o), f["out"][:, T], "bf16", f"decode at {T} after prefill")


def test_decode_checkpoint_restore_bit_identical():
    """The whole decode state is the rings, the position and m_{p-1}: run 3
    steps, copy that state out, run 6 more (crossing p = 511 -> 512), restore
    the copy and run the same 6 steps again. Every output and the final state
    must be bit-identical between the two runs."""
    seed = 47
    gen = torch.Generator(device="cuda")
    gen.manual_seed(seed)
    m0 = synth.normal(seed, synth.TID["m_prev"], (B, D), sub=1 << 29)
    G = GpuDecoder(seed, dev(m0))

    def inputs():
        return [tuple(torch.randn(B, H, HD, generator=gen, device="cuda").to(torch.bfloat16) for _ in range(3))
                for _ in range(L)]

    p0 = 507
    for s in range(3):
        G.step(torch.full((B,), p0 + s, dtype=torch.int64, device="cuda"), inputs())
    saved = ([(kr.clone(), vr.clone()) for kr, vr in G.rings], G.m.clone(), p0 + 3)
    steps = [inputs() for _ in range(6)]

    def run():
        outs = []
        for s, qkv in enumerate(steps):
            G.step(torch.full((B,), saved[2] + s, dtype=torch.int64, device="cuda"), qkv)
            outs.append([o.clone() for o in G.out] + [G.m.clone()])
        return outs, [(kr.clone(), vr.clone()) for kr, vr in G.rings]

    first, rings1 = run()
    for (kr, vr), (k0, v0) in zip(G.rings, saved[0]):
        kr.copy_(k0)
        vr.copy_(v0)
    G.m.copy_(saved[1])
    second, rings2 = run()
    torch.cuda.synchronize()
    for s, (a, b) in enumerate(zip(first, second)):
        for i, (x, y) in enumerate(zip(a, b)):
            assert torch.equal(x, y), (s, i)
    for (k1, v1), (k2, v2) in zip(rings1, rings2):
        assert torch.equal(k1, k2) and torch.equal(v1, v2)
