"""A prefiller Q and a decoder P that share one memory, as C-ABI calls.

"Maglev: Sliding Recurrent Memory", paper.rainbus.top, 方法步骤详情: the
prefiller reads the segment without memory and produces m' (its final state
after RMSNorm); the decoder reads the shifted memory m'_{t-1} through one
projection shared by all its layers, and the consistency loss ties its own
final state m to m'. gptget.net, Abstract: Q interleaves full and
sliding-window layers (SLSL), P uses sliding-window layers throughout.

One training step:
  forward   Q layers (no injection) -> memory_state(O_Q last) = m', m_shift
            mem_project(m_shift) = R_k, R_v (once, shared)
            P layers (injected, reading R_k, R_v) -> memory_state(O_P last) = m
            consistency_loss(m, m') -> loss, dm, dm'
  backward  memory_state_bwd(dm) + dout -> P's last layer; P layers in reverse,
            summing dR_k, dR_v in fp32 (rounded once, by layer 0);
            mem_project_bwd -> dm_shift, dW_mk, dW_mv;
            memory_state_bwd(dm' + shifted dm_shift) + dout -> Q's last layer;
            Q layers in reverse.
Every layer's own upstream gradient `dout` comes from the caller. This module
owns buffers and issues library calls only; all arithmetic runs in libmaglev.

Variants (paper.rainbus.top, 未来方向, lists a per-layer memory projection;
方法步骤详情 mixes the value "likewise", which also reads as the value reusing the
key's gates): per_layer_wrec gives every P layer its own W^rec (weights
[L, D, D]; each layer projects the shifted memory itself, and the backward sums
the layers' dR^l W^l in one fp32 accumulation); shared_kv_gates makes each P
layer's gate logits [2, H] (loc, rec) for both K and V.
"""
from __future__ import annotations

import torch

from . import (MAGLEV_DR_ADD, MAGLEV_DR_FIRST, MAGLEV_DR_LAST, MAGLEV_DR_WRITE, SwaDesc, maglev_consistency_loss,
               maglev_consistency_workspace_bytes, maglev_inject_swa_bwd, maglev_inject_swa_fwd, maglev_mem_project,
               maglev_mem_project_bwd, maglev_mem_project_bwd_layers, maglev_memory_state, maglev_memory_state_bwd,
               maglev_swa_bwd_workspace_bytes, maglev_swa_saved_bytes)
from .layer import CODE, TORCH_DTYPE, _bytes


class _LayerBufs:
    def __init__(self, desc, B, T, H, hd, td, device, inject):
        self.desc = desc
        self.out = torch.empty(B, T, H, hd, dtype=td, device=device)
        self.lse = torch.empty(B, H, T, dtype=torch.float32, device=device)
        self.saved = _bytes(maglev_swa_saved_bytes(desc), device)
        self.dq = torch.empty(B, T, H, hd, dtype=td, device=device)
        self.dk = torch.empty_like(self.dq)
        self.dv = torch.empty_like(self.dq)
        ng = 2 if desc.shared_kv_gates else 4
        self.dgate = torch.empty(ng, H, dtype=torch.float32, device=device) if inject else None


class PrefillerDecoderStack:
    """Buffers and call sequence of one Q + P training step.

    q_windows / p_windows: the window of each layer (W >= T is full causal).
    All layers have H heads of hd channels and d = H * hd memory channels.
    """

    def __init__(self, B, T, H, hd, q_windows, p_windows, lam=0.1, dtype="bf16", device="cuda",
                 rope_base=10000.0, eps=1e-6, spin_limit=0, per_layer_wrec=False, shared_kv_gates=False):
        self.B, self.T, self.H, self.hd = B, T, H, hd
        self.d = H * hd
        self.lam, self.eps, self.dtype, self.device = lam, eps, dtype, device
        self.per_layer_wrec = per_layer_wrec
        td = TORCH_DTYPE[dtype]
        code = CODE[dtype]

        def desc(w, inject):
            return SwaDesc(B=B, T=T, H=H, hd=hd, d_mem=self.d, window=w, rope_base=rope_base, rms_eps=eps,
                           inject=int(inject), pos0=0, dtype=code, spin_limit=spin_limit,
                           shared_kv_gates=int(shared_kv_gates and inject))

        self.q = [_LayerBufs(desc(w, False), B, T, H, hd, td, device, False) for w in q_windows]
        self.p = [_LayerBufs(desc(w, True), B, T, H, hd, td, device, True) for w in p_windows]
        ws = max(maglev_swa_bwd_workspace_bytes(L.desc) for L in self.q + self.p)
        self.workspace = _bytes(ws, device)  # layers run one after another on one stream
        d = self.d
        e = lambda *s, t=td: torch.empty(*s, dtype=t, device=device)
        self.m_prime, self.m_shift, self.m = e(B, T, d), e(B, T, d), e(B, T, d)
        self.rstd_q, self.rstd_p = e(B * T, t=torch.float32), e(B * T, t=torch.float32)
        nL = len(self.p)
        if per_layer_wrec:  # each P layer's own R^l and dL/dR^l, layer-strided
            self.R_k, self.R_v = e(nL, B, T, d), e(nL, B, T, d)
            self.dR_k, self.dR_v = e(nL, B, T, d), e(nL, B, T, d)
            self.dR_acc_k = self.dR_acc_v = None
            self.dw_mk, self.dw_mv = e(nL, d, d), e(nL, d, d)
        else:
            self.R_k, self.R_v = e(B, T, d), e(B, T, d)
            self.dR_k, self.dR_v = e(B, T, d), e(B, T, d)
            # fp32 running sums of dL/dR over P's layers (rounded once into dR_k, dR_v)
            n_acc = 1 if nL > 1 else 0
            self.dR_acc_k = e(n_acc * B, T, d, t=torch.float32) if n_acc else None
            self.dR_acc_v = e(n_acc * B, T, d, t=torch.float32) if n_acc else None
            self.dw_mk, self.dw_mv = e(d, d), e(d, d)
        self.dm, self.dm_prime, self.dm_shift = e(B, T, d), e(B, T, d), e(B, T, d)
        self.dout_p_last, self.dout_q_last = e(B, T, H, hd), e(B, T, H, hd)
        self.loss = torch.zeros((), dtype=torch.float32, device=device)
        self.loss_ws = _bytes(maglev_consistency_workspace_bytes(B * T, d), device)

    def _R(self, i):
        return (self.R_k[i], self.R_v[i]) if self.per_layer_wrec else (self.R_k, self.R_v)

    def forward(self, q_inputs, p_inputs, w_mk, w_mv, stream=None):
        """q_inputs: per Q layer (q, k, v); p_inputs: per P layer (q, k, v, gate_logits).
        w_mk, w_mv: [D, D], or [L_P, D, D] with per_layer_wrec."""
        B, T, d, code = self.B, self.T, self.d, CODE[self.dtype]
        for L, (q, k, v) in zip(self.q, q_inputs):
            maglev_inject_swa_fwd(L.desc, q, k, v, None, None, None, None, None, None, L.out, L.lse, L.saved,
                                  stream)
        maglev_memory_state(B, T, d, self.eps, code, self.q[-1].out, self.m_prime, self.m_shift, self.rstd_q,
                            stream)
        if self.per_layer_wrec:
            for i in range(len(self.p)):
                maglev_mem_project(self.p[i].desc, self.m_shift, w_mk[i], w_mv[i], self.R_k[i], self.R_v[i], stream)
        else:
            maglev_mem_project(self.p[0].desc, self.m_shift, w_mk, w_mv, self.R_k, self.R_v, stream)
        for i, (L, (q, k, v, g)) in enumerate(zip(self.p, p_inputs)):
            Rk, Rv = self._R(i)
            maglev_inject_swa_fwd(L.desc, q, k, v, None, None, None, Rk, Rv, g, L.out, L.lse, L.saved, stream)
        maglev_memory_state(B, T, d, self.eps, code, self.p[-1].out, self.m, None, self.rstd_p, stream)
        maglev_consistency_loss(self.m, self.m_prime, B * T, d, code, self.lam, 0.0, self.loss, self.dm,
                                self.dm_prime, False, self.loss_ws, stream)
        return self.loss

    def backward(self, q_inputs, p_inputs, q_douts, p_douts, w_mk, w_mv, stream=None):
        """q_douts / p_douts: each layer's upstream gradient of its output."""
        B, T, d, code = self.B, self.T, self.d, CODE[self.dtype]
        maglev_memory_state_bwd(B, T, d, code, self.p[-1].out, self.rstd_p, self.dm, None, p_douts[-1],
                                self.dout_p_last, stream)
        n = len(self.p)
        for i in reversed(range(n)):
            L = self.p[i]
            _, k, v, g = p_inputs[i]
            dout = self.dout_p_last if i == n - 1 else p_douts[i]
            Rk, Rv = self._R(i)
            if self.per_layer_wrec:
                dRk, dRv, mode = self.dR_k[i], self.dR_v[i], MAGLEV_DR_WRITE
            else:
                dRk, dRv, mode = self.dR_k, self.dR_v, self._dr_mode(i, n)
            maglev_inject_swa_bwd(L.desc, k, v, Rk, Rv, g, L.out, L.lse, L.saved, dout, L.dq, L.dk, L.dv, dRk, dRv,
                                  self.dR_acc_k, self.dR_acc_v, mode, L.dgate, None, None, None, None, None, None,
                                  self.workspace, stream)
        if self.per_layer_wrec:
            maglev_mem_project_bwd_layers(self.p[0].desc, n, self.m_shift, w_mk, w_mv, self.dR_k, self.dR_v,
                                          self.dm_shift, self.dw_mk, self.dw_mv, stream)
        else:
            maglev_mem_project_bwd(self.p[0].desc, self.m_shift, w_mk, w_mv, self.dR_k, self.dR_v, self.dm_shift,
                                   self.dw_mk, self.dw_mv, stream)
        maglev_memory_state_bwd(B, T, d, code, self.q[-1].out, self.rstd_q, self.dm_prime, self.dm_shift,
                                q_douts[-1], self.dout_q_last, stream)
        n = len(self.q)
        for i in reversed(range(n)):
            L = self.q[i]
            _, k, v = q_inputs[i]
            dout = self.dout_q_last if i == n - 1 else q_douts[i]
            maglev_inject_swa_bwd(L.desc, k, v, None, None, None, L.out, L.lse, L.saved, dout, L.dq, L.dk, L.dv,
                                  None, None, None, None, MAGLEV_DR_WRITE, None, None, None, None, None, None,
                                  None, self.workspace, stream)

    @staticmethod
    def _dr_mode(i, n):
        """P's backward runs from layer n-1 down to 0: the first call starts the
        fp32 sum, the last one adds its share and rounds the total into dR."""
        if n == 1:
            return MAGLEV_DR_WRITE
        if i == n - 1:
            return MAGLEV_DR_FIRST
        return MAGLEV_DR_LAST if i == 0 else MAGLEV_DR_ADD

    def step(self, q_inputs, p_inputs, q_douts, p_douts, w_mk, w_mv, stream=None):
        self.forward(q_inputs, p_inputs, w_mk, w_mv, stream)
        self.backward(q_inputs, p_inputs, q_douts, p_douts, w_mk, w_mv, stream)
        return self.loss
