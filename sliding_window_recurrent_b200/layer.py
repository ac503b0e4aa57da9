"""Torch-allocated buffers around the C ABI (device memory and streams only).

InjectedSWALayer owns the outputs, saved activations, gradients and scratch
of one layer and calls the library entry points; it performs no arithmetic.
"""
from __future__ import annotations

import torch

from . import (DecodeDesc, MAGLEV_BF16, MAGLEV_BWD_PREPARED, MAGLEV_DR_WRITE, MAGLEV_F32, SwaDesc,
               maglev_consistency_loss, maglev_consistency_loss_prepare_bwd, maglev_consistency_workspace_bytes, maglev_decode_mem_project, maglev_decode_step,
               maglev_decode_workspace_bytes,
               maglev_inject_swa_bwd, maglev_inject_swa_fwd, maglev_swa_bwd_workspace_bytes,
               maglev_swa_saved_bytes)

TORCH_DTYPE = {"bf16": torch.bfloat16, "f32": torch.float32}
CODE = {"bf16": MAGLEV_BF16, "f32": MAGLEV_F32}


def _bytes(n: int, device) -> torch.Tensor:
    return torch.empty(max(int(n), 16), dtype=torch.uint8, device=device)


class InjectedSWALayer:
    def __init__(self, B, T, H, hd, d_mem, window, dtype="bf16", inject=True, pos0=0,
                 rope_base=10000.0, eps=1e-6, device="cuda", spin_limit=0, shared_kv_gates=False):
        self.shape = (B, T, H, hd)
        self.d_mem, self.dtype, self.device = d_mem, dtype, device
        self.inject = bool(inject)
        self.desc = SwaDesc(B=B, T=T, H=H, hd=hd, d_mem=d_mem, window=window, rope_base=rope_base,
                            rms_eps=eps, inject=int(inject), pos0=pos0, dtype=CODE[dtype],
                            spin_limit=spin_limit, shared_kv_gates=int(shared_kv_gates))
        td = TORCH_DTYPE[dtype]
        D = H * hd
        self.out = torch.empty(B, T, H, hd, dtype=td, device=device)
        self.lse = torch.empty(B, H, T, dtype=torch.float32, device=device)
        self.saved = _bytes(maglev_swa_saved_bytes(self.desc), device)
        self.workspace = _bytes(maglev_swa_bwd_workspace_bytes(self.desc), device)
        self.R_k = torch.empty(B, T, D, dtype=td, device=device) if inject else None
        self.R_v = torch.empty(B, T, D, dtype=td, device=device) if inject else None
        self.dq = torch.empty(B, T, H, hd, dtype=td, device=device)
        self.dk = torch.empty_like(self.dq)
        self.dv = torch.empty_like(self.dq)
        self.dR_k = torch.empty(B, T, D, dtype=td, device=device) if inject else None
        self.dR_v = torch.empty(B, T, D, dtype=td, device=device) if inject else None
        self.dgate = torch.empty(2 if shared_kv_gates else 4, H, dtype=torch.float32,
                                 device=device) if inject else None
        self.dm_shift = torch.empty(B, T, d_mem, dtype=td, device=device) if inject else None
        self.dw_mk = torch.empty(D, d_mem, dtype=td, device=device) if inject else None
        self.dw_mv = torch.empty(D, d_mem, dtype=td, device=device) if inject else None
        self.loss = torch.zeros((), dtype=torch.float32, device=device)
        self.loss_ws = _bytes(maglev_consistency_workspace_bytes(B * T, D), device)

    def forward(self, q, k, v, gates=None, m_shift=None, w_mk=None, w_mv=None, stream=None):
        """m_shift given: project it here; m_shift None: R_k/R_v already hold the projection."""
        maglev_inject_swa_fwd(self.desc, q, k, v, m_shift if self.inject else None, w_mk, w_mv,
                              self.R_k, self.R_v, gates, self.out, self.lse, self.saved, stream)
        return self.out

    def consistency(self, m, target, lam, dm=None, accumulate_dm=False, inv_count=0.0, stream=None):
        rows = m.numel() // m.shape[-1]
        maglev_consistency_loss(m, target, rows, m.shape[-1], CODE[self.dtype], lam, inv_count,
                                self.loss, dm, None, accumulate_dm, self.loss_ws, stream)
        return self.loss

    def consistency_prepare_bwd(self, target, lam, dout, inv_count=0.0, stream=None):
        """The consistency loss of this layer's own output against target,
        added into dout, together with the backward's first pass (the next
        backward call is given prepared=True)."""
        maglev_consistency_loss_prepare_bwd(self.desc, self.out, target, lam, inv_count, self.loss, dout,
                                            self.workspace, self.loss_ws, stream)
        return self.loss

    def backward(self, k, v, dout, gates=None, m_shift=None, w_mk=None, w_mv=None,
                 dR_mode=MAGLEV_DR_WRITE, dR_acc=(None, None), stream=None, prepared=False):
        """dR_mode / dR_acc: how dL/dR is stored (maglev_dr_mode) and the fp32
        running sums it reads or writes when several layers share W^rec;
        prepared: consistency_prepare_bwd ran on this out and dout."""
        maglev_inject_swa_bwd(self.desc, k, v, self.R_k, self.R_v, gates, self.out, self.lse,
                              self.saved, dout, self.dq, self.dk, self.dv, self.dR_k, self.dR_v,
                              dR_acc[0], dR_acc[1], dR_mode | (MAGLEV_BWD_PREPARED if prepared else 0), self.dgate,
                              m_shift if self.inject else None, w_mk, w_mv,
                              self.dm_shift, self.dw_mk, self.dw_mv, self.workspace, stream)


class DecodeLayerState:
    """Buffers of one decode step of one layer (rings are caller tensors)."""

    def __init__(self, B, H, hd, d_mem, window, dtype="bf16", inject=True, rope_base=10000.0,
                 eps=1e-6, device="cuda", shared_kv_gates=False):
        self.desc = DecodeDesc(B=B, H=H, hd=hd, d_mem=d_mem, window=window, rope_base=rope_base,
                               rms_eps=eps, inject=int(inject), dtype=CODE[dtype], spin_limit=0,
                               shared_kv_gates=int(shared_kv_gates))
        td = TORCH_DTYPE[dtype]
        self.krec = torch.empty(B, H, hd, dtype=td, device=device)
        self.vrec = torch.empty(B, H, hd, dtype=td, device=device)
        self.out = torch.empty(B, H, hd, dtype=td, device=device)
        # zero-filled once; every completed step leaves it zero-filled
        self.workspace = torch.zeros(max(16, maglev_decode_workspace_bytes(self.desc)), dtype=torch.uint8,
                                     device=device)

    def mem_project(self, pos, m_prev, w_mk, w_mv, stream=None):
        maglev_decode_mem_project(self.desc, pos, m_prev, w_mk, w_mv, self.krec, self.vrec, stream)

    def step(self, pos, q, k, v, gates, k_ring, v_ring, stream=None):
        maglev_decode_step(self.desc, pos, q, k, v, self.krec, self.vrec, gates, k_ring, v_ring,
                           self.out, self.workspace, stream)
        return self.out
