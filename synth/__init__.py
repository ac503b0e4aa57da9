"""Seeded synthetic inputs for Maglev's injected sliding-window attention.

This module is the only code shared by the CUDA path (tests, bench) and the
CPU oracle. It holds no arithmetic of the method: it draws random numbers,
rounds them to the storage type, and names the workload shapes.

Every tensor is drawn from numpy's Philox counter-based generator keyed by
(seed, tensor id, sub-stream), so any tensor -- or any (layer, batch-row)
slice of one -- can be regenerated on its own.

Workload shapes follow the d20 model of the Maglev pages (arXiv 2608.02870,
paper.rainbus.top, section "实验结果": L=20, d=1280, 10 heads x 128, context
2048, window 512). The pages train on FineWeb-Edu; no dataset is used here:
these seeded Gaussian inputs stand in for it.
"""
from __future__ import annotations

import dataclasses
import numpy as np

# Stable tensor ids; a layer index is folded in as tid + 64 * layer.
TID = {
    "q": 1, "k": 2, "v": 3, "mtraj": 4, "w_mk": 5, "w_mv": 6, "gates": 7,
    "dout": 8, "target": 9, "k_ring": 10, "v_ring": 11, "m_prev": 12,
    "h0": 13, "pos": 14, "dq_seed": 15, "w_qkv": 16,
}


def _gen(seed: int, tid: int, sub: int = 0) -> np.random.Generator:
    key = np.array([int(seed) & (2**64 - 1), ((int(tid) << 32) | int(sub)) & (2**64 - 1)],
                   dtype=np.uint64)
    return np.random.Generator(np.random.Philox(key=key))


def round_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float -> bf16 bit pattern (uint16), round-to-nearest-even. Inputs are finite."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


@dataclasses.dataclass
class Tensor:
    """A host tensor in its storage form plus its exact float64 value.

    ``bits`` is uint16 (bf16 bit patterns) for dtype "bf16" and float32 for "f32".
    """
    bits: np.ndarray
    dtype: str

    @property
    def f64(self) -> np.ndarray:
        if self.dtype == "bf16":
            return bf16_bits_to_f64(self.bits)
        return self.bits.astype(np.float64)

    @property
    def shape(self):
        return self.bits.shape

    @staticmethod
    def from_float(x: np.ndarray, dtype: str) -> "Tensor":
        if dtype == "bf16":
            return Tensor(round_to_bf16_bits(x), "bf16")
        if dtype == "f32":
            return Tensor(np.ascontiguousarray(x, dtype=np.float32), "f32")
        raise ValueError(dtype)


def normal(seed: int, tid: int, shape, std: float = 1.0, dtype: str = "bf16", sub: int = 0) -> Tensor:
    x = _gen(seed, tid, sub).standard_normal(size=tuple(shape), dtype=np.float32)
    if std != 1.0:
        x = (x.astype(np.float64) * std).astype(np.float32)
    return Tensor.from_float(x, dtype)


def uniform(seed: int, tid: int, shape, lo: float, hi: float, sub: int = 0) -> np.ndarray:
    """float32 uniform draws in [lo, hi)."""
    g = _gen(seed, tid, sub)
    return (lo + (hi - lo) * g.random(size=tuple(shape), dtype=np.float64)).astype(np.float32)


# ---------------------------------------------------------------------------
# Workloads. Positions are 0-based; the window holds W keys, self included.
# ---------------------------------------------------------------------------
WORKLOADS = {
    # B=1, T=256, d_model=128, 2 heads x 64, W=64, fp32, lambda=1, independent target.
    "tiny_f32": dict(B=1, T=256, H=2, hd=64, d=128, W=64, dtype="f32", lam=1.0,
                     rope_base=10000.0, eps=1e-6, target="independent"),
    # B=4, T=2048, d=1280, 10 heads x 128, W=512, bf16, lambda=0.1 (fwd+bwd adds the loss).
    "layer_bf16": dict(B=4, T=2048, H=10, hd=128, d=1280, W=512, dtype="bf16", lam=0.1,
                       rope_base=10000.0, eps=1e-6, target="trajectory"),
    # 20-layer SSSS decoder P with injection plus a 20-layer SLSL prefiller Q, B=8.
    "stack20_bf16": dict(B=8, T=2048, H=10, hd=128, d=1280, W=512, L=20, dtype="bf16", lam=0.1,
                         rope_base=10000.0, eps=1e-6, target="trajectory"),
    # Recurrent decode: 64 sequences, 20 layers, rolling 512-entry ring per layer.
    "decode_bf16": dict(B=64, L=20, H=10, hd=128, d=1280, W=512, dtype="bf16", steps=4096,
                        rope_base=10000.0, eps=1e-6, first_pos=512),
}


def layer_inputs(wl: dict, seed: int, layer: int = 0, inject: bool = True) -> dict:
    """Seeded inputs of one injected-SWA layer.

    q, k, v [B,T,H,hd] (pre-RoPE) ~ N(0,1): this is the exact marginal law of
    RMSNorm(x) W^T with W ~ N(0, 1/d), so the projection itself is not run.
    mtraj [B,T+1,d]: rows 1..T ~ N(0,1), row 0 = 0 (the pages set m'_0 = 0).
    m_shift = mtraj[:, :T]; target = mtraj[:, 1:] ("trajectory") or a second
    independent N(0,1) tensor ("independent"). W_mk, W_mv [D,d] ~ N(0,1/d).
    gate logits [4,H] ~ U[-2,2] (k_loc, k_rec, v_loc, v_rec). dout ~ N(0,1).
    """
    B, T, H, hd, d, dt = wl["B"], wl["T"], wl["H"], wl["hd"], wl["d"], wl["dtype"]
    D = H * hd
    off = 64 * layer
    out = {
        "q": normal(seed, TID["q"] + off, (B, T, H, hd), dtype=dt),
        "k": normal(seed, TID["k"] + off, (B, T, H, hd), dtype=dt),
        "v": normal(seed, TID["v"] + off, (B, T, H, hd), dtype=dt),
        "gates": uniform(seed, TID["gates"] + off, (4, H), -2.0, 2.0),
        "dout": normal(seed, TID["dout"] + off, (B, T, H, hd), dtype=dt),
    }
    if inject:
        mt = _gen(seed, TID["mtraj"]).standard_normal(size=(B, T + 1, d), dtype=np.float32)
        mt[:, 0, :] = 0.0
        mtraj = Tensor.from_float(mt, dt)
        out["mtraj"] = mtraj
        out["m_shift"] = Tensor(np.ascontiguousarray(mtraj.bits[:, :T]), dt)
        if wl.get("target", "trajectory") == "independent":
            out["target"] = normal(seed, TID["target"], (B, T, D), dtype=dt)
        else:
            out["target"] = Tensor(np.ascontiguousarray(mtraj.bits[:, 1:]), dt)
        out["w_mk"] = normal(seed, TID["w_mk"], (D, d), std=1.0 / np.sqrt(d), dtype=dt)
        out["w_mv"] = normal(seed, TID["w_mv"], (D, d), std=1.0 / np.sqrt(d), dtype=dt)
    return out


def stack_inputs(wl: dict, seed: int, q_windows, p_windows, per_layer_wrec: bool = False,
                 shared_kv_gates: bool = False) -> dict:
    """Seeded inputs of a prefiller Q (no injection) and a decoder P sharing a
    memory: per layer q, k, v, dout ~ N(0,1) [B,T,H,hd]; P's gate logits
    ~ U[-2,2] ([4,H], or [2,H] with shared_kv_gates); W_mk, W_mv [D,D]
    ~ N(0,1/D), and with per_layer_wrec one more pair per P layer (in its layer
    dict). P's layer l draws with layer index l, Q's layer l with index 32 + l."""
    B, T, H, hd, dt = wl["B"], wl["T"], wl["H"], wl["hd"], wl["dtype"]
    D = H * hd

    def one(layer, gates):
        off = 64 * layer
        x = {k: normal(seed, TID[k] + off, (B, T, H, hd), dtype=dt) for k in ("q", "k", "v", "dout")}
        if gates:
            x["gates"] = uniform(seed, TID["gates"] + off, (2 if shared_kv_gates else 4, H), -2.0, 2.0)
            if per_layer_wrec:
                x["w_mk"] = normal(seed, TID["w_mk"] + off, (D, D), std=1.0 / np.sqrt(D), dtype=dt, sub=1)
                x["w_mv"] = normal(seed, TID["w_mv"] + off, (D, D), std=1.0 / np.sqrt(D), dtype=dt, sub=1)
        return x

    q_layers = [dict(one(32 + l, False), window=w) for l, w in enumerate(q_windows)]
    p_layers = [dict(one(l, True), window=w) for l, w in enumerate(p_windows)]
    return {"q_layers": q_layers, "p_layers": p_layers,
            "w_mk": normal(seed, TID["w_mk"], (D, D), std=1.0 / np.sqrt(D), dtype=dt),
            "w_mv": normal(seed, TID["w_mv"], (D, D), std=1.0 / np.sqrt(D), dtype=dt)}


def ring_slice(seed: int, layer: int, b: int, H: int, W: int, hd: int, which: str, dtype: str = "bf16") -> Tensor:
    """Pre-filled ring entries of one (layer, batch row): [H, W, hd] ~ N(0,1)."""
    return normal(seed, TID[which], (H, W, hd), dtype=dtype, sub=(layer << 16) | b)


def decode_inputs(seed: int, B: int, H: int, hd: int, d: int, W: int, pos, dtype: str = "bf16",
                  layer: int = 0, step: int = 0) -> dict:
    """Seeded inputs of one decode step of one layer (ring drawn per batch row)."""
    D = H * hd
    sub = (layer << 20) | step
    pos = np.asarray(pos, dtype=np.int64).reshape(B)
    rk = np.stack([ring_slice(seed, layer, b, H, W, hd, "k_ring", dtype).bits for b in range(B)])
    rv = np.stack([ring_slice(seed, layer, b, H, W, hd, "v_ring", dtype).bits for b in range(B)])
    return {
        "pos": pos,
        "q": normal(seed, TID["q"], (B, H, hd), dtype=dtype, sub=sub),
        "k": normal(seed, TID["k"], (B, H, hd), dtype=dtype, sub=sub),
        "v": normal(seed, TID["v"], (B, H, hd), dtype=dtype, sub=sub),
        "m_prev": normal(seed, TID["m_prev"], (B, d), dtype=dtype, sub=sub),
        "w_mk": normal(seed, TID["w_mk"], (D, d), std=1.0 / np.sqrt(d), dtype=dtype),
        "w_mv": normal(seed, TID["w_mv"], (D, d), std=1.0 / np.sqrt(d), dtype=dtype),
        "gates": uniform(seed, TID["gates"] + 64 * layer, (4, H), -2.0, 2.0),
        "k_ring": Tensor(rk, dtype),
        "v_ring": Tensor(rv, dtype),
    }
