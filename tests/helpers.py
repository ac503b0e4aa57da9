"""Shared test plumbing: host <-> device transfer of synth tensors and error metrics."""
import numpy as np

import synth

TOL = {"f32": 1e-4, "bf16": 2e-2}


def dev(t, device="cuda"):
    """synth.Tensor (or float32 ndarray) -> torch tensor on the device, same bits."""
    import torch
    if isinstance(t, synth.Tensor):
        if t.dtype == "bf16":
            return torch.from_numpy(t.bits.view(np.int16).copy()).view(torch.bfloat16).to(device)
        return torch.from_numpy(t.bits.copy()).to(device)
    return torch.from_numpy(np.ascontiguousarray(t)).to(device)


def host(x):
    """torch tensor -> float64 numpy (exact)."""
    import torch
    return x.detach().to(torch.float64).cpu().numpy()


def normwise(gpu, ref):
    """max |gpu - ref| / max |ref| over the tensor."""
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert gpu.shape == ref.shape, (gpu.shape, ref.shape)
    den = np.max(np.abs(ref))
    if den == 0:
        return float(np.max(np.abs(gpu)))
    return float(np.max(np.abs(gpu - ref)) / den)


def rowwise(gpu, ref, row_len=None):
    """Normwise error of each row of the trailing axis, worst row reported:
    max over rows r of max |gpu_r - ref_r| / max |ref_r|. Small tensors whose
    entries differ in scale (gate gradients [4, H], LSE [B, H, T]) are judged
    row by row, so that a small row cannot hide behind a large one."""
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert gpu.shape == ref.shape, (gpu.shape, ref.shape)
    n = row_len or ref.shape[-1]
    g2, r2 = gpu.reshape(-1, n), ref.reshape(-1, n)
    den = np.max(np.abs(r2), axis=1)
    num = np.max(np.abs(g2 - r2), axis=1)
    err = np.where(den > 0, num / np.where(den > 0, den, 1.0), num)
    return float(err.max())


def elementwise(gpu, ref):
    """max_i |gpu_i - ref_i| / max(|ref_i|, rms(ref)): the element-wise relative
    error, with the tensor's RMS as the floor below which an entry's error is
    measured against the RMS instead of its own (near-zero) value."""
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert gpu.shape == ref.shape, (gpu.shape, ref.shape)
    rms = float(np.sqrt(np.mean(ref * ref)))
    if rms == 0:
        return float(np.max(np.abs(gpu)))
    return float(np.max(np.abs(gpu - ref) / np.maximum(np.abs(ref), rms)))


def assert_close(gpu, ref, dtype, name="", metric="normwise"):
    """metric: "normwise" (whole tensor), "rows" (each row of the last axis) or
    "elementwise" (per entry, RMS floor)."""
    fn = {"normwise": normwise, "rows": rowwise, "elementwise": elementwise}[metric]
    err = fn(gpu, ref)
    assert np.all(np.isfinite(np.asarray(gpu))), f"{name}: non-finite values"
    assert err <= TOL[dtype], f"{name}: {metric} error {err:.3e} > {TOL[dtype]:.0e}"
    return err
