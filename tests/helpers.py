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


def assert_close(gpu, ref, dtype, name=""):
    err = normwise(gpu, ref)
    assert np.all(np.isfinite(np.asarray(gpu))), f"{name}: non-finite values"
    assert err <= TOL[dtype], f"{name}: normwise error {err:.3e} > {TOL[dtype]:.0e}"
    return err
