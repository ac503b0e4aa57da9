"""Shared test plumbing: host <-> device transfer of synth tensors and error metrics."""
import numpy as np

import synth

TOL = {"f32": 1e-4, "bf16": 2e-2}
# Gate gradients, per entry against the RMS size of the B*T*hd products each
# sums (see `scaled`). Derived from the arithmetic: rounding the operands the
# bf16 kernels round (q_rot, k_bar, v_bar, P, dS, dk_bar, dv_bar) in an fp64
# emulation of the backward moves these sums by up to 2.0e-2 of that scale at
# T = 2048 (each dk_bar sums ~512 dS q products with heavy cancellation, and the
# rounding of dS does not cancel with it); 5e-2 leaves room for the spread
# between rounding realisations. fp32 storage keeps the fp32 bound.
GATE_TOL = {"f32": 1e-4, "bf16": 5e-2}


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


def logwise(gpu, ref):
    """Error of a log-domain quantity (LSE) row by row, each row's normwise error
    with a floor of 1 below the row's largest magnitude: an absolute error d in
    a log-sum-exp is a relative error e^d - 1 ~ d of the partition function, so
    near zero the error is judged in absolute terms."""
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert gpu.shape == ref.shape, (gpu.shape, ref.shape)
    n = ref.shape[-1]
    g2, r2 = gpu.reshape(-1, n), ref.reshape(-1, n)
    den = np.maximum(np.max(np.abs(r2), axis=1), 1.0)
    return float(np.max(np.max(np.abs(g2 - r2), axis=1) / den))


def scaled(gpu, ref, scale):
    """max_i |gpu_i - ref_i| / scale_i: the error of each entry of a reduced
    quantity against the RMS size of the summands it adds up (the scale of its
    rounding error; see the oracle's dgate_scale)."""
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    scale = np.asarray(scale, dtype=np.float64)
    assert gpu.shape == ref.shape == scale.shape, (gpu.shape, ref.shape, scale.shape)
    return float(np.max(np.abs(gpu - ref) / np.where(scale > 0, scale, 1.0)))


def assert_close(gpu, ref, dtype, name="", metric="normwise", scale=None):
    """metric: "normwise" (whole tensor), "rows" (each row of the last axis),
    "log" (LSE rows, floor 1), "elementwise" (per entry, RMS floor) or
    "scaled" (per entry against `scale`)."""
    if metric == "scaled":
        err = scaled(gpu, ref, scale)
    else:
        fn = {"normwise": normwise, "rows": rowwise, "log": logwise, "elementwise": elementwise}[metric]
        err = fn(gpu, ref)
    tol = GATE_TOL[dtype] if metric == "scaled" else TOL[dtype]
    assert np.all(np.isfinite(np.asarray(gpu))), f"{name}: non-finite values"
    assert err <= tol, f"{name}: {metric} error {err:.3e} > {tol:.0e}"
    return err
