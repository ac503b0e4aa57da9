"""Python binding of libmaglev: Maglev's injected sliding-window attention on B200.

Each function has the name of the C entry point it wraps (see include/maglev.h)
and only marshals arguments: torch tensors become device pointers, None becomes
NULL, and a non-OK status raises MaglevError with the library's message. All
arithmetic runs in libmaglev's CUDA kernels; there is no fallback: the first
call loads libmaglev.so and raises ImportError if it is missing (build it with
`python -m sliding_window_recurrent_b200.build`).
"""
from __future__ import annotations

import ctypes
import os
import re

_HERE = os.path.dirname(os.path.abspath(__file__))
# MAGLEV_DEBUG=1 selects the debug build (in-kernel index checks that record
# MAGLEV_ERR_BOUNDS), libmaglev_debug.so from `build.py --debug`.
LIB_PATH = os.path.join(_HERE, "libmaglev_debug.so" if os.environ.get("MAGLEV_DEBUG") == "1" else "libmaglev.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "maglev.h")

MAGLEV_OK, MAGLEV_ERR_INVALID_ARG, MAGLEV_ERR_UNSUPPORTED, MAGLEV_ERR_CUDA, MAGLEV_ERR_TIMEOUT, MAGLEV_ERR_BOUNDS = range(6)
MAGLEV_F32, MAGLEV_BF16 = 0, 1
MAGLEV_DR_WRITE, MAGLEV_DR_FIRST, MAGLEV_DR_ADD, MAGLEV_DR_LAST = range(4)
MAGLEV_BWD_PREPARED = 16


class MaglevError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"maglev status {status}: {msg}")
        self.status = status


class SwaDesc(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("T", ctypes.c_int), ("H", ctypes.c_int), ("hd", ctypes.c_int),
                ("d_mem", ctypes.c_int), ("window", ctypes.c_int), ("rope_base", ctypes.c_float),
                ("rms_eps", ctypes.c_float), ("inject", ctypes.c_int), ("pos0", ctypes.c_int),
                ("dtype", ctypes.c_int), ("spin_limit", ctypes.c_int64), ("shared_kv_gates", ctypes.c_int)]


class DecodeDesc(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("hd", ctypes.c_int), ("d_mem", ctypes.c_int),
                ("window", ctypes.c_int), ("rope_base", ctypes.c_float), ("rms_eps", ctypes.c_float),
                ("inject", ctypes.c_int), ("dtype", ctypes.c_int), ("spin_limit", ctypes.c_int64),
                ("shared_kv_gates", ctypes.c_int)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          f"`python -m sliding_window_recurrent_b200.build` (nvcc, sm_100a)")
    return ctypes.CDLL(LIB_PATH)


_P = ctypes.c_void_p
_I = ctypes.c_int
_I64 = ctypes.c_int64
_F = ctypes.c_float
_SZ = ctypes.c_size_t
_SIGS = {
    "maglev_version": ([], ctypes.c_char_p),
    "maglev_launch_count": ([], ctypes.c_longlong),
    "maglev_profile_enable": ([_I], None),
    "maglev_profile_report": ([ctypes.c_char_p, _SZ], _SZ),
    "maglev_last_error": ([ctypes.c_char_p, _SZ], _SZ),
    "maglev_device_status": ([_P, ctypes.POINTER(_I)], _I),
    "maglev_swa_saved_bytes": ([ctypes.POINTER(SwaDesc)], _SZ),
    "maglev_swa_bwd_workspace_bytes": ([ctypes.POINTER(SwaDesc)], _SZ),
    "maglev_consistency_workspace_bytes": ([_I64, _I], _SZ),
    "maglev_mem_project": ([ctypes.POINTER(SwaDesc)] + [_P] * 6, _I),
    "maglev_inject_swa_fwd": ([ctypes.POINTER(SwaDesc)] + [_P] * 13, _I),
    "maglev_inject_swa_bwd": ([ctypes.POINTER(SwaDesc)] + [_P] * 16 + [_I] + [_P] * 9, _I),
    "maglev_mem_project_bwd": ([ctypes.POINTER(SwaDesc)] + [_P] * 9, _I),
    "maglev_mem_project_bwd_layers": ([ctypes.POINTER(SwaDesc), _I] + [_P] * 9, _I),
    "maglev_consistency_loss": ([_P, _P, _I64, _I, _I, _F, _F, _P, _P, _P, _I, _P, _P], _I),
    "maglev_consistency_loss_prepare_bwd": ([ctypes.POINTER(SwaDesc), _P, _P, _F, _F, _P, _P, _P, _P, _P], _I),
    "maglev_consistency_loss_noalloc": ([_P, _P, _I64, _I, _I, _F, _F, _P, _P, _P, _I, _P], _I),
    "maglev_memory_state": ([_I, _I, _I, _F, _I] + [_P] * 5, _I),
    "maglev_memory_state_bwd": ([_I, _I, _I, _I] + [_P] * 7, _I),
    "maglev_decode_mem_project": ([ctypes.POINTER(DecodeDesc)] + [_P] * 7, _I),
    "maglev_decode_step": ([ctypes.POINTER(DecodeDesc)] + [_P] * 12, _I),
    "maglev_decode_workspace_bytes": ([ctypes.POINTER(DecodeDesc)], _SZ),
    "maglev_decode_prefill": ([ctypes.POINTER(SwaDesc)] + [_P] * 4, _I),
    "maglev_wait_selftest": ([_P, _I, _I64, _P], _I),
    "maglev_lm_head_workspace_bytes": ([_I64, _I, _I], _SZ),
    "maglev_lm_head_ce": ([_I64, _I, _I, _I, _F, _F] + [_P] * 8 + [_I64, _P], _I),
}


class _Lazy:
    """Loads libmaglev.so and sets the C signatures on first attribute access."""

    def __init__(self):
        self._dll = None

    def __getattr__(self, name):
        if self._dll is None:
            dll = _load()
            for fname, (args, res) in _SIGS.items():
                fn = getattr(dll, fname)
                fn.argtypes = args
                fn.restype = res
            self._dll = dll
        return getattr(self._dll, name)


_lib = _Lazy()


def header_symbols() -> list[str]:
    """Names of the functions declared in include/maglev.h."""
    text = open(HEADER_PATH).read()
    return sorted(set(re.findall(r"\b(maglev_[a-z0-9_]+)\s*\(", text)))


def last_error() -> str:
    buf = ctypes.create_string_buffer(1024)
    _lib.maglev_last_error(buf, 1024)
    return buf.value.decode(errors="replace")


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(s):
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _check(status: int):
    if status != MAGLEV_OK:
        raise MaglevError(status, last_error())


def maglev_version() -> str:
    return _lib.maglev_version().decode()


def maglev_launch_count() -> int:
    return int(_lib.maglev_launch_count())


def maglev_profile_enable(on: bool = True) -> None:
    _lib.maglev_profile_enable(1 if on else 0)


def maglev_profile_report() -> list[tuple[str, int, float]]:
    """[(trace name, kernels, milliseconds)] of the launches traced since the last report."""
    n = _lib.maglev_profile_report(None, 0)
    buf = ctypes.create_string_buffer(n + 1)
    _lib.maglev_profile_report(buf, n + 1)
    rows = []
    for line in buf.value.decode().splitlines():
        name, k, ms = line.split()
        rows.append((name, int(k), float(ms)))
    return rows


def maglev_device_status(stream=None) -> int:
    code = ctypes.c_int(0)
    _check(_lib.maglev_device_status(_stream(stream), ctypes.byref(code)))
    return code.value


def maglev_swa_saved_bytes(desc: SwaDesc) -> int:
    return _lib.maglev_swa_saved_bytes(ctypes.byref(desc))


def maglev_swa_bwd_workspace_bytes(desc: SwaDesc) -> int:
    return _lib.maglev_swa_bwd_workspace_bytes(ctypes.byref(desc))


def maglev_consistency_workspace_bytes(rows: int, d: int) -> int:
    return _lib.maglev_consistency_workspace_bytes(rows, d)


def maglev_mem_project(desc, m_shift, w_mk, w_mv, R_k, R_v, stream=None):
    _check(_lib.maglev_mem_project(ctypes.byref(desc), _ptr(m_shift), _ptr(w_mk), _ptr(w_mv),
                                   _ptr(R_k), _ptr(R_v), _stream(stream)))


def maglev_inject_swa_fwd(desc, q, k, v, m_shift, w_mk, w_mv, R_k, R_v, gate_logits, out, lse, saved,
                          stream=None):
    _check(_lib.maglev_inject_swa_fwd(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(m_shift),
                                      _ptr(w_mk), _ptr(w_mv), _ptr(R_k), _ptr(R_v), _ptr(gate_logits),
                                      _ptr(out), _ptr(lse), _ptr(saved), _stream(stream)))


def maglev_inject_swa_bwd(desc, k, v, R_k, R_v, gate_logits, out, lse, saved, dout, dq, dk, dv,
                          dR_k, dR_v, dR_acc_k, dR_acc_v, dR_mode, dgate_logits, m_shift, w_mk, w_mv,
                          dm_shift, dw_mk, dw_mv, workspace, stream=None):
    _check(_lib.maglev_inject_swa_bwd(
        ctypes.byref(desc), _ptr(k), _ptr(v), _ptr(R_k), _ptr(R_v), _ptr(gate_logits), _ptr(out),
        _ptr(lse), _ptr(saved), _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dR_k), _ptr(dR_v),
        _ptr(dR_acc_k), _ptr(dR_acc_v), int(dR_mode), _ptr(dgate_logits), _ptr(m_shift), _ptr(w_mk),
        _ptr(w_mv), _ptr(dm_shift), _ptr(dw_mk), _ptr(dw_mv), _ptr(workspace), _stream(stream)))


def maglev_mem_project_bwd(desc, m_shift, w_mk, w_mv, dR_k, dR_v, dm_shift, dw_mk, dw_mv, stream=None):
    _check(_lib.maglev_mem_project_bwd(ctypes.byref(desc), _ptr(m_shift), _ptr(w_mk), _ptr(w_mv),
                                       _ptr(dR_k), _ptr(dR_v), _ptr(dm_shift), _ptr(dw_mk),
                                       _ptr(dw_mv), _stream(stream)))


def maglev_mem_project_bwd_layers(desc, n_layers, m_shift, w_mk, w_mv, dR_k, dR_v, dm_shift, dw_mk, dw_mv,
                                  stream=None):
    _check(_lib.maglev_mem_project_bwd_layers(ctypes.byref(desc), int(n_layers), _ptr(m_shift), _ptr(w_mk),
                                              _ptr(w_mv), _ptr(dR_k), _ptr(dR_v), _ptr(dm_shift), _ptr(dw_mk),
                                              _ptr(dw_mv), _stream(stream)))


def maglev_consistency_loss(m, m_target, rows, d, dtype, lam, inv_count, loss, dm, dm_target,
                            accumulate_dm, workspace, stream=None):
    _check(_lib.maglev_consistency_loss(_ptr(m), _ptr(m_target), int(rows), int(d), int(dtype),
                                        float(lam), float(inv_count), _ptr(loss), _ptr(dm),
                                        _ptr(dm_target), int(accumulate_dm), _ptr(workspace),
                                        _stream(stream)))


def maglev_consistency_loss_prepare_bwd(desc, out, m_target, lam, inv_count, loss, dout, bwd_workspace,
                                        loss_workspace, stream=None):
    _check(_lib.maglev_consistency_loss_prepare_bwd(ctypes.byref(desc), _ptr(out), _ptr(m_target), float(lam),
                                                    float(inv_count), _ptr(loss), _ptr(dout),
                                                    _ptr(bwd_workspace), _ptr(loss_workspace), _stream(stream)))


def maglev_consistency_loss_noalloc(m, m_target, rows, d, dtype, lam, inv_count, loss, dm, dm_target,
                                    accumulate_dm, stream=None):
    """Scratch-free consistency loss: same results as maglev_consistency_loss,
    no workspace argument (for callers that cannot allocate device memory)."""
    _check(_lib.maglev_consistency_loss_noalloc(_ptr(m), _ptr(m_target), int(rows), int(d), int(dtype),
                                                float(lam), float(inv_count), _ptr(loss), _ptr(dm),
                                                _ptr(dm_target), int(accumulate_dm), _stream(stream)))


def maglev_memory_state(B, T, d, eps, dtype, o, m, m_shift, rstd, stream=None):
    _check(_lib.maglev_memory_state(int(B), int(T), int(d), float(eps), int(dtype), _ptr(o), _ptr(m),
                                    _ptr(m_shift), _ptr(rstd), _stream(stream)))


def maglev_memory_state_bwd(B, T, d, dtype, o, rstd, dm, dm_shift, dout_in, d_o, stream=None):
    _check(_lib.maglev_memory_state_bwd(int(B), int(T), int(d), int(dtype), _ptr(o), _ptr(rstd), _ptr(dm),
                                        _ptr(dm_shift), _ptr(dout_in), _ptr(d_o), _stream(stream)))


def maglev_decode_mem_project(desc, pos, m_prev, w_mk, w_mv, krec_rot, vrec, stream=None):
    _check(_lib.maglev_decode_mem_project(ctypes.byref(desc), _ptr(pos), _ptr(m_prev), _ptr(w_mk),
                                          _ptr(w_mv), _ptr(krec_rot), _ptr(vrec), _stream(stream)))


def maglev_decode_workspace_bytes(desc) -> int:
    return _lib.maglev_decode_workspace_bytes(ctypes.byref(desc))


def maglev_decode_step(desc, pos, q, k, v, krec_rot, vrec, gate_logits, k_ring, v_ring, out, workspace,
                       stream=None):
    _check(_lib.maglev_decode_step(ctypes.byref(desc), _ptr(pos), _ptr(q), _ptr(k), _ptr(v),
                                   _ptr(krec_rot), _ptr(vrec), _ptr(gate_logits), _ptr(k_ring),
                                   _ptr(v_ring), _ptr(out), _ptr(workspace), _stream(stream)))


def maglev_decode_prefill(desc, saved, k_ring, v_ring, stream=None):
    _check(_lib.maglev_decode_prefill(ctypes.byref(desc), _ptr(saved), _ptr(k_ring), _ptr(v_ring),
                                      _stream(stream)))


def maglev_lm_head_workspace_bytes(N: int, d: int, V: int) -> int:
    return _lib.maglev_lm_head_workspace_bytes(int(N), int(d), int(V))


def maglev_lm_head_ce(N, d, V, dtype, softcap, inv_count, m, U, targets, loss, lse, dm, dU, workspace,
                      spin_limit=0, stream=None):
    _check(_lib.maglev_lm_head_ce(int(N), int(d), int(V), int(dtype), float(softcap), float(inv_count), _ptr(m),
                                  _ptr(U), _ptr(targets), _ptr(loss), _ptr(lse), _ptr(dm), _ptr(dU),
                                  _ptr(workspace), int(spin_limit), _stream(stream)))


def maglev_wait_selftest(src, nbytes, spin_limit, stream=None):
    _check(_lib.maglev_wait_selftest(_ptr(src), int(nbytes), int(spin_limit), _stream(stream)))
