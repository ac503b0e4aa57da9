"""Host-side checks of the C ABI: the library loads, exports every entry point
include/maglev.h declares, and validates its arguments before any launch
(no GPU needed: no call here reaches a kernel)."""
import ctypes

import pytest

from sliding_window_recurrent_b200 import build as _build

_build.build(quiet=True)

import sliding_window_recurrent_b200 as mg  # noqa: E402


def desc(**kw):
    base = dict(B=1, T=16, H=2, hd=64, d_mem=32, window=8, rope_base=10000.0, rms_eps=1e-6,
                inject=1, pos0=0, dtype=mg.MAGLEV_F32, spin_limit=0)
    base.update(kw)
    return mg.SwaDesc(**base)


def test_every_declared_symbol_is_exported():
    names = mg.header_symbols()
    assert len(names) >= 13
    lib = ctypes.CDLL(mg.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n


def test_version():
    assert "sm_100a" in mg.maglev_version()


def test_sizes():
    d = desc(B=2, T=100, H=3, hd=128, dtype=mg.MAGLEV_BF16)
    n = 2 * 100 * 3 * 128 * 2
    assert mg.maglev_swa_saved_bytes(d) >= 3 * n
    assert mg.maglev_swa_bwd_workspace_bytes(d) >= 2 * (n * 2)
    assert mg.maglev_swa_saved_bytes(desc(hd=96)) == 0          # invalid desc -> 0
    assert mg.maglev_consistency_workspace_bytes(1000, 1280) >= 4


FAKE = 1 << 20   # aligned, never dereferenced: validation fails first


@pytest.mark.parametrize("bad,status", [
    (dict(hd=96), mg.MAGLEV_ERR_UNSUPPORTED),
    (dict(window=0), mg.MAGLEV_ERR_INVALID_ARG),
    (dict(H=0), mg.MAGLEV_ERR_INVALID_ARG),
    (dict(T=-1), mg.MAGLEV_ERR_INVALID_ARG),
    (dict(dtype=7), mg.MAGLEV_ERR_INVALID_ARG),
    (dict(pos0=-3), mg.MAGLEV_ERR_INVALID_ARG),
    (dict(rope_base=0.5), mg.MAGLEV_ERR_INVALID_ARG),
    (dict(d_mem=0), mg.MAGLEV_ERR_INVALID_ARG),
])
def test_fwd_rejects_bad_desc(bad, status):
    with pytest.raises(mg.MaglevError) as e:
        mg.maglev_inject_swa_fwd(desc(**bad), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                                 FAKE, FAKE, FAKE, stream=0)
    assert e.value.status == status


def test_fwd_rejects_null_and_misaligned_pointers():
    with pytest.raises(mg.MaglevError) as e:
        mg.maglev_inject_swa_fwd(desc(), None, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                                 FAKE, FAKE, FAKE, stream=0)
    assert e.value.status == mg.MAGLEV_ERR_INVALID_ARG and "q" in str(e.value)
    with pytest.raises(mg.MaglevError) as e:
        mg.maglev_inject_swa_fwd(desc(), FAKE, FAKE + 4, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                                 FAKE, FAKE, FAKE, stream=0)
    assert "aligned" in str(e.value)
    # injection needs gate logits
    with pytest.raises(mg.MaglevError):
        mg.maglev_inject_swa_fwd(desc(), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None,
                                 FAKE, FAKE, FAKE, stream=0)


def test_empty_problems_enqueue_nothing():
    # B = 0 or T = 0 is valid and returns before any launch.
    for d in (desc(B=0), desc(T=0)):
        mg.maglev_inject_swa_fwd(d, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                                 FAKE, FAKE, stream=0)
        mg.maglev_inject_swa_bwd(d, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                                 FAKE, FAKE, FAKE, FAKE, None, None, mg.MAGLEV_DR_WRITE, FAKE, FAKE,
                                 FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, stream=0)
    mg.maglev_consistency_loss(FAKE, FAKE, 0, 16, mg.MAGLEV_F32, 1.0, 0.0, FAKE, None, None, 0,
                               FAKE, stream=0)


def test_loss_prepare_bwd_validation():
    """The fused loss / backward-preparation call checks its descriptor and
    pointers before any launch; an empty problem enqueues nothing; the flag it
    pairs with is accepted by the backward's dR_mode check (mode 7 | flag is not)."""
    mg.maglev_consistency_loss_prepare_bwd(desc(B=0), FAKE, FAKE, 0.1, 0.0, FAKE, FAKE, FAKE, FAKE, stream=0)
    with pytest.raises(mg.MaglevError) as e:
        mg.maglev_consistency_loss_prepare_bwd(desc(), FAKE, FAKE, 0.1, 0.0, None, FAKE, FAKE, FAKE, stream=0)
    assert e.value.status == mg.MAGLEV_ERR_INVALID_ARG and "loss" in str(e.value)
    with pytest.raises(mg.MaglevError) as e:
        mg.maglev_consistency_loss_prepare_bwd(desc(), FAKE, FAKE, 0.1, 0.0, FAKE, FAKE, None, FAKE, stream=0)
    assert e.value.status == mg.MAGLEV_ERR_INVALID_ARG and "bwd_workspace" in str(e.value)
    with pytest.raises(mg.MaglevError) as e:
        mg.maglev_consistency_loss_prepare_bwd(desc(), FAKE, FAKE, float("inf"), 0.0, FAKE, FAKE, FAKE, FAKE,
                                               stream=0)
    assert e.value.status == mg.MAGLEV_ERR_INVALID_ARG
    with pytest.raises(mg.MaglevError) as e:
        mg.maglev_consistency_loss_prepare_bwd(desc(hd=96), FAKE, FAKE, 0.1, 0.0, FAKE, FAKE, FAKE, FAKE,
                                               stream=0)
    assert e.value.status == mg.MAGLEV_ERR_UNSUPPORTED
    with pytest.raises(mg.MaglevError) as e:
        mg.maglev_inject_swa_bwd(desc(), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                                 FAKE, FAKE, FAKE, None, None, FAKE, FAKE, 7 | mg.MAGLEV_BWD_PREPARED, FAKE,
                                 None, FAKE, FAKE, None, None, None, FAKE, stream=0)
    assert e.value.status == mg.MAGLEV_ERR_INVALID_ARG and "dR_mode 7" in str(e.value)


def test_bwd_and_loss_and_decode_validation():
    with pytest.raises(mg.MaglevError):  # dR_k is needed in mode WRITE
        mg.maglev_inject_swa_bwd(desc(), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                                 FAKE, FAKE, FAKE, None, FAKE, None, None, mg.MAGLEV_DR_WRITE, FAKE,
                                 None, None, None, None, None, None, FAKE, stream=0)
    for mode, acc, m_shift, what in [(mg.MAGLEV_DR_ADD, None, None, "dR_acc_k"),
                                     (7, FAKE, None, "dR_mode"),
                                     (mg.MAGLEV_DR_FIRST, FAKE, FAKE, "m_shift")]:
        with pytest.raises(mg.MaglevError) as e:
            mg.maglev_inject_swa_bwd(desc(), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                                     FAKE, FAKE, FAKE, None, None, acc, acc, mode, FAKE,
                                     m_shift, FAKE, FAKE, None, None, None, FAKE, stream=0)
        assert e.value.status == mg.MAGLEV_ERR_INVALID_ARG and what in str(e.value), str(e.value)
    with pytest.raises(mg.MaglevError):
        mg.maglev_consistency_loss(FAKE, FAKE, 10, 0, mg.MAGLEV_F32, 1.0, 0.0, FAKE, None, None,
                                   0, FAKE, stream=0)
    with pytest.raises(mg.MaglevError):
        mg.maglev_consistency_loss(FAKE, FAKE, 10, 8, mg.MAGLEV_F32, float("nan"), 0.0, FAKE,
                                   None, None, 0, FAKE, stream=0)
    dd = mg.DecodeDesc(B=2, H=2, hd=64, d_mem=16, window=0, rope_base=1e4, rms_eps=1e-6,
                       inject=1, dtype=mg.MAGLEV_F32, spin_limit=0)
    with pytest.raises(mg.MaglevError):
        mg.maglev_decode_step(dd, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, stream=0)
    dd.window = 64
    dd.hd = 80
    with pytest.raises(mg.MaglevError) as e:
        mg.maglev_decode_step(dd, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, stream=0)
    assert e.value.status == mg.MAGLEV_ERR_UNSUPPORTED
    dd.hd = 64
    dd.B = 0
    mg.maglev_decode_step(dd, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, stream=0)


def test_driver_modules_only_call_bound_entry_points():
    """Every maglev_* name the Python drivers (layer.py, stack.py) call is
    imported there and bound by the package (a missing import only shows at
    call time, on the GPU)."""
    import re
    import sliding_window_recurrent_b200.layer as layer
    import sliding_window_recurrent_b200.stack as stack
    for mod in (layer, stack):
        src = open(mod.__file__).read()
        for name in set(re.findall(r"\b(maglev_[a-z0-9_]+)\(", src)):
            assert hasattr(mod, name), (mod.__name__, name)
            assert hasattr(mg, name), name


def test_debug_build_exports_every_symbol():
    """The debug build (-DMAGLEV_DEBUG: in-kernel index checks that record
    MAGLEV_ERR_BOUNDS) is a drop-in for the release library."""
    path = _build.build(quiet=True, debug=True)
    lib = ctypes.CDLL(path)
    for n in mg.header_symbols():
        assert hasattr(lib, n), n
    assert mg.MAGLEV_ERR_BOUNDS == 5
