"""The C-ABI library loads without a GPU, exports every entry point that
include/flashmask.h declares, and rejects bad arguments on the host before
touching a device (CPU only; no compute calls)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "flashmask.h")


@pytest.fixture(scope="module")
def lib():
    from column_sparse_masked_b200 import build

    build.build()
    import column_sparse_masked_b200 as fm

    return fm.load_library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(flashmask_[a-z_]+)\s*\(", text)))


def test_header_declares_entry_points():
    names = declared_functions()
    for n in ("flashmask_fwd", "flashmask_bwd", "flashmask_classify", "flashmask_localize",
              "flashmask_fwd_workspace_size", "flashmask_bwd_workspace_size", "flashmask_get_status"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for n in declared_functions():
        assert hasattr(lib, n), n


def test_exported_symbols_are_c_linkage(lib):
    # dlsym by the plain C name succeeds (no C++ mangling)
    for n in declared_functions():
        assert ctypes.cast(getattr(lib, n), ctypes.c_void_p).value


def test_strerror_and_version(lib):
    lib.flashmask_strerror.restype = ctypes.c_char_p
    for code in range(0, -8, -1):
        assert lib.flashmask_strerror(code)
    assert b"unknown" in lib.flashmask_strerror(-99)
    assert lib.flashmask_version() >= 100


def _dims(**kw):
    from column_sparse_masked_b200._binding import _Dims

    base = dict(B=1, Hq=4, Hkv=2, Hm=1, Nq=1000, Nk=777, d=128)
    base.update(kw)
    return _Dims(*[base[k] for k in ("B", "Hq", "Hkv", "Hm", "Nq", "Nk", "d")])


def test_workspace_sizes(lib):
    d = _dims()
    f = lib.flashmask_fwd_workspace_size(ctypes.byref(d))
    b = lib.flashmask_bwd_workspace_size(ctypes.byref(d))
    assert 0 < f < b
    # backward holds at least D and LSE2 over whole 128-row tiles (B=1, Hq=4, 8 tiles)
    assert b - f >= 2 * 1 * 4 * 8 * 128 * 4
    assert lib.flashmask_fwd_workspace_size(ctypes.byref(_dims(d=96))) == 0


def test_fwd_pairing_toggle_and_workspace(lib):
    """Host-only: the pairing switch accepts 0 and 1, and the forward workspace size covers the
    paired layout (one list per q-tile) whichever setting a later call uses."""
    assert lib.flashmask_get_fwd_pairing() == 1
    assert lib.flashmask_set_fwd_pairing(2) == -1
    assert lib.flashmask_set_fwd_pairing(0) == 0 and lib.flashmask_get_fwd_pairing() == 0
    f_off = lib.flashmask_fwd_workspace_size(ctypes.byref(_dims(Nq=4096, Nk=4096)))
    assert lib.flashmask_set_fwd_pairing(1) == 0 and lib.flashmask_get_fwd_pairing() == 1
    f_on = lib.flashmask_fwd_workspace_size(ctypes.byref(_dims(Nq=4096, Nk=4096)))
    assert f_on == f_off > 0  # the size does not depend on the switch


@pytest.mark.parametrize("kw,code", [
    (dict(d=96), -2), (dict(Hq=3, Hkv=2), -1), (dict(Hm=2), -1), (dict(Nq=-1), -1), (dict(Hkv=0), -1),
])
def test_host_side_validation(lib, kw, code):
    d = _dims(**kw)
    rc = lib.flashmask_fwd(None, None, None, None, None, None, None, ctypes.c_float(0.0), ctypes.byref(d),
                           None, None, None, ctypes.c_size_t(0), None)
    assert rc == code


def test_mask_pair_must_be_complete(lib):
    d = _dims()
    buf = (ctypes.c_int32 * 4096)()
    rc = lib.flashmask_fwd(None, None, None, ctypes.cast(buf, ctypes.c_void_p), None, None, None,
                           ctypes.c_float(0.0), ctypes.byref(d), None, None, None, ctypes.c_size_t(0), None)
    assert rc == -1


def test_timeout_info_rejects_null(lib):
    # checked on the host before any device access
    assert lib.flashmask_get_timeout_info(None) == -1


def test_localize_argument_checks(lib):
    assert lib.flashmask_localize(None, None, ctypes.c_int64(-1), 0, 1, None) == -1
    assert lib.flashmask_localize(None, None, ctypes.c_int64(10), 5, 2, None) == -1
    assert lib.flashmask_localize(None, None, ctypes.c_int64(0), 0, 1, None) == 0
    a = (ctypes.c_int32 * 2)(0, 5)
    b = (ctypes.c_int32 * 2)(10, 20)  # overlapping chunks
    assert lib.flashmask_localize_multi(None, None, ctypes.c_int64(4), a, b, 2, None) == -1


def test_checks_build_exports_every_declared_symbol():
    """The checks build (FLASHMASK_CHECKS) has the same C ABI."""
    from column_sparse_masked_b200 import build

    path = build.build(checks=True)
    chk = ctypes.CDLL(path)
    for n in declared_functions():
        assert hasattr(chk, n), n
    chk.flashmask_strerror.restype = ctypes.c_char_p
    assert b"checks build" in chk.flashmask_strerror(-9)
