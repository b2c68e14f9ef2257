"""The C-ABI library loads and exports every declared entry point (no GPU).

Only host-side argument checks that run before any CUDA call are exercised
here; compute calls need a GPU and live in the gpu-marked tests.
"""
import ctypes
import os
import re

import pytest

from group_circulant_linear_b200 import eqlin

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "eqlin.h")


def declared_symbols():
    with open(HEADER) as f:
        src = f.read()
    return sorted(set(re.findall(r"EQLIN_API\s+[^;(]*?\b(eqlin_\w+)\s*\(", src)))


def test_header_declares_the_abi():
    syms = declared_symbols()
    for name in ("eqlin_create", "eqlin_set_weights", "eqlin_forward", "eqlin_backward_dx",
                 "eqlin_backward_dw", "eqlin_get_error", "eqlin_status_string", "eqlin_destroy"):
        assert name in syms
    assert set(syms) == set(eqlin.SIGNATURES), "binding and header disagree"


def test_library_exports_every_declared_symbol():
    L = eqlin.lib()
    for name in declared_symbols():
        assert hasattr(L, name), name
    # and nothing else leaks out under the eqlin_ prefix
    out = os.popen(f"nm -D --defined-only {eqlin.LIB_PATH}").read()
    exported = sorted(set(re.findall(r" T (eqlin_\w+)", out)))
    assert exported == declared_symbols()


def test_status_strings():
    L = eqlin.lib()
    for code in eqlin.STATUS:
        assert L.eqlin_status_string(code)
    assert L.eqlin_status_string(-6) == b"device-side wait timed out"


def test_create_rejects_bad_arguments_before_touching_cuda():
    L = eqlin.lib()
    out = ctypes.c_void_p()
    assert L.eqlin_create(5, 16, 16, eqlin.F32, ctypes.byref(out)) == -2   # T = 5
    assert L.eqlin_create(12, 16, 16, eqlin.F32, ctypes.byref(out)) == -2  # T = 12
    assert L.eqlin_create(16, 16, 16, eqlin.F32, ctypes.byref(out)) == -2  # T = 16
    assert L.eqlin_create(4, 0, 16, eqlin.F32, ctypes.byref(out)) == -1
    assert L.eqlin_create(4, 16, -1, eqlin.F32, ctypes.byref(out)) == -1
    assert L.eqlin_create(4, 16, 16, 7, ctypes.byref(out)) == -1
    assert L.eqlin_create(4, 16, 16, eqlin.F32, None) == -1
    assert L.eqlin_create_group(2, 4, 16, 16, eqlin.F32, ctypes.byref(out)) == -1   # no such group
    assert L.eqlin_create_group(eqlin.DIHEDRAL, 7, 16, 16, eqlin.F32, ctypes.byref(out)) == -2
    assert L.eqlin_create_group(eqlin.DIHEDRAL, 0, 16, 16, eqlin.F32, ctypes.byref(out)) == -2
    assert L.eqlin_create_group(eqlin.CYCLIC, 5, 16, 16, eqlin.F32, ctypes.byref(out)) == -2
    assert L.eqlin_create_group(eqlin.DIHEDRAL, 1, 3, 8, eqlin.F16, ctypes.byref(out)) == -3  # 12-byte rows
    assert L.eqlin_create(1, 3, 8, eqlin.F16, ctypes.byref(out)) == -3     # 6-byte rows
    assert out.value is None


def test_null_handle_calls():
    L = eqlin.lib()
    assert L.eqlin_forward(None, None, None, 0, None) == -1
    assert L.eqlin_backward_dx(None, None, None, 0, None) == -1
    assert L.eqlin_backward_dw(None, None, None, None, None, 0, None) == -1
    assert L.eqlin_set_weights(None, None, None, None) == -1
    assert L.eqlin_get_error(None) == -1
    assert L.eqlin_backend_name(None) == b"none"
    assert L.eqlin_forward_stash(None, None, None, None, 0, None) == -1
    assert L.eqlin_backward_dx_stash(None, None, None, None, 0, None) == -1
    assert L.eqlin_backward_dw_spectra(None, None, None, None, None, 0, None) == -1
    assert L.eqlin_backward(None, None, None, None, None, None, None, 0, None) == -1
    assert L.eqlin_set_tail_split(None, 1) == -1
    assert L.eqlin_set_wait_limit(None, 1) == -1
    L.eqlin_destroy(None)


def test_spectra_row_pitch():
    L = eqlin.lib()
    assert [L.eqlin_spectra_ld(n) for n in (0, 1, 63, 64, 65, 12608, 401408)] == \
        [0, 64, 64, 64, 128, 12608, 401408]
    assert L.eqlin_spectra_ld(-1) == -1


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(eqlin, "_lib", None)
    monkeypatch.setattr(eqlin, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="missing"):
        eqlin.lib()
