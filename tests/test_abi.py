"""The C-ABI library builds, loads and exports every symbol the header declares; host
argument checks that need no device.  CPU only (no compute calls)."""
import ctypes
import os
import re

import pytest
import torch

import muon_newton_schulz_06_b200 as mb
from muon_newton_schulz_06_b200 import build as mbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "muon.h")


@pytest.fixture(scope="module")
def lib():
    mbuild.build()
    return mb.load_library()


def declared_symbols():
    text = open(HEADER).read()
    return re.findall(r"MUON_API\s+[\w\s\*]+?\b(muon_\w+)\s*\(", text)


def test_header_declares_the_binding_names():
    names = declared_symbols()
    assert sorted(names) == sorted(mb.EXPORTED)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name


def test_status_strings(lib):
    names = ["MUON_OK", "MUON_ERR_INVALID_ARG", "MUON_ERR_UNSUPPORTED", "MUON_ERR_OOM", "MUON_ERR_CUDA",
             "MUON_ERR_TIMEOUT", "MUON_ERR_TOO_LARGE", "MUON_ERR_CORRUPT"]
    for code, name in enumerate(names):
        assert mb.muon_status_string(code).startswith(name)
        assert getattr(mb, name) == code
    assert "unknown" in mb.muon_status_string(99)


def test_null_handle_is_rejected_before_any_device_call(lib):
    assert lib.muon_destroy(None) == mb.MUON_OK
    assert lib.muon_step(None, None, 0, 0.02, 0.95, 1, None, 5, 1e-7, 0, None) == mb.MUON_ERR_INVALID_ARG
    assert lib.muon_newton_schulz(None, None, None, None, None, 0, 1, None, 5, 1e-7, 0, None) \
        == mb.MUON_ERR_INVALID_ARG
    assert lib.muon_sync(None) == mb.MUON_ERR_INVALID_ARG
    assert lib.muon_set_launch_mode(None, 0) == mb.MUON_ERR_INVALID_ARG
    assert lib.muon_selftest_fail_next_alloc(None) == mb.MUON_ERR_INVALID_ARG
    assert lib.muon_selftest_stall_persistent(None, 1000) == mb.MUON_ERR_INVALID_ARG
    assert lib.muon_selftest_corrupt_guard(None) == mb.MUON_ERR_INVALID_ARG
    assert lib.muon_workspace_bytes(None) == 0
    assert lib.muon_last_error(None) == b""
    out = ctypes.c_void_p()
    assert lib.muon_init(None, 0) == mb.MUON_ERR_INVALID_ARG


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device path")
def test_init_without_device_fails_cleanly(lib):
    out = ctypes.c_void_p(1234)
    code = lib.muon_init(ctypes.byref(out), 0)
    assert code in (mb.MUON_ERR_CUDA, mb.MUON_ERR_INVALID_ARG, mb.MUON_ERR_UNSUPPORTED)
    assert out.value is None
    with pytest.raises(mb.MuonError):
        mb.muon_init(0)


def test_binding_rejects_cpu_tensors(lib):
    w = torch.zeros(4, 4)
    with pytest.raises(TypeError):
        mb.muon_step(None, [w], [w], [w], lr=0.1)
