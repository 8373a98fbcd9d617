"""Allocation-free entry point (muon_newton_schulz_noalloc), for callers that may not
allocate device memory when they need the update.  Called through the C ABI and
compared with the allocating entry point, muon_newton_schulz, on two calls in a row.

Collected last on purpose (file name), so that a run stopping at the first failure has
already run every other test; it also passes alone in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu

BF16_TOL = 2e-2


@pytest.fixture(scope="module")
def mb():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import muon_newton_schulz_06_b200 as m
    from muon_newton_schulz_06_b200 import build
    build.build()
    return m


def rel(a, b):
    a = a.double().cpu().numpy()
    b = b.double().cpu().numpy()
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def call_noalloc(lib, x, out, status=None, ns_steps=5):
    stream = torch.cuda.current_stream().cuda_stream
    dt = 1 if x.dtype == torch.bfloat16 else 0
    return lib.muon_newton_schulz_noalloc(ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(out.data_ptr()),
                                          x.shape[0], x.shape[1], dt, None, ns_steps, ctypes.c_float(1e-7),
                                          ctypes.c_void_p(status.data_ptr() if status is not None else None),
                                          ctypes.c_void_p(stream))


@pytest.mark.parametrize("rows,cols", [(1024, 3072), (300, 200), (130, 130), (64, 1000)])
def test_noalloc_matches_allocating_entry_point_twice(mb, rows, cols):
    lib = mb.load_library()
    x = synth.random_matrix(rows, cols, seed=rows + cols, device="cuda", dtype=torch.bfloat16)
    ref = torch.empty_like(x)
    h = mb.muon_init(torch.cuda.current_device())
    try:
        mb.muon_newton_schulz(h, [x], [ref])
        torch.cuda.synchronize()
        mb.muon_sync(h)
    finally:
        mb.muon_destroy(h)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for call in range(2):
        out = torch.full_like(x, float("nan"))
        assert call_noalloc(lib, x, out, status) == mb.MUON_OK
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        err = rel(out, ref)
        assert err < BF16_TOL, (call, rows, cols, err)


def test_noalloc_rejects_matrices_beyond_the_scratch(mb):
    lib = mb.load_library()
    x = torch.zeros(2048, 2048, dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(x)
    assert call_noalloc(lib, x, out) == mb.MUON_ERR_TOO_LARGE
    assert "fixed scratch" in mb.muon_status_string(mb.MUON_ERR_TOO_LARGE)
