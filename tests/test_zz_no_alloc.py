"""Allocation-free entry point (muon_newton_schulz_noalloc), for callers that may not
allocate device memory when they need the update: runtimes that reserve all device
memory for their own pool at start-up, or engines that forbid allocation once they
run.  Called through the C ABI and compared with the allocating entry point,
muon_newton_schulz (same kernels in the same order, so the same bits), on two calls
in a row, and with the float64 oracle within the bf16 bar.

Collected last on purpose (file name), so that a run stopping at the first failure has
already run every other test; it also passes alone in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu

BF16_TOL = 2e-2
Q = oracle.QUINTIC
# invented per-step table (rows differ; each step bounded on (0, 1.3])
TABLE5 = [Q, tuple(0.9 * v for v in Q), oracle.CUBIC, (2.0, -1.5, 0.5), (3.0, -3.2, 1.2)]


@pytest.fixture(scope="module")
def mb():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import muon_newton_schulz_06_b200 as m
    from muon_newton_schulz_06_b200 import build
    build.build()
    return m


def rel(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def to64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def c_table(table):
    if table is None:
        return None
    flat = [float(v) for row in table for v in row]
    return (ctypes.c_float * len(flat))(*flat)


def call_noalloc(lib, x, out, status=None, table=None, x_ptr=None, out_ptr=None, stream=None):
    """Raw C-ABI call; x_ptr / out_ptr override the tensors' addresses."""
    stream = torch.cuda.current_stream().cuda_stream if stream is None else stream
    dt = 1 if x.dtype == torch.bfloat16 else 0
    ns = len(table) if table is not None else 5
    return lib.muon_newton_schulz_noalloc(
        ctypes.c_void_p(x.data_ptr() if x_ptr is None else x_ptr),
        ctypes.c_void_p(out.data_ptr() if out_ptr is None else out_ptr),
        x.shape[0], x.shape[1], dt, c_table(table), ns, ctypes.c_float(1e-7),
        ctypes.c_void_p(status.data_ptr() if status is not None else None), ctypes.c_void_p(stream))


def reference(mb, x, table=None):
    """The allocating entry point on the same input (its own handle and workspace)."""
    ref = torch.empty_like(x)
    h = mb.muon_init(torch.cuda.current_device())
    try:
        mb.muon_newton_schulz(h, [x], [ref], coeffs=table, ns_steps=len(table) if table else 5)
        torch.cuda.synchronize()
        mb.muon_sync(h)
    finally:
        mb.muon_destroy(h)
    return ref


def ns_oracle(x, table=None):
    return oracle.newton_schulz(oracle.frobenius_normalise(to64(x), 1e-7), table or [Q] * 5)


CASES = [(1024, 3072, torch.bfloat16), (300, 200, torch.bfloat16), (130, 130, torch.bfloat16),
         (64, 1000, torch.bfloat16), (1000, 517, torch.bfloat16), (517, 300, torch.float32),
         (96, 1000, torch.float32)]


@pytest.mark.parametrize("rows,cols,dtype", CASES)
def test_noalloc_matches_allocating_entry_point_twice(mb, rows, cols, dtype):
    lib = mb.load_library()
    x = synth.random_matrix(rows, cols, seed=rows + cols, device="cuda", dtype=dtype)
    ref = reference(mb, x)
    want = ns_oracle(x)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for call in range(2):
        out = torch.full_like(x, float("nan"))
        assert call_noalloc(lib, x, out, status) == mb.MUON_OK
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        assert torch.equal(out, ref), (call, rows, cols)
        err = rel(to64(out), want)
        assert err < BF16_TOL, (call, rows, cols, err)


def test_noalloc_coefficient_table_and_no_status(mb):
    """A per-step table whose rows differ, status = NULL: the same bits as the
    allocating entry point with that table, and the oracle's result with it."""
    lib = mb.load_library()
    for i, (r, c) in enumerate([(300, 130), (130, 301), (512, 1024)]):
        x = synth.random_matrix(r, c, seed=70 + i, device="cuda", dtype=torch.bfloat16)
        ref = reference(mb, x, TABLE5)
        for call in range(2):
            out = torch.full_like(x, float("nan"))
            assert call_noalloc(lib, x, out, None, TABLE5) == mb.MUON_OK
            torch.cuda.synchronize()
            assert torch.equal(out, ref), (call, r, c)
        assert rel(to64(out), ns_oracle(x, TABLE5)) < BF16_TOL
        assert rel(to64(out), ns_oracle(x)) > 0.1  # the table was used


def test_noalloc_allocates_nothing(mb):
    """After a first call (which loads the kernels), further calls leave the device's
    free memory unchanged."""
    lib = mb.load_library()
    x = synth.random_matrix(700, 1500, seed=5, device="cuda", dtype=torch.bfloat16)
    out = torch.empty_like(x)
    assert call_noalloc(lib, x, out) == mb.MUON_OK
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(3):
        assert call_noalloc(lib, x, out) == mb.MUON_OK
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0


def test_noalloc_rejects_memory_of_another_device_before_enqueueing(mb):
    """Host memory (pinned or pageable) in place of device memory of the current device
    is an argument error, returned before anything is enqueued."""
    lib = mb.load_library()
    x = synth.random_matrix(128, 256, seed=9, device="cuda", dtype=torch.bfloat16)
    out = torch.full_like(x, float("nan"))
    pinned = torch.zeros(128, 256, dtype=torch.bfloat16).pin_memory()
    pageable = torch.zeros(128, 256, dtype=torch.bfloat16)
    assert call_noalloc(lib, x, out, out_ptr=pinned.data_ptr()) == mb.MUON_ERR_INVALID_ARG
    assert call_noalloc(lib, x, out, x_ptr=pageable.data_ptr()) == mb.MUON_ERR_INVALID_ARG
    status_host = torch.zeros(4, dtype=torch.int32).pin_memory()
    assert lib.muon_newton_schulz_noalloc(ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(out.data_ptr()), 128, 256,
                                          1, None, 5, ctypes.c_float(1e-7), ctypes.c_void_p(status_host.data_ptr()),
                                          ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)) \
        == mb.MUON_ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert torch.isnan(out.float()).all()
    assert torch.count_nonzero(pinned) == 0
    # the binding checks devices too
    with pytest.raises(TypeError):
        mb.muon_newton_schulz_noalloc(x, pageable)


def test_noalloc_rejects_matrices_beyond_the_scratch(mb):
    lib = mb.load_library()
    x = torch.zeros(2048, 2048, dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(x)
    assert call_noalloc(lib, x, out) == mb.MUON_ERR_TOO_LARGE
    assert "fixed scratch" in mb.muon_status_string(mb.MUON_ERR_TOO_LARGE)
