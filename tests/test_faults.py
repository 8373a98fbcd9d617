"""Failure detection without a GPU fault, and the hygiene paths around it.

The library bounds every device-side wait; when one expires, the kernel records a
time-out in the handle's status word and returns, and the host reports
MUON_ERR_TIMEOUT.  Here the wait runs out on purpose: a diagnostic kernel waits on a
barrier that nothing completes, with a 1 ms limit.  Nothing faults, traps or hangs.
"""
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mb():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import muon_newton_schulz_06_b200 as m
    from muon_newton_schulz_06_b200 import build
    build.build()
    return m


def test_timeout_is_reported_by_sync_and_cleared(mb):
    h = mb.muon_init(0)
    try:
        mb.muon_selftest_wait_timeout(h, 1_000_000)
        with pytest.raises(mb.MuonError) as e:
            mb.muon_sync(h)
        assert e.value.code == mb.MUON_ERR_TIMEOUT
        mb.muon_sync(h)  # cleared
    finally:
        mb.muon_destroy(h)


def test_timeout_is_reported_by_the_next_call_then_work_continues(mb):
    h = mb.muon_init(0)
    try:
        w = torch.zeros(64, 32, device="cuda")
        g = torch.randn(64, 32, device="cuda")
        m = torch.zeros(64, 32, device="cuda")
        mb.muon_selftest_wait_timeout(h, 1_000_000)
        torch.cuda.synchronize()
        with pytest.raises(mb.MuonError) as e:
            mb.muon_step(h, [w], [g], [m], lr=1.0)
        assert e.value.code == mb.MUON_ERR_TIMEOUT
        assert torch.count_nonzero(m) == 0  # the failed call enqueued nothing
        mb.muon_step(h, [w], [g], [m], lr=1.0)
        torch.cuda.synchronize()
        mb.muon_sync(h)
        assert torch.count_nonzero(w) > 0 and torch.equal(m, g)
    finally:
        mb.muon_destroy(h)


def test_wait_that_is_satisfied_reports_nothing(mb):
    h = mb.muon_init(0)
    try:
        w = torch.zeros(16, 16, device="cuda")
        mb.muon_step(h, [w], [torch.ones(16, 16, device="cuda")], [torch.zeros(16, 16, device="cuda")], lr=0.1)
        torch.cuda.synchronize()
        mb.muon_sync(h)
    finally:
        mb.muon_destroy(h)


def test_selftest_rejects_bad_limits(mb):
    h = mb.muon_init(0)
    try:
        with pytest.raises(mb.MuonError) as e:
            mb.muon_selftest_wait_timeout(h, -1)
        assert e.value.code == mb.MUON_ERR_INVALID_ARG
    finally:
        mb.muon_destroy(h)


# ---------------------------------------------------------------- allocation failure (injected on the host)

def test_injected_allocation_failure_leaves_the_handle_usable(mb):
    """The workspace allocation is made to fail on the host (no device fault): the call
    returns MUON_ERR_OOM with nothing enqueued, and the next call allocates and runs."""
    h = mb.muon_init(0)
    try:
        w = torch.zeros(64, 32, device="cuda")
        g = torch.randn(64, 32, device="cuda")
        m = torch.zeros(64, 32, device="cuda")
        mb.muon_selftest_fail_next_alloc(h)
        with pytest.raises(mb.MuonError) as e:
            mb.muon_step(h, [w], [g], [m], lr=1.0)
        assert e.value.code == mb.MUON_ERR_OOM
        assert "injected" in str(e.value)
        torch.cuda.synchronize()
        assert torch.count_nonzero(m) == 0 and torch.count_nonzero(w) == 0
        assert mb.muon_workspace_bytes(h) == 0
        mb.muon_step(h, [w], [g], [m], lr=1.0)
        torch.cuda.synchronize()
        mb.muon_sync(h)
        assert torch.equal(m, g) and torch.count_nonzero(w) > 0
        held = mb.muon_workspace_bytes(h)
        assert held > 0
        # a handle that holds a workspace and must grow it: the old one is released first
        W = [torch.zeros(512, 256, device="cuda") for _ in range(3)]
        G = [torch.randn(512, 256, device="cuda") for _ in range(3)]
        M = [torch.zeros(512, 256, device="cuda") for _ in range(3)]
        mb.muon_selftest_fail_next_alloc(h)
        with pytest.raises(mb.MuonError) as e:
            mb.muon_step(h, W, G, M, lr=1.0)
        assert e.value.code == mb.MUON_ERR_OOM
        assert mb.muon_workspace_bytes(h) == 0
        torch.cuda.synchronize()
        assert all(torch.count_nonzero(x) == 0 for x in M)
        mb.muon_step(h, W, G, M, lr=1.0)
        torch.cuda.synchronize()
        mb.muon_sync(h)
        assert all(torch.equal(a, b) for a, b in zip(M, G))
        assert mb.muon_workspace_bytes(h) > held
    finally:
        mb.muon_destroy(h)


# ---------------------------------------------------------------- checkpoint / resume

def test_checkpoint_and_resume_is_bit_exact(mb):
    """The optimizer's whole state is the weights and the momentum buffers: saving them
    after two steps and resuming on a fresh handle gives the third step's bits."""
    import synth
    data = synth.make_matrix_set(1, layers=[0])
    G = [g.cuda() for g in data["G"]]
    W = [w.cuda().clone() for w in data["W"]]
    M = [m.cuda().clone() for m in data["M"]]
    h1 = mb.muon_init(0)
    try:
        for _ in range(2):
            mb.muon_step(h1, W, G, M, lr=0.02)
        torch.cuda.synchronize()
        saved = {"W": [w.cpu().clone() for w in W], "M": [m.cpu().clone() for m in M]}
        mb.muon_step(h1, W, G, M, lr=0.02)
        torch.cuda.synchronize()
        mb.muon_sync(h1)
    finally:
        mb.muon_destroy(h1)
    W2 = [w.cuda() for w in saved["W"]]
    M2 = [m.cuda() for m in saved["M"]]
    h2 = mb.muon_init(0)
    try:
        mb.muon_step(h2, W2, G, M2, lr=0.02)
        torch.cuda.synchronize()
        mb.muon_sync(h2)
    finally:
        mb.muon_destroy(h2)
    for a, b in zip(W, W2):
        assert torch.equal(a, b)
    for a, b in zip(M, M2):
        assert torch.equal(a, b)


# ---------------------------------------------------------------- MUON_LOG

def test_log_environment_variable_reports_plans_and_errors():
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    code = (
        "import torch, muon_newton_schulz_06_b200 as mb\n"
        "h = mb.muon_init(0)\n"
        "w = torch.zeros(300, 100, device='cuda'); g = torch.randn(300, 100, device='cuda')\n"
        "m = torch.zeros(300, 100, device='cuda')\n"
        "mb.muon_step(h, [w], [g], [m], lr=0.1); torch.cuda.synchronize()\n"
        "try:\n"
        "    mb.muon_step(h, [w], [g], [m], lr=float('nan'))\n"
        "except mb.MuonError:\n"
        "    pass\n"
        "mb.muon_destroy(h)\n")
    env = dict(os.environ, MUON_LOG="1", PYTHONPATH=root)
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    assert "muon: plan: 1 matrices" in r.stderr
    assert "group s=100 L=300 n=1" in r.stderr
    assert "MUON_ERR_INVALID_ARG" in r.stderr and "lr must be finite" in r.stderr
    env["MUON_LOG"] = "0"
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and "muon:" not in r.stderr


# ---------------------------------------------------------------- debug mode: workspace guard bands

def _debug_handle(mb, mode="auto"):
    import os
    old = os.environ.get("MUON_DEBUG")
    os.environ["MUON_DEBUG"] = "1"
    try:
        h = mb.muon_init(0)
    finally:
        if old is None:
            del os.environ["MUON_DEBUG"]
        else:
            os.environ["MUON_DEBUG"] = old
    mb.muon_set_launch_mode(h, mode)
    return h


@pytest.mark.parametrize("launch,mode", [("phases", "bf16"), ("persistent", "bf16"), ("auto", "fp32"),
                                         ("auto", "fp32_simt")])
def test_debug_guard_bands_stay_intact_and_results_match(mb, launch, mode):
    """A debug-mode handle (guard bands after every workspace region, checked after every
    call) gives the same bits as a plain handle, and no band changes: on a depth-8 layer
    and on ragged shapes, through muon_step and muon_newton_schulz."""
    import synth
    data = synth.make_matrix_set(1, layers=[0])
    G = [g.cuda() for g in data["G"]]
    ragged = [(300, 130), (130, 301), (7, 1003), (45, 45)]
    xs = [synth.random_matrix(r, c, seed=50 + i, device="cuda", dtype=torch.bfloat16 if mode == "bf16"
                              else torch.float32) for i, (r, c) in enumerate(ragged)]
    outs = {}
    for debug in (False, True):
        h = _debug_handle(mb, launch) if debug else mb.muon_init(0)
        try:
            if not debug:
                mb.muon_set_launch_mode(h, launch)
            W = [w.cuda().clone() for w in data["W"]]
            M = [m.cuda().clone() for m in data["M"]]
            for _ in range(2):
                mb.muon_step(h, W, G, M, lr=0.02, mode=mode)
            o = [torch.empty_like(x) for x in xs]
            mb.muon_newton_schulz(h, xs, o, mode=mode)
            torch.cuda.synchronize()
            mb.muon_sync(h)
            outs[debug] = (W, M, o, mb.muon_workspace_bytes(h))
        finally:
            mb.muon_destroy(h)
    for a, b in zip(outs[False][0] + outs[False][1] + outs[False][2], outs[True][0] + outs[True][1] + outs[True][2]):
        assert torch.equal(a, b)
    assert outs[True][3] > outs[False][3]  # the bands take room


def test_debug_guard_detects_an_overwritten_band(mb):
    """One byte of a guard band is overwritten on purpose (a memset, on the host's
    request): the next call reports MUON_ERR_CORRUPT naming the region, re-arms the
    bands, and the call after it is clean."""
    h = _debug_handle(mb)
    try:
        w = torch.zeros(256, 64, device="cuda")
        g = torch.randn(256, 64, device="cuda")
        m = torch.zeros(256, 64, device="cuda")
        mb.muon_step(h, [w], [g], [m], lr=0.1)
        mb.muon_selftest_corrupt_guard(h)
        with pytest.raises(mb.MuonError) as e:
            mb.muon_step(h, [w], [g], [m], lr=0.1)
        assert e.value.code == mb.MUON_ERR_CORRUPT
        assert "guard" in str(e.value) and "follows the tile lists" in str(e.value)
        mb.muon_step(h, [w], [g], [m], lr=0.1)
        torch.cuda.synchronize()
        mb.muon_sync(h)
    finally:
        mb.muon_destroy(h)
    h = mb.muon_init(0)
    try:
        with pytest.raises(mb.MuonError) as e:
            mb.muon_selftest_corrupt_guard(h)
        assert e.value.code == mb.MUON_ERR_INVALID_ARG
    finally:
        mb.muon_destroy(h)


def test_nvtx_ranges_leave_results_unchanged(mb):
    """MUON_NVTX=1 at handle creation wraps every call and launch in an NVTX range (seen
    by a timeline profiler when one is attached); the results keep their bits."""
    import os
    import synth
    data = synth.make_matrix_set(1, layers=[0])
    G = [g.cuda() for g in data["G"]]
    outs = []
    for nvtx in ("0", "1"):
        old = os.environ.get("MUON_NVTX")
        os.environ["MUON_NVTX"] = nvtx
        try:
            h = mb.muon_init(0)
        finally:
            if old is None:
                del os.environ["MUON_NVTX"]
            else:
                os.environ["MUON_NVTX"] = old
        try:
            W = [w.cuda().clone() for w in data["W"]]
            M = [m.cuda().clone() for m in data["M"]]
            mb.muon_profile_enable(h, True)
            mb.muon_step(h, W, G, M, lr=0.02)
            torch.cuda.synchronize()
            mb.muon_sync(h)
            prof = mb.muon_profile_read(h)
            outs.append((W, M, sum(n for _, n in prof.values())))
        finally:
            mb.muon_destroy(h)
    for a, b in zip(outs[0][0] + outs[0][1], outs[1][0] + outs[1][1]):
        assert torch.equal(a, b)
    assert outs[0][2] == outs[1][2] > 0


# ---------------------------------------------------------------- concurrency between handles

_THREADS_SCRIPT = """
import hashlib, sys, threading, torch
import muon_newton_schulz_06_b200 as mb, synth
mode = sys.argv[1]
sets = [synth.make_matrix_set(1, layers=[0], device="cuda"), synth.make_matrix_set(2, layers=[0], device="cuda")]
out = [None, None]
def run(data, i):
    stream = torch.cuda.Stream()
    h = mb.muon_init(0)
    try:
        mb.muon_set_launch_mode(h, mode)
        W = [w.clone() for w in data["W"]]
        M = [m.clone() for m in data["M"]]
        for _ in range(3):
            mb.muon_step(h, W, data["G"], M, lr=0.02, stream=stream)
        stream.synchronize()
        mb.muon_sync(h)
        d = hashlib.sha256()
        for t in W + M:
            d.update(t.cpu().contiguous().view(torch.uint8).numpy().tobytes())
        out[i] = d.hexdigest()
    finally:
        mb.muon_destroy(h)
threads = [threading.Thread(target=run, args=(data, i)) for i, data in enumerate(sets)]
for t in threads: t.start()
for t in threads: t.join(timeout=300)
print(out[0], out[1])
"""


@pytest.mark.parametrize("mode", ["phases", "persistent"])
def test_two_handles_on_two_threads(mb, mode):
    """Distinct handles may be used from distinct host threads (each on its own stream).
    In a fresh process, two threads make their first calls at the same time (the
    per-device set-up runs once, under a lock) and run three steps each; their results
    have the bits of the same steps run one after the other."""
    import hashlib
    import os
    import subprocess
    import sys
    import synth
    digests = []
    for cfg in (1, 2):
        data = synth.make_matrix_set(cfg, layers=[0], device="cuda")
        h = mb.muon_init(0)
        try:
            mb.muon_set_launch_mode(h, mode)
            W = [w.clone() for w in data["W"]]
            M = [m.clone() for m in data["M"]]
            for _ in range(3):
                mb.muon_step(h, W, data["G"], M, lr=0.02)
            torch.cuda.synchronize()
            mb.muon_sync(h)
        finally:
            mb.muon_destroy(h)
        d = hashlib.sha256()
        for t in W + M:
            d.update(t.cpu().contiguous().view(torch.uint8).numpy().tobytes())
        digests.append(d.hexdigest())
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "-c", _THREADS_SCRIPT, mode], capture_output=True, text=True, timeout=600,
                       env=dict(os.environ, PYTHONPATH=root), cwd=root)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.split() == digests


def test_init_rejects_a_device_out_of_range(mb):
    lib = mb.load_library()
    import ctypes
    out = ctypes.c_void_p()
    assert lib.muon_init(ctypes.byref(out), torch.cuda.device_count() + 3) == mb.MUON_ERR_INVALID_ARG
    assert lib.muon_init(ctypes.byref(out), -1) == mb.MUON_ERR_INVALID_ARG
    assert out.value is None
