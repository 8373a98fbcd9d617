"""Failure detection without a GPU fault.

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
