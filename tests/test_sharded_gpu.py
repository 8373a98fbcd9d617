"""The matrix-sharded step (muon_newton_schulz_06_b200.sharded) with the CUDA kernels, at
world size 1 (one GPU per run here; the partition and the all-gather are covered by
the two-rank gloo test).  Every matrix against the oracle, and the same bits as the
replicated muon_step.  Needs a B200.
"""
import numpy as np
import pytest
import torch

import oracle
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
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def test_sharded_step_world_one_against_the_oracle(mb):
    """Float32 zero weights in the flat buffer and lr = 1: W' = -fl32(scale * O), so O of
    every matrix is compared with the oracle; momentum bit for bit."""
    from muon_newton_schulz_06_b200 import sharded
    data = synth.make_matrix_set(1, layers=[0, 1])
    params = [torch.zeros(s.rows, s.cols, device="cuda") for s in data["specs"]]
    G = [g.cuda() for g in data["G"]]
    sm = sharded.ShardedMuon(params, device="cuda")
    try:
        assert sm.owned() == list(range(len(params)))
        # the flat buffer's views start at 16-byte boundaries, as the library requires
        assert all(p.data_ptr() % 16 == 0 for p in sm.params)
        sm.step(G, lr=1.0, momentum=0.95)
        torch.cuda.synchronize()
        for i, spec in enumerate(data["specs"]):
            g = data["G"][i].float().numpy()
            _, m_new, o_ref = oracle.muon_step_matrix(np.zeros((spec.rows, spec.cols)), g,
                                                      np.zeros((spec.rows, spec.cols), np.float32), lr=1.0,
                                                      mu=0.95, nesterov=True, eps=1e-7)
            assert np.array_equal(sm.moms[i].cpu().numpy(), m_new), spec
            o = -sm.params[i].double().cpu().numpy() / oracle.update_scale(spec.rows, spec.cols)
            assert rel(o, o_ref) < BF16_TOL, (spec, rel(o, o_ref))
    finally:
        sm.close()


def test_sharded_step_world_one_matches_the_replicated_step(mb):
    """bf16 weights, three steps: the sharded object's views and momentum give the same
    bits as muon_step on separately allocated tensors."""
    from muon_newton_schulz_06_b200 import sharded
    data = synth.make_matrix_set(1, layers=[0])
    G = [g.cuda() for g in data["G"]]
    W_ref = [w.cuda().clone() for w in data["W"]]
    M_ref = [torch.zeros(s.rows, s.cols, device="cuda") for s in data["specs"]]
    sm = sharded.ShardedMuon([w.clone() for w in W_ref], device="cuda")
    h = mb.muon_init(0)
    try:
        for _ in range(3):
            sm.step(G, lr=0.02, momentum=0.95)
            mb.muon_step(h, W_ref, G, M_ref, lr=0.02, momentum=0.95)
        torch.cuda.synchronize()
        mb.muon_sync(h)
        for i in range(len(G)):
            assert torch.equal(sm.params[i], W_ref[i]), i
            assert torch.equal(sm.moms[i], M_ref[i]), i
    finally:
        mb.muon_destroy(h)
        sm.close()
