"""Options of muon_step_ex on the GPU: interpolation-form momentum, weight decay and
cautious weight decay (through the C ABI, against the oracle)."""
import math

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


def expected_apply(w, o, lrs, lrwd, cautious):
    """fl32(W - fl32(lrs*O)), then fl32(. - fl32(lrwd*W)) where the decay applies."""
    w = w.astype(np.float32)
    o = o.astype(np.float32)
    wn = np.subtract(w, np.multiply(np.float32(lrs), o, dtype=np.float32), dtype=np.float32)
    if lrwd:
        agree = ((o >= 0) & (w >= 0)) | ((o <= 0) & (w <= 0))
        dec = np.subtract(wn, np.multiply(np.float32(lrwd), w, dtype=np.float32), dtype=np.float32)
        wn = np.where(agree | (not cautious), dec, wn)
    return wn


def readback_o(mb, data, **kw):
    """O of one step (fp32 zero weights, lr = 1: W' = -scale*O exactly for scale 1, 2)."""
    specs = data["specs"]
    scales = [math.sqrt(max(1.0, s.rows / s.cols)) for s in specs]
    W = [torch.zeros(s.rows, s.cols, device="cuda") for s in specs]
    M = [m.clone() for m in data["M"]]
    h = mb.muon_init(0)
    try:
        mb.muon_step_ex(h, W, data["G"], M, lr=1.0, **kw)
        torch.cuda.synchronize()
        mb.muon_sync(h)
    finally:
        mb.muon_destroy(h)
    return [(-w / sc) for w, sc in zip(W, scales)], M, scales


def test_lerp_momentum_bitexact_and_o_within_tolerance(mb):
    data = synth.make_matrix_set(1, device="cuda", layers=[0])
    O, M, _ = readback_o(mb, data, momentum=0.9, momentum_form="lerp")
    for i, spec in enumerate(data["specs"]):
        g = data["G"][i].float().cpu().numpy()
        m_ref, _ = oracle.nesterov_momentum_f32(g, data["M"][i].cpu().numpy(), 0.9, True, lerp=True)
        assert np.array_equal(M[i].cpu().numpy(), m_ref), spec
        _, _, o_ref = oracle.muon_step_matrix(np.zeros((spec.rows, spec.cols)), g, data["M"][i].cpu().numpy(),
                                              lr=1.0, mu=0.9, nesterov=True, lerp=True)
        assert rel(O[i].double().cpu().numpy(), o_ref) < BF16_TOL, spec


@pytest.mark.parametrize("cautious", [False, True])
def test_weight_decay_apply_is_exact(mb, cautious):
    data = synth.make_matrix_set(1, device="cuda", layers=[0])
    O, _, scales = readback_o(mb, data)
    W = [w.clone() for w in data["W"]]
    M = [m.clone() for m in data["M"]]
    h = mb.muon_init(0)
    lr, wd = 0.02, 0.1
    try:
        mb.muon_step_ex(h, W, data["G"], M, lr=lr, weight_decay=wd, cautious=cautious)
        torch.cuda.synchronize()
        mb.muon_sync(h)
    finally:
        mb.muon_destroy(h)
    for i in range(len(W)):
        want = expected_apply(data["W"][i].float().cpu().numpy(), O[i].cpu().numpy(), np.float32(lr * scales[i]),
                              np.float32(lr * wd), cautious)
        assert torch.equal(W[i].cpu(), torch.from_numpy(want).to(torch.bfloat16)), i


def test_cautious_decay_matches_oracle_in_fp32_mode(mb):
    """fp32 weights and fp32 mode (separate apply pass): the weight change matches the
    oracle's W - lr*scale*O - lr*wd*mask*W within the fp32 tolerance."""
    data = synth.make_matrix_set(0)
    W = [torch.randn(w.shape, generator=torch.Generator().manual_seed(3)).cuda() for w in data["W"]]
    W0 = [w.clone() for w in W]
    G = [g.cuda() for g in data["G"]]
    M = [m.cuda() for m in data["M"]]
    h = mb.muon_init(0)
    try:
        mb.muon_step_ex(h, W, G, M, lr=0.05, weight_decay=0.2, cautious=True, mode="fp32")
        torch.cuda.synchronize()
        mb.muon_sync(h)
    finally:
        mb.muon_destroy(h)
    for i, spec in enumerate(data["specs"]):
        w0 = W0[i].double().cpu().numpy()
        w_ref, _, _ = oracle.muon_step_matrix(w0, data["G"][i].numpy(), data["M"][i].numpy(), lr=0.05, mu=0.95,
                                              weight_decay=0.2, cautious=True)
        err = rel(W[i].double().cpu().numpy() - w0, w_ref - w0)
        assert err < 1e-4, (spec, err)


def test_fused_and_separate_apply_agree_with_decay(mb):
    n = 800  # more than one fused table (768 matrices) holds
    shapes = [(16, 8) if i % 2 else (8, 24) for i in range(n)]
    G = [synth.random_matrix(r, c, seed=3000 + i, device="cuda", dtype=torch.bfloat16) for i, (r, c) in
         enumerate(shapes)]
    W0 = [synth.random_matrix(r, c, seed=7000 + i, device="cuda", dtype=torch.bfloat16) for i, (r, c) in
          enumerate(shapes)]
    kw = dict(lr=0.05, weight_decay=0.3, cautious=True, momentum_form="lerp")
    W1, M1 = [w.clone() for w in W0], [torch.zeros(r, c, device="cuda") for r, c in shapes]
    W2, M2 = [w.clone() for w in W0], [torch.zeros(r, c, device="cuda") for r, c in shapes]
    h1, h2 = mb.muon_init(0), mb.muon_init(0)
    try:
        mb.muon_step_ex(h1, W1, G, M1, **kw)
        mb.muon_step_ex(h2, W2[:400], G[:400], M2[:400], **kw)
        mb.muon_step_ex(h2, W2[400:], G[400:], M2[400:], **kw)
        torch.cuda.synchronize()
    finally:
        mb.muon_destroy(h1)
        mb.muon_destroy(h2)
    for a, b in zip(W1, W2):
        assert torch.equal(a, b)
    for a, b in zip(M1, M2):
        assert torch.equal(a, b)


def test_bad_options_are_rejected(mb):
    w = torch.zeros(8, 8, device="cuda")
    h = mb.muon_init(0)
    try:
        with pytest.raises(mb.MuonError):
            mb.muon_step_ex(h, [w], [w.clone()], [w.clone()], lr=0.1, weight_decay=-1.0)
        with pytest.raises(ValueError):
            mb.muon_step_ex(h, [w], [w.clone()], [w.clone()], lr=0.1, momentum_form="adam")
    finally:
        mb.muon_destroy(h)


# ---------------------------------------------------------------- NorMuon

def normuon_run(mb, data, states, steps, **kw):
    """`steps` NorMuon steps with fp32 zero weights reset before each step and lr = 1, so
    that W' = -scale*O'' exactly (scale in {1, 2}); returns O'' of the last step."""
    specs = data["specs"]
    scales = [math.sqrt(max(1.0, s.rows / s.cols)) for s in specs]
    M = [m.clone() for m in data["M"]]
    h = mb.muon_init(0)
    try:
        for _ in range(steps):
            W = [torch.zeros(s.rows, s.cols, device="cuda") for s in specs]
            mb.muon_step_ex(h, W, data["G"], M, lr=1.0, normuon_state=states, **kw)
        torch.cuda.synchronize()
        mb.muon_sync(h)
    finally:
        mb.muon_destroy(h)
    return [(-w / sc) for w, sc in zip(W, scales)], M


@pytest.mark.parametrize("mode,tol", [("bf16", BF16_TOL), ("fp32", 1e-4), ("fp32_simt", 1e-4)])
def test_normuon_two_steps_vs_oracle(mb, mode, tol):
    if mode == "bf16":
        data = synth.make_matrix_set(1, device="cuda", layers=[0])
    else:
        d0 = synth.make_matrix_set(0)
        data = {k: ([x.cuda() for x in v] if k in ("W", "G", "M") else v) for k, v in d0.items()}
    states = [torch.zeros(min(s.rows, s.cols), device="cuda") for s in data["specs"]]
    O2, M = normuon_run(mb, data, states, 2, mode=mode, normuon_beta2=0.9, normuon_eps=1e-8)
    for i, spec in enumerate(data["specs"]):
        g = data["G"][i].float().cpu().numpy()
        m = data["M"][i].cpu().numpy()
        v = np.zeros(min(spec.rows, spec.cols))
        for _ in range(2):
            _, m, o2, v = oracle.muon_step_matrix(np.zeros((spec.rows, spec.cols)), g, m, lr=1.0, mu=0.95,
                                                  normuon_state=v, normuon_beta2=0.9, normuon_eps=1e-8)
        err = rel(O2[i].double().cpu().numpy(), o2)
        assert err < tol, (spec, err)
        vt = states[i].double().cpu().numpy()
        assert rel(vt, v) < 2 * tol + 1e-6, (spec, rel(vt, v))
