"""Per-step coefficient tables whose rows differ, and bf16 steps on row lengths that are
not a multiple of 8, through the C ABI against the CPU oracle.  Needs a B200.

The autoresearch train.py review (MuonAdamW paragraph) gives every Newton-Schulz step
its own precomputed (a, b, c) triple ("Polar Express") but prints no values.  The
tables here are invented, chosen only so that each step stays bounded on (0, 1.3]:
the quintic triple, the quintic scaled by 0.9, the classical cubic (1.5, -0.5, 0),
and two more.  Reversing the table moves O by about 20 % (relative Frobenius), far
above the bf16 bar, so a kernel that used the wrong row would fail.

Tolerances as in the other parity tests: relative Frobenius error of O per matrix
2e-2 in bf16 mode and 1e-4 in fp32 mode; momentum buffers and applied weights bit for
bit.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu

BF16_TOL = 2e-2
F32_TOL = 1e-4

Q = oracle.QUINTIC
TABLE5 = [Q, tuple(0.9 * v for v in Q), oracle.CUBIC, (2.0, -1.5, 0.5), (3.0, -3.2, 1.2)]
# an even number of rows ends in the other ping-pong buffer
TABLE6 = TABLE5 + [(1.5, -0.6, 0.1)]


@pytest.fixture(scope="module")
def mb():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import muon_newton_schulz_06_b200 as m
    from muon_newton_schulz_06_b200 import build
    build.build()
    return m


@pytest.fixture(scope="module")
def handle(mb):
    h = mb.muon_init(0)
    yield h
    mb.muon_destroy(h)


def rel(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def to64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def well_conditioned(r, c, seed, dtype):
    """U diag(s) V^T with s in [0.05, 1]: the comparison then measures the kernels, not
    the amplification of the input's rounding in tiny singular directions."""
    g = torch.Generator().manual_seed(seed)
    k = min(r, c)
    u, _ = torch.linalg.qr(torch.randn(r, k, generator=g, dtype=torch.float64))
    v, _ = torch.linalg.qr(torch.randn(c, k, generator=g, dtype=torch.float64))
    s = 0.05 + 0.95 * torch.rand(k, generator=g, dtype=torch.float64)
    return ((u * s) @ v.T).to(dtype).cuda().contiguous()


def ns_oracle(x, table, eps=1e-7):
    return oracle.newton_schulz(oracle.frobenius_normalise(to64(x), eps), table)


def ns_gpu(mb, handle, xs, mode, table):
    outs = [torch.empty_like(x) for x in xs]
    mb.muon_newton_schulz(handle, xs, outs, coeffs=table, ns_steps=len(table), mode=mode)
    torch.cuda.synchronize()
    mb.muon_sync(handle)
    return outs


SHAPES = [(300, 130), (130, 301), (256, 256), (513, 257), (64, 1000), (1000, 517)]


@pytest.mark.parametrize("table", [TABLE5, TABLE6], ids=["5rows", "6rows"])
@pytest.mark.parametrize("mode,dtype,tol", [("fp32", torch.float32, F32_TOL), ("fp32_simt", torch.float32, F32_TOL),
                                            ("bf16", torch.bfloat16, BF16_TOL)])
def test_newton_schulz_table_rows_differ(mb, handle, mode, dtype, tol, table):
    """Grouped muon_newton_schulz with a table whose rows differ, and with the same rows
    reversed: each matches the oracle run with its own table, and the two differ."""
    xs = [well_conditioned(r, c, 40 + i, dtype) for i, (r, c) in enumerate(SHAPES)]
    rev = list(reversed(table))
    outs = ns_gpu(mb, handle, xs, mode, table)
    outs_rev = ns_gpu(mb, handle, xs, mode, rev)
    for x, o, orv in zip(xs, outs, outs_rev):
        want, want_rev = ns_oracle(x, table), ns_oracle(x, rev)
        assert rel(to64(o), want) < tol, (tuple(x.shape), rel(to64(o), want))
        assert rel(to64(orv), want_rev) < tol, (tuple(x.shape), rel(to64(orv), want_rev))
        # the row order matters: the reversed table is far away from the forward one
        assert rel(want_rev, want) > 0.1
        assert rel(to64(orv), to64(o)) > 0.1, tuple(x.shape)


@pytest.mark.parametrize("mode,tol", [("fp32", F32_TOL), ("fp32_simt", F32_TOL), ("bf16", BF16_TOL)])
def test_step_table_rows_differ(mb, handle, mode, tol):
    """Two whole steps (momentum, normalisation, Newton-Schulz, update) of the tiny set
    with the 5-row table: momentum bit for bit, weight change against the oracle."""
    data = synth.make_matrix_set(0)
    W = [w.cuda() for w in data["W"]]
    G = [g.cuda() for g in data["G"]]
    M = [m.cuda() for m in data["M"]]
    ow = [to64(w) for w in data["W"]]
    om = [m.numpy() for m in data["M"]]
    for step in range(2):
        prev = [to64(w) for w in W]
        mb.muon_step(handle, W, G, M, lr=0.02, momentum=0.95, nesterov=True, coeffs=TABLE5, ns_steps=5,
                     mode=mode)
        torch.cuda.synchronize()
        mb.muon_sync(handle)
        for i, spec in enumerate(data["specs"]):
            w_new, m_new, _ = oracle.muon_step_matrix(ow[i], data["G"][i].numpy(), om[i], lr=0.02, mu=0.95,
                                                      nesterov=True, coeffs=TABLE5, eps=1e-7)
            assert np.array_equal(M[i].cpu().numpy(), m_new), (step, spec)
            err = rel(to64(W[i]) - prev[i], w_new - ow[i])
            assert err < tol, (step, spec, err)
            ow[i], om[i] = w_new, m_new


def test_step_bf16_layer_table_rows_differ(mb, handle):
    """One depth-8 layer (bf16 gradients: copy-engine momentum pass and the fused weight
    update) with the 5-row table; fp32 zero weights and lr = 1 read O back exactly."""
    data = synth.make_matrix_set(1, layers=[0])
    G = [g.cuda() for g in data["G"]]
    M = [m.cuda() for m in data["M"]]
    W = [torch.zeros(s.rows, s.cols, device="cuda") for s in data["specs"]]
    mb.muon_step(handle, W, G, M, lr=1.0, momentum=0.95, nesterov=True, coeffs=TABLE5, ns_steps=5)
    torch.cuda.synchronize()
    mb.muon_sync(handle)
    for i, spec in enumerate(data["specs"]):
        g = data["G"][i].float().numpy()
        _, m_new, o_ref = oracle.muon_step_matrix(np.zeros((spec.rows, spec.cols)), g, data["M"][i].numpy(),
                                                  lr=1.0, mu=0.95, nesterov=True, coeffs=TABLE5, eps=1e-7)
        assert np.array_equal(M[i].cpu().numpy(), m_new), spec
        o = -to64(W[i]) / oracle.update_scale(spec.rows, spec.cols)
        assert rel(o, o_ref) < BF16_TOL, (spec, rel(o, o_ref))


# ------------------------------------------------------------- bf16 steps, ragged row lengths

RAGGED = [(300, 130), (130, 301), (1000, 517), (7, 1003), (1003, 7), (257, 999), (45, 45)]


def test_bf16_step_ragged_widths(mb, handle):
    """bf16 gradients and weights whose row length is not a multiple of 8: the register
    tile momentum kernel with bf16 gradients and the element-wise branch of the fused
    weight update.

    Run 1 (float32 zero weights, lr = 1) gives W' = -fl32(f * O) with f = fl32(scale);
    O is bf16, so bf16(-W' / f) recovers it exactly (checked by recomputing W').  Run 2,
    from the same state with bf16 weights and lr = 0.02, must give
    RNE(fl32(W - fl32(f2 * O))) bit for bit.  Momentum bit for bit in both runs, O
    against the oracle within the bf16 bar."""
    gen = torch.Generator().manual_seed(77)
    G32 = [torch.randn(r, c, generator=gen) for r, c in RAGGED]
    M32 = [0.01 * torch.randn(r, c, generator=gen) for r, c in RAGGED]
    W0 = [0.02 * torch.randn(r, c, generator=gen) for r, c in RAGGED]
    G = [g.to(torch.bfloat16).cuda() for g in G32]
    # run 1: exact read-back of O
    M = [m.cuda() for m in M32]
    Wz = [torch.zeros(r, c, device="cuda") for r, c in RAGGED]
    mb.muon_step(handle, Wz, G, M, lr=1.0, momentum=0.95, nesterov=True)
    torch.cuda.synchronize()
    mb.muon_sync(handle)
    O = []
    for i, (r, c) in enumerate(RAGGED):
        g = G[i].float().cpu().numpy()
        m_ref, _ = oracle.nesterov_momentum_f32(g, M32[i].numpy(), 0.95, True)
        assert np.array_equal(M[i].cpu().numpy(), m_ref), (r, c)
        f = np.float32(1.0 * math.sqrt(max(1.0, r / c)))
        wp = Wz[i].cpu().numpy()
        o = torch.from_numpy(-wp / f).to(torch.bfloat16).float().numpy()
        assert np.array_equal(np.negative(np.multiply(f, o, dtype=np.float32)), wp), (r, c)
        O.append(o)
        _, _, o_ref = oracle.muon_step_matrix(np.zeros((r, c)), g, M32[i].numpy(), lr=1.0, mu=0.95,
                                              nesterov=True, eps=1e-7)
        assert rel(o, o_ref) < BF16_TOL, ((r, c), rel(o, o_ref))
    # run 2: bf16 weights from the same state
    M = [m.cuda() for m in M32]
    W = [w.to(torch.bfloat16).cuda() for w in W0]
    W_before = [w.float().cpu().numpy() for w in W]
    lr = 0.02
    mb.muon_step(handle, W, G, M, lr=lr, momentum=0.95, nesterov=True)
    torch.cuda.synchronize()
    mb.muon_sync(handle)
    for i, (r, c) in enumerate(RAGGED):
        # the library forms fl32(lr * scale) in double from the float32 lr it receives
        f2 = np.float32(float(np.float32(lr)) * math.sqrt(max(1.0, r / c)))
        want = np.subtract(W_before[i], np.multiply(f2, O[i], dtype=np.float32), dtype=np.float32)
        assert torch.equal(W[i].cpu(), torch.from_numpy(want).to(torch.bfloat16)), (r, c)
        m_ref, _ = oracle.nesterov_momentum_f32(G[i].float().cpu().numpy(), M32[i].numpy(), 0.95, True)
        assert np.array_equal(M[i].cpu().numpy(), m_ref), (r, c)
