"""CUDA path vs the CPU oracle, through the C ABI (the Python binding only marshals
arguments).  Needs a B200.

Tolerances (relative Frobenius error of the orthogonalised update per matrix):
bf16 mode 2e-2, fp32 validation mode 1e-4; momentum buffers bit-exact.
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


def ns_gpu(mb, handle, xs, mode, coeffs=None, ns_steps=5, eps=1e-7):
    outs = [torch.empty_like(x) for x in xs]
    mb.muon_newton_schulz(handle, xs, outs, coeffs=coeffs, ns_steps=ns_steps, eps=eps, mode=mode)
    torch.cuda.synchronize()
    mb.muon_sync(handle)
    return outs


def ns_oracle(x, coeffs, eps=1e-7):
    return oracle.newton_schulz(oracle.frobenius_normalise(to64(x), eps), coeffs)


EDGE_SHAPES = [(1, 9), (9, 1), (1, 1), (63, 130), (130, 63), (64, 64), (65, 257), (257, 65), (129, 129),
               (127, 300), (300, 255), (96, 96), (256, 32), (384, 1000)]


# ------------------------------------------------------------- single Newton-Schulz step algebra

# One step in fp32: the CUDA-core mode rounds each product to 24 bits, the 3xTF32 mode keeps
# about 22 bits of each operand (hi + lo), hence 4x the CUDA-core tolerance for it.
@pytest.mark.parametrize("mode,dtype,tol", [("fp32", torch.float32, 4e-5), ("fp32_simt", torch.float32, 1e-5),
                                            ("bf16", torch.bfloat16, 1.5e-2)])
@pytest.mark.parametrize("abc", [(1.0, 0.0, 0.0), (0.0, 1.0, 0.0), (0.0, 0.0, 1.0), (0.5, -1.0, 2.0)])
def test_one_step_each_product(mb, handle, mode, dtype, tol, abc):
    """(1,0,0) passes X through; (0,1,0) is X X^T X (Gram + update); (0,0,1) is (X X^T)^2 X
    (Gram + polynomial + update)."""
    shapes = [(200, 136), (136, 200), (256, 512), (130, 130), (40, 700)]
    xs = [synth.random_matrix(r, c, seed=10 + i, device="cuda", dtype=dtype) for i, (r, c) in enumerate(shapes)]
    outs = ns_gpu(mb, handle, xs, mode, coeffs=[abc], ns_steps=1)
    for x, o in zip(xs, outs):
        want = ns_oracle(x, [abc])
        assert rel(to64(o), want) < tol, (x.shape, abc, rel(to64(o), want))


# ------------------------------------------------------------- full Newton-Schulz

@pytest.mark.parametrize("mode,dtype,tol", [("fp32", torch.float32, F32_TOL), ("fp32_simt", torch.float32, F32_TOL),
                                            ("bf16", torch.bfloat16, BF16_TOL)])
def test_newton_schulz_edge_shapes(mb, handle, mode, dtype, tol):
    """Shapes around the 64 / 128 / 256 tile edges, tall, wide, square and degenerate,
    all in one grouped call.  Inputs are well conditioned (singular values in
    [0.05, 1]) so the comparison measures the kernels, not the input rounding."""
    xs = []
    for i, (r, c) in enumerate(EDGE_SHAPES):
        g = torch.Generator().manual_seed(500 + i)
        k = min(r, c)
        u, _ = torch.linalg.qr(torch.randn(r, k, generator=g, dtype=torch.float64))
        v, _ = torch.linalg.qr(torch.randn(c, k, generator=g, dtype=torch.float64))
        s = 0.05 + 0.95 * torch.rand(k, generator=g, dtype=torch.float64)
        xs.append(((u * s) @ v.T).to(dtype).cuda().contiguous())
    outs = ns_gpu(mb, handle, xs, mode)
    for x, o in zip(xs, outs):
        want = ns_oracle(x, [oracle.QUINTIC] * 5)
        err = rel(to64(o), want)
        assert err < tol, (tuple(x.shape), err)


def test_newton_schulz_gaussian_bf16(mb, handle):
    """Gaussian inputs (tiny singular values included) at the 2e-2 bar."""
    shapes = [(512, 512), (2048, 512), (512, 2048), (768, 768)]
    xs = [synth.random_matrix(r, c, seed=70 + i, device="cuda", dtype=torch.bfloat16) for i, (r, c) in
          enumerate(shapes)]
    outs = ns_gpu(mb, handle, xs, "bf16")
    for x, o in zip(xs, outs):
        err = rel(to64(o), ns_oracle(x, [oracle.QUINTIC] * 5))
        assert err < BF16_TOL, (tuple(x.shape), err)


def test_transpose_equivariance_gpu(mb, handle):
    x = synth.random_matrix(300, 130, seed=3, device="cuda", dtype=torch.bfloat16)
    xt = x.T.contiguous()
    o, ot = ns_gpu(mb, handle, [x, xt], "bf16")
    # both orientations run the same kernels on the same wide-orientation data; only the
    # norm's summation order differs
    assert rel(to64(o).T, to64(ot)) < 1e-2


# ------------------------------------------------------------- whole step, tiny set

@pytest.mark.parametrize("mode,tol", [("fp32", F32_TOL), ("fp32_simt", F32_TOL), ("bf16", BF16_TOL)])
def test_tiny_set_three_steps(mb, handle, mode, tol):
    """Tiny set: 128x64, 64x128, 96x96, 256x32, fp32, N(0,1) grads, M = W = 0, mu 0.95
    Nesterov, lr 0.02, quintic x5, eps 1e-7, three steps with the same gradient."""
    data = synth.make_matrix_set(0)
    W = [w.cuda() for w in data["W"]]
    G = [g.cuda() for g in data["G"]]
    M = [m.cuda() for m in data["M"]]
    ow = [to64(w) for w in data["W"]]
    om = [m.numpy() for m in data["M"]]
    for step in range(3):
        prev = [to64(w) for w in W]
        mb.muon_step(handle, W, G, M, lr=0.02, momentum=0.95, nesterov=True, mode=mode)
        torch.cuda.synchronize()
        mb.muon_sync(handle)
        for i, spec in enumerate(data["specs"]):
            w_new, m_new, o = oracle.muon_step_matrix(ow[i], data["G"][i].numpy(), om[i], lr=0.02, mu=0.95,
                                                      nesterov=True, eps=1e-7)
            # momentum: bit-exact
            assert np.array_equal(M[i].cpu().numpy(), m_new), (step, spec)
            # update: W_new - W_prev vs -lr*scale*O
            dw = to64(W[i]) - prev[i]
            err = rel(dw, w_new - ow[i])
            assert err < tol, (step, spec, err)
            ow[i], om[i] = w_new, m_new


# ------------------------------------------------------------- apply exactness and momentum (bf16 sets)

def test_apply_exact_and_momentum_bitexact(mb, handle):
    """With fp32 zero weights and lr = 1, W' = -fl32(scale*O) is exact for scale in {1, 2}, so
    O is read back; a second run from the same state with bf16 weights must give
    RNE(fl32(W - fl32(lr*scale)*O)) bit for bit.  Momentum vs NumPy float32, bit for bit."""
    data = synth.make_matrix_set(1, layers=[0, 1])
    G = [g.cuda() for g in data["G"]]
    M0 = [m.cuda() for m in data["M"]]
    scales = [math.sqrt(max(1.0, s.rows / s.cols)) for s in data["specs"]]
    assert set(scales) <= {1.0, 2.0}
    # run 1: fp32 zeros, lr = 1
    M = [m.clone() for m in M0]
    Wz = [torch.zeros(s.rows, s.cols, device="cuda") for s in data["specs"]]
    mb.muon_step(handle, Wz, G, M, lr=1.0, momentum=0.95, nesterov=True)
    torch.cuda.synchronize()
    mb.muon_sync(handle)
    O = [(-w / sc) for w, sc in zip(Wz, scales)]
    for i in range(len(G)):
        m_ref, _ = oracle.nesterov_momentum_f32(data["G"][i].float().numpy(), data["M"][i].numpy(), 0.95, True)
        assert np.array_equal(M[i].cpu().numpy(), m_ref)
    # run 2: same state, bf16 weights
    M = [m.clone() for m in M0]
    W = [w.cuda().clone() for w in data["W"]]
    W_before = [w.clone() for w in W]
    lr = 0.02
    mb.muon_step(handle, W, G, M, lr=lr, momentum=0.95, nesterov=True)
    torch.cuda.synchronize()
    for i in range(len(G)):
        lrs = np.float32(lr * scales[i])
        o = O[i].cpu().numpy().astype(np.float32)
        want = np.subtract(W_before[i].float().cpu().numpy(), np.multiply(lrs, o, dtype=np.float32),
                           dtype=np.float32)
        want_bf16 = torch.from_numpy(want).to(torch.bfloat16)
        assert torch.equal(W[i].cpu(), want_bf16), i
    # and O itself is the oracle's within the bf16 bar
    for i in range(len(G)):
        _, _, o_ref = oracle.muon_step_matrix(np.zeros((data["specs"][i].rows, data["specs"][i].cols)),
                                              data["G"][i].float().numpy(), data["M"][i].numpy(), lr=1.0,
                                              mu=0.95, nesterov=True, eps=1e-7)
        assert rel(to64(O[i]), o_ref) < BF16_TOL, i


@pytest.mark.parametrize("lerp", [False, True])
def test_copy_engine_momentum_pass_edges(mb, handle, lerp):
    """bf16 momentum pass through the copy engine at its edges: tall matrices with ragged
    64 x 64 tiles (tensor-map path: zero fill on load, clipping on store, transposed
    workspace), wide matrices whose element count leaves a partial last 4096-element
    unit (bulk-copy path), and one matrix per path in a single grouped call.  Momentum
    bit-exact; O within the bf16 bar."""
    shapes = [(1000, 136), (700, 8), (130, 72), (2100, 520), (5, 1000), (100, 808), (3, 8), (40, 4104)]
    gen = torch.Generator().manual_seed(11)
    G32 = [torch.randn(r, c, generator=gen) for r, c in shapes]
    M32 = [0.01 * torch.randn(r, c, generator=gen) for r, c in shapes]
    G = [g.to(torch.bfloat16).cuda() for g in G32]
    M = [m.cuda() for m in M32]
    W = [torch.zeros(r, c, device="cuda") for r, c in shapes]
    kw = {"momentum_form": "lerp"} if lerp else {}
    mb.muon_step_ex(handle, W, G, M, lr=1.0, momentum=0.95, nesterov=True, **kw)
    torch.cuda.synchronize()
    mb.muon_sync(handle)
    for i, (r, c) in enumerate(shapes):
        g = G[i].float().cpu().numpy()
        m_ref, _ = oracle.nesterov_momentum_f32(g, M32[i].numpy(), 0.95, True, lerp=lerp)
        assert np.array_equal(M[i].cpu().numpy(), m_ref), (r, c)
        _, _, o_ref = oracle.muon_step_matrix(np.zeros((r, c)), g, M32[i].numpy(), lr=1.0, mu=0.95,
                                              nesterov=True, eps=1e-7, lerp=lerp)
        o = -to64(W[i]) / oracle.update_scale(r, c)
        assert rel(o, o_ref) < BF16_TOL, ((r, c), rel(o, o_ref))


def test_grouped_step_matches_single_matrix_calls(mb, handle):
    """Packing many shapes into one grouped launch gives the same bits as one call per matrix."""
    data = synth.make_matrix_set(1, layers=[0])
    G = [g.cuda() for g in data["G"]]
    W1 = [w.cuda().clone() for w in data["W"]]
    M1 = [m.cuda().clone() for m in data["M"]]
    W2 = [w.clone() for w in W1]
    M2 = [m.clone() for m in M1]
    mb.muon_step(handle, W1, G, M1, lr=0.02)
    h2 = mb.muon_init(0)
    try:
        for i in range(len(G)):
            mb.muon_step(h2, [W2[i]], [G[i]], [M2[i]], lr=0.02)
        torch.cuda.synchronize()
    finally:
        mb.muon_destroy(h2)
    for a, b in zip(W1, W2):
        assert torch.equal(a, b)
    for a, b in zip(M1, M2):
        assert torch.equal(a, b)


def test_fused_and_separate_apply_agree(mb, handle):
    """More matrices than one fused weight-update table holds (768) take the separate
    apply pass; the same matrices in two smaller calls take the fused epilogue.  Both
    must give the same bits."""
    n = 1100
    shapes = [(16, 8) if i % 2 else (8, 24) for i in range(n)]
    G = [synth.random_matrix(r, c, seed=2000 + i, device="cuda", dtype=torch.bfloat16) for i, (r, c) in
         enumerate(shapes)]
    W0 = [synth.random_matrix(r, c, seed=9000 + i, device="cuda", dtype=torch.bfloat16) for i, (r, c) in
          enumerate(shapes)]
    W1 = [w.clone() for w in W0]
    M1 = [torch.zeros(r, c, device="cuda") for r, c in shapes]
    mb.muon_step(handle, W1, G, M1, lr=0.05)
    W2 = [w.clone() for w in W0]
    M2 = [torch.zeros(r, c, device="cuda") for r, c in shapes]
    h2 = mb.muon_init(0)
    try:
        half = n // 2
        mb.muon_step(h2, W2[:half], G[:half], M2[:half], lr=0.05)
        mb.muon_step(h2, W2[half:], G[half:], M2[half:], lr=0.05)
        torch.cuda.synchronize()
    finally:
        mb.muon_destroy(h2)
    torch.cuda.synchronize()
    for a, b in zip(W1, W2):
        assert torch.equal(a, b)
    for a, b in zip(M1, M2):
        assert torch.equal(a, b)


def test_zero_gradient_leaves_weights(mb, handle):
    W = [torch.randn(256, 128, device="cuda").to(torch.bfloat16), torch.randn(64, 300, device="cuda")]
    G = [torch.zeros_like(w) for w in W]
    M = [torch.zeros(w.shape, device="cuda") for w in W]
    before = [w.clone() for w in W]
    mb.muon_step(handle, W, G, M, lr=0.1)
    torch.cuda.synchronize()
    mb.muon_sync(handle)
    for a, b in zip(W, before):
        assert torch.equal(a, b)
    for m in M:
        assert torch.count_nonzero(m) == 0


def test_nesterov_off(mb, handle):
    data = synth.make_matrix_set(0)
    W = [torch.zeros_like(w).cuda() for w in data["W"]]
    G = [g.cuda() for g in data["G"]]
    M = [(0.5 * g).cuda() for g in data["G"]]
    mb.muon_step(handle, W, G, M, lr=1.0, momentum=0.9, nesterov=False, mode="fp32")
    torch.cuda.synchronize()
    for i, spec in enumerate(data["specs"]):
        w_new, _, _ = oracle.muon_step_matrix(np.zeros((spec.rows, spec.cols)), data["G"][i].numpy(),
                                              (0.5 * data["G"][i]).numpy(), lr=1.0, mu=0.9, nesterov=False)
        assert rel(to64(W[i]), w_new) < F32_TOL


# ------------------------------------------------------------- argument errors (host-side)

def test_invalid_arguments(mb, handle):
    w = torch.zeros(64, 64, device="cuda")
    g = torch.zeros(64, 64, device="cuda")
    m = torch.zeros(64, 64, device="cuda")
    with pytest.raises(mb.MuonError) as e:
        mb.muon_step(handle, [w], [g], [m], lr=float("nan"))
    assert e.value.code == mb.MUON_ERR_INVALID_ARG
    with pytest.raises(mb.MuonError):
        mb.muon_step(handle, [w], [g], [m], lr=0.1, momentum=1.0)
    with pytest.raises(mb.MuonError):
        mb.muon_step(handle, [w], [g], [m], lr=0.1, ns_steps=0)
    with pytest.raises(mb.MuonError):
        mb.muon_step(handle, [w], [w], [m], lr=0.1)  # param aliases grad
    with pytest.raises(mb.MuonError):
        mb.muon_step(handle, [w, w], [g, g], [m, m], lr=0.1)
    mis = torch.zeros(64 * 64 + 1, device="cuda")[1:].view(64, 64)
    with pytest.raises(mb.MuonError) as e:
        mb.muon_step(handle, [mis], [g], [m], lr=0.1)
    assert e.value.code == mb.MUON_ERR_INVALID_ARG
    # nothing was enqueued by the failed calls and the handle still works
    mb.muon_step(handle, [w], [g], [m], lr=0.1)
    torch.cuda.synchronize()
    mb.muon_sync(handle)


def test_empty_call_is_a_no_op(mb, handle):
    mb.muon_step(handle, [], [], [], lr=0.1)
    mb.muon_newton_schulz(handle, [], [])


def test_cuda_graph_capture_replays_bit_exact(mb, handle):
    """After a first call has built the plan, a muon_step captured in a CUDA graph and
    replayed gives the same bits as the same number of eager calls."""
    data = synth.make_matrix_set(1, layers=[0])
    G = [g.cuda() for g in data["G"]]
    W_e = [w.cuda().clone() for w in data["W"]]
    M_e = [m.cuda().clone() for m in data["M"]]
    W_g = [w.clone() for w in W_e]
    M_g = [m.clone() for m in M_e]
    h2 = mb.muon_init(0)
    try:
        s = torch.cuda.Stream()
        with torch.cuda.stream(s):
            # plan + workspace are built outside capture, on a throw-away copy
            mb.muon_step(h2, [w.clone() for w in W_g], G, [m.clone() for m in M_g], lr=0.02, stream=s)
        s.synchronize()
        mb.muon_sync(h2)  # no status copy pending while capturing
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=s):
            mb.muon_step(h2, W_g, G, M_g, lr=0.02, stream=s)
        for _ in range(3):
            graph.replay()
        torch.cuda.synchronize()
        for _ in range(3):
            mb.muon_step(handle, W_e, G, M_e, lr=0.02)
        torch.cuda.synchronize()
        mb.muon_sync(h2)
    finally:
        mb.muon_destroy(h2)
    for a, b in zip(W_e, W_g):
        assert torch.equal(a, b)
    for a, b in zip(M_e, M_g):
        assert torch.equal(a, b)


@pytest.mark.parametrize("mode,dtype,tol", [("fp32", torch.float32, F32_TOL), ("fp32_simt", torch.float32, F32_TOL),
                                            ("bf16", torch.bfloat16, BF16_TOL)])
def test_random_shapes_grouped(mb, handle, mode, dtype, tol):
    """30 seeded random shapes (1..700 x 1..700, many sharing a group) in one call."""
    rng = np.random.default_rng(2024)
    shapes = [(int(rng.integers(1, 701)), int(rng.integers(1, 701))) for _ in range(24)]
    shapes += [shapes[0], shapes[1], (shapes[2][1], shapes[2][0]), (256, 256), (512, 128), (128, 512)]
    xs = []
    for i, (r, c) in enumerate(shapes):
        g = torch.Generator().manual_seed(900 + i)
        k = min(r, c)
        u, _ = torch.linalg.qr(torch.randn(r, k, generator=g, dtype=torch.float64))
        v, _ = torch.linalg.qr(torch.randn(c, k, generator=g, dtype=torch.float64))
        sv = 0.05 + 0.95 * torch.rand(k, generator=g, dtype=torch.float64)
        xs.append(((u * sv) @ v.T).to(dtype).cuda().contiguous())
    outs = ns_gpu(mb, handle, xs, mode)
    for x, o in zip(xs, outs):
        err = rel(to64(o), ns_oracle(x, [oracle.QUINTIC] * 5))
        assert err < tol, (tuple(x.shape), err)


# ------------------------------------------------------------- the two fp32 validation modes

def test_fp32_modes_agree_and_bound_the_error(mb, handle):
    """3xTF32 tensor-core mode and the CUDA-core fp32 mode on the same inputs: both within
    the 1e-4 bar of the float64 oracle, and within 5e-5 of each other (the split keeps
    about 22 significant bits per operand, the CUDA-core mode 24; five steps amplify the
    difference)."""
    shapes = [(512, 512), (2048, 512), (512, 2048), (300, 130), (33, 700)]
    xs = [synth.random_matrix(r, c, seed=90 + i, device="cuda", dtype=torch.float32) for i, (r, c) in
          enumerate(shapes)]
    tc = ns_gpu(mb, handle, xs, "fp32")
    simt = ns_gpu(mb, handle, xs, "fp32_simt")
    for x, a, b in zip(xs, tc, simt):
        want = ns_oracle(x, [oracle.QUINTIC] * 5)
        assert rel(to64(a), want) < F32_TOL, (tuple(x.shape), rel(to64(a), want))
        assert rel(to64(b), want) < F32_TOL, (tuple(x.shape), rel(to64(b), want))
        assert rel(to64(a), to64(b)) < 5e-5, (tuple(x.shape), rel(to64(a), to64(b)))


# ------------------------------------------------------------- extremes

@pytest.mark.parametrize("mode,dtype,tol", [("bf16", torch.bfloat16, BF16_TOL), ("fp32", torch.float32, F32_TOL)])
def test_extreme_aspect_ratios(mb, handle, mode, dtype, tol):
    """One row or one column of 16384, and 2 x 8000 / 8000 x 3 (s = 1..3, contractions of
    up to 256 k-blocks), in one grouped call."""
    shapes = [(1, 16384), (16384, 1), (2, 8000), (8000, 3)]
    xs = [synth.random_matrix(r, c, seed=600 + i, device="cuda", dtype=dtype) for i, (r, c) in enumerate(shapes)]
    outs = ns_gpu(mb, handle, xs, mode)
    for x, o in zip(xs, outs):
        err = rel(to64(o), ns_oracle(x, [oracle.QUINTIC] * 5))
        assert err < tol, (tuple(x.shape), err)


@pytest.mark.parametrize("mode,dtype,tol", [("bf16", torch.bfloat16, BF16_TOL), ("fp32", torch.float32, F32_TOL),
                                            ("fp32_simt", torch.float32, F32_TOL)])
def test_sixteen_steps(mb, handle, mode, dtype, tol):
    """The most steps a call takes (16), quintic rows then cubic rows, per-phase launches
    and both fp32 modes."""
    table = [oracle.QUINTIC] * 8 + [oracle.CUBIC] * 8
    shapes = [(300, 130), (256, 256), (130, 700)]
    xs = [synth.random_matrix(r, c, seed=700 + i, device="cuda", dtype=dtype) for i, (r, c) in enumerate(shapes)]
    h = mb.muon_init(0)
    try:
        mb.muon_set_launch_mode(h, "phases")
        outs = [torch.empty_like(x) for x in xs]
        mb.muon_newton_schulz(h, xs, outs, coeffs=table, ns_steps=16, mode=mode)
        torch.cuda.synchronize()
        mb.muon_sync(h)
    finally:
        mb.muon_destroy(h)
    for x, o in zip(xs, outs):
        err = rel(to64(o), ns_oracle(x, table))
        assert err < tol, (tuple(x.shape), err)


@pytest.mark.parametrize("mode", ["bf16", "fp32"])
def test_nan_gradient_stays_in_its_matrix(mb, mode):
    """A NaN in one gradient makes that matrix's update NaN (nothing checks for it on the
    hot path) and leaves the other matrices of the same grouped call, and the next call,
    exactly as without it."""
    shapes = [(256, 128), (256, 128), (128, 300)]
    G = [synth.random_matrix(r, c, seed=800 + i, device="cuda") for i, (r, c) in enumerate(shapes)]
    Gn = [g.clone() for g in G]
    Gn[0][3, 5] = float("nan")
    res = []
    for grads in (G, Gn, G):
        W = [torch.zeros(r, c, device="cuda") for r, c in shapes]
        M = [torch.zeros(r, c, device="cuda") for r, c in shapes]
        h = mb.muon_init(0)
        try:
            mb.muon_step(h, W, grads, M, lr=0.1, mode=mode)
            torch.cuda.synchronize()
            mb.muon_sync(h)
        finally:
            mb.muon_destroy(h)
        res.append(W)
    assert torch.isnan(res[1][0]).all()
    for i in (1, 2):
        assert torch.equal(res[0][i], res[1][i])
    for a, b in zip(res[0], res[2]):
        assert torch.equal(a, b)


def test_fp32_validation_mode_uses_cuda_cores_for_long_contractions(mb, handle):
    """The 3xTF32 form's accumulation error grows with the contraction length, so the fp32
    validation mode runs a call whose longest side exceeds 8192 on CUDA cores: the bits of
    MUON_MODE_FP32_SIMT there, the tensor-core form at 8192; both within 1e-4."""
    x_long = synth.random_matrix(64, 9000, seed=901, device="cuda")
    x_edge = synth.random_matrix(64, 8192, seed=902, device="cuda")
    (a,) = ns_gpu(mb, handle, [x_long], "fp32")
    (b,) = ns_gpu(mb, handle, [x_long], "fp32_simt")
    assert torch.equal(a, b)
    (c,) = ns_gpu(mb, handle, [x_edge], "fp32")
    (d,) = ns_gpu(mb, handle, [x_edge], "fp32_simt")
    assert not torch.equal(c, d)  # different arithmetic: the tensor-core form ran
    for x, o in ((x_long, a), (x_edge, c), (x_edge, d)):
        assert rel(to64(o), ns_oracle(x, [oracle.QUINTIC] * 5)) < F32_TOL


def test_host_memory_is_rejected_by_the_c_abi(mb):
    """Through the C ABI directly (the binding already refuses CPU tensors): a gradient in
    pinned or pageable host memory, or an output in host memory, is an argument error
    returned before anything is enqueued, and the handle keeps working."""
    import ctypes
    lib = mb.load_library()
    h = mb.muon_init(0)
    try:
        w = torch.zeros(64, 32, device="cuda")
        g = torch.randn(64, 32, device="cuda")
        m = torch.zeros(64, 32, device="cuda")
        stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
        for host in (torch.randn(64, 32).pin_memory(), torch.randn(64, 32)):
            arr = (mb.muon_matrix * 1)()
            arr[0] = mb.muon_matrix(w.data_ptr(), host.data_ptr(), m.data_ptr(), 64, 32, mb.MUON_F32, mb.MUON_F32)
            code = lib.muon_step(h, arr, 1, 0.1, 0.95, 1, None, 5, ctypes.c_float(1e-7), 0, stream)
            assert code == mb.MUON_ERR_INVALID_ARG
            assert b"not device memory" in lib.muon_last_error(h)
        out_host = torch.empty(64, 32).pin_memory()
        xin = (ctypes.c_void_p * 1)(g.data_ptr())
        xout = (ctypes.c_void_p * 1)(out_host.data_ptr())
        rows = (ctypes.c_int64 * 1)(64)
        cols = (ctypes.c_int64 * 1)(32)
        assert lib.muon_newton_schulz(h, xin, xout, rows, cols, 1, mb.MUON_F32, None, 5, ctypes.c_float(1e-7), 0,
                                      stream) == mb.MUON_ERR_INVALID_ARG
        torch.cuda.synchronize()
        assert torch.count_nonzero(m) == 0 and torch.count_nonzero(w) == 0
        mb.muon_step(h, [w], [g], [m], lr=0.1)
        torch.cuda.synchronize()
        mb.muon_sync(h)
        assert torch.equal(m, g)
    finally:
        mb.muon_destroy(h)
