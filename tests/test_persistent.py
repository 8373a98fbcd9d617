"""The persistent Newton-Schulz launch (MUON_LAUNCH_PERSISTENT) against the per-phase
launches and the oracle, through the C ABI.  Needs a B200.

Both forms compute every 256 x 256 tile with the same products in the same order and
the same epilogue arithmetic, so every comparison between them is bit for bit; the
oracle comparisons use the bf16 bar (2e-2 relative Frobenius error per matrix).
"""
import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu

BF16_TOL = 2e-2
Q = oracle.QUINTIC
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


def handle(mb, mode):
    h = mb.muon_init(0)
    mb.muon_set_launch_mode(h, mode)
    return h


def run_steps(mb, mode, W, G, M, steps=1, ex=False, **kw):
    h = handle(mb, mode)
    try:
        for _ in range(steps):
            if ex:
                mb.muon_step_ex(h, W, G, M, **kw)
            else:
                mb.muon_step(h, W, G, M, **kw)
        torch.cuda.synchronize()
        mb.muon_sync(h)
        return mb.muon_last_launch_count(h)
    finally:
        mb.muon_destroy(h)


def ns_both(mb, xs, **kw):
    outs = {}
    for mode in ("phases", "persistent"):
        h = handle(mb, mode)
        try:
            o = [torch.full_like(x, float("nan")) for x in xs]
            mb.muon_newton_schulz(h, xs, o, **kw)
            torch.cuda.synchronize()
            mb.muon_sync(h)
            outs[mode] = o
        finally:
            mb.muon_destroy(h)
    return outs["phases"], outs["persistent"]


@pytest.mark.parametrize("config,layers", [(1, [0, 1]), (2, [0]), (4, [0])])
def test_persistent_step_matches_per_phase_bits(mb, config, layers):
    """Three bf16 steps (fused weight update in the last Update) of depth-8 / depth-12
    layers and of one 3.8B-shape layer: weights and momentum bit for bit."""
    data = synth.make_matrix_set(config, layers=layers)
    G = [g.cuda() for g in data["G"]]
    res = {}
    for mode in ("phases", "persistent"):
        W = [w.cuda().clone() for w in data["W"]]
        M = [m.cuda().clone() for m in data["M"]]
        n = run_steps(mb, mode, W, G, M, steps=3 if config != 4 else 1, lr=0.02)
        res[mode] = (W, M, n)
    for a, b in zip(res["phases"][0], res["persistent"][0]):
        assert torch.equal(a, b)
    for a, b in zip(res["phases"][1], res["persistent"][1]):
        assert torch.equal(a, b)
    # one kernel for all Newton-Schulz steps instead of three per step
    assert res["persistent"][2] == res["phases"][2] - 15 + 1


def test_persistent_step_against_oracle_with_table(mb):
    """A depth-8 layer, 5-row table whose rows differ: fp32 zero weights and lr = 1 read
    O back exactly; O against the oracle, momentum bit for bit."""
    data = synth.make_matrix_set(1, layers=[0])
    G = [g.cuda() for g in data["G"]]
    M = [m.cuda() for m in data["M"]]
    W = [torch.zeros(s.rows, s.cols, device="cuda") for s in data["specs"]]
    run_steps(mb, "persistent", W, G, M, lr=1.0, momentum=0.95, coeffs=TABLE5, ns_steps=5)
    for i, spec in enumerate(data["specs"]):
        g = data["G"][i].float().numpy()
        _, m_new, o_ref = oracle.muon_step_matrix(np.zeros((spec.rows, spec.cols)), g, data["M"][i].numpy(),
                                                  lr=1.0, mu=0.95, nesterov=True, coeffs=TABLE5, eps=1e-7)
        assert np.array_equal(M[i].cpu().numpy(), m_new), spec
        o = -to64(W[i]) / oracle.update_scale(spec.rows, spec.cols)
        assert rel(o, o_ref) < BF16_TOL, (spec, rel(o, o_ref))


@pytest.mark.parametrize("ns_steps", [1, 2, 6, 16])
def test_persistent_newton_schulz_step_counts(mb, ns_steps):
    """muon_newton_schulz (separate export pass) for 1, 2, 6 and 16 steps (the most a call
    takes); shapes around the tile edges in 8 shape groups."""
    shapes = [(300, 130), (130, 300), (256, 256), (513, 257), (64, 1000), (1, 9), (9, 1), (129, 129),
              (300, 130), (256, 256)]
    xs = [synth.random_matrix(r, c, seed=300 + i, device="cuda", dtype=torch.bfloat16) for i, (r, c) in
          enumerate(shapes)]
    table = ((TABLE5 + [(1.5, -0.6, 0.1)]) * 3)[:ns_steps]
    a, b = ns_both(mb, xs, coeffs=table, ns_steps=ns_steps)
    for x, oa, ob in zip(xs, a, b):
        assert torch.equal(oa, ob), tuple(x.shape)
        want = oracle.newton_schulz(oracle.frobenius_normalise(to64(x), 1e-7), table)
        assert rel(to64(ob), want) < BF16_TOL, (tuple(x.shape), rel(to64(ob), want))


def test_persistent_edge_shapes(mb):
    """Degenerate and ragged shapes (one and two 256-blocks, tall and wide), in calls of
    at most 8 shape groups each."""
    edge = [(1, 9), (9, 1), (1, 1), (63, 130), (130, 63), (64, 64), (65, 257), (257, 65), (129, 129),
            (127, 300), (300, 255), (96, 96), (256, 32), (384, 1000), (513, 700), (700, 513)]
    for part in (edge[:8], edge[8:]):
        xs = [synth.random_matrix(r, c, seed=r * 7 + c, device="cuda", dtype=torch.bfloat16) for r, c in part]
        a, b = ns_both(mb, xs)
        for x, oa, ob in zip(xs, a, b):
            assert torch.equal(oa, ob), tuple(x.shape)


def test_persistent_options_match_per_phase_bits(mb):
    """Cautious weight decay (fused weight update) and NorMuon (separate weight update)
    in the persistent form: the per-phase form's bits."""
    data = synth.make_matrix_set(1, layers=[0])
    G = [g.cuda() for g in data["G"]]
    for kw in ({"weight_decay": 0.1, "cautious": True, "momentum_form": "lerp"}, {"normuon": True}):
        res = {}
        for mode in ("phases", "persistent"):
            W = [w.cuda().clone() for w in data["W"]]
            M = [m.cuda().clone() for m in data["M"]]
            opts = dict(kw)
            if opts.pop("normuon", False):
                opts["normuon_state"] = [torch.zeros(min(w.shape), device="cuda") for w in W]
            run_steps(mb, mode, W, G, M, steps=2, ex=True, lr=0.02, **opts)
            res[mode] = (W, M, opts.get("normuon_state"))
        for a, b in zip(res["phases"][0], res["persistent"][0]):
            assert torch.equal(a, b), kw
        for a, b in zip(res["phases"][1], res["persistent"][1]):
            assert torch.equal(a, b), kw
        if res["phases"][2] is not None:
            for a, b in zip(res["phases"][2], res["persistent"][2]):
                assert torch.equal(a, b)


def test_persistent_many_matrices_one_group(mb):
    """600 small matrices of two shapes (many items per cluster, fused weight-update table
    near its size limit): the per-phase form's bits."""
    shapes = [(40, 72) if i % 2 else (96, 33) for i in range(600)]
    G = [synth.random_matrix(r, c, seed=4000 + i, device="cuda", dtype=torch.bfloat16) for i, (r, c) in
         enumerate(shapes)]
    W0 = [synth.random_matrix(r, c, seed=7000 + i, device="cuda", dtype=torch.bfloat16) for i, (r, c) in
          enumerate(shapes)]
    res = {}
    for mode in ("phases", "persistent"):
        W = [w.clone() for w in W0]
        M = [torch.zeros(r, c, device="cuda") for r, c in shapes]
        run_steps(mb, mode, W, G, M, steps=2, lr=0.05)
        res[mode] = (W, M)
    for a, b in zip(res["phases"][0], res["persistent"][0]):
        assert torch.equal(a, b)


def test_persistent_cuda_graph_replays_bit_exact(mb):
    """The persistent step (counter reset and kernel) captured in a CUDA graph replays to
    the bits of eager persistent calls."""
    data = synth.make_matrix_set(1, layers=[0])
    G = [g.cuda() for g in data["G"]]
    W_e = [w.cuda().clone() for w in data["W"]]
    M_e = [m.cuda().clone() for m in data["M"]]
    W_g = [w.clone() for w in W_e]
    M_g = [m.clone() for m in M_e]
    h = handle(mb, "persistent")
    h2 = handle(mb, "persistent")
    try:
        s = torch.cuda.Stream()
        with torch.cuda.stream(s):
            mb.muon_step(h2, [w.clone() for w in W_g], G, [m.clone() for m in M_g], lr=0.02, stream=s)
        s.synchronize()
        mb.muon_sync(h2)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=s):
            mb.muon_step(h2, W_g, G, M_g, lr=0.02, stream=s)
        for _ in range(3):
            graph.replay()
        torch.cuda.synchronize()
        for _ in range(3):
            mb.muon_step(h, W_e, G, M_e, lr=0.02)
        torch.cuda.synchronize()
        mb.muon_sync(h)
        mb.muon_sync(h2)
        del graph
    finally:
        mb.muon_destroy(h)
        mb.muon_destroy(h2)
    for a, b in zip(W_e, W_g):
        assert torch.equal(a, b)
    for a, b in zip(M_e, M_g):
        assert torch.equal(a, b)


def test_launch_mode_argument_checks(mb):
    h = mb.muon_init(0)
    try:
        with pytest.raises(ValueError):
            mb.muon_set_launch_mode(h, "fast")
        lib = mb.load_library()
        assert lib.muon_set_launch_mode(h, 7) == mb.MUON_ERR_INVALID_ARG
        assert lib.muon_set_launch_mode(None, 0) == mb.MUON_ERR_INVALID_ARG
    finally:
        mb.muon_destroy(h)


def test_persistent_abort_path_reports_timeout_and_recovers(mb):
    """A dependency wait of the persistent launch is made to run out (1 ms limit, a count
    nothing reaches): the launch gives up, the time-out is reported by muon_sync, and
    the handle's next step gives the per-phase form's bits.  Nothing faults or hangs."""
    data = synth.make_matrix_set(1, layers=[0])
    G = [g.cuda() for g in data["G"]]
    h = handle(mb, "persistent")
    try:
        W = [w.cuda().clone() for w in data["W"]]
        M = [m.cuda().clone() for m in data["M"]]
        mb.muon_selftest_stall_persistent(h, 1_000_000)
        mb.muon_step(h, W, G, M, lr=0.02)
        torch.cuda.synchronize()
        with pytest.raises(mb.MuonError) as e:
            mb.muon_sync(h)
        assert e.value.code == mb.MUON_ERR_TIMEOUT
        mb.muon_sync(h)  # cleared
        # a clean step on the same handle from fresh state
        W = [w.cuda().clone() for w in data["W"]]
        M = [m.cuda().clone() for m in data["M"]]
        mb.muon_step(h, W, G, M, lr=0.02)
        torch.cuda.synchronize()
        mb.muon_sync(h)
    finally:
        mb.muon_destroy(h)
    W2 = [w.cuda().clone() for w in data["W"]]
    M2 = [m.cuda().clone() for m in data["M"]]
    run_steps(mb, "phases", W2, G, M2, lr=0.02)
    for a, b in zip(W, W2):
        assert torch.equal(a, b)
    for a, b in zip(M, M2):
        assert torch.equal(a, b)
    lib = mb.load_library()
    assert lib.muon_selftest_stall_persistent(None, 1000) == mb.MUON_ERR_INVALID_ARG


def test_persistent_launches_on_two_streams_at_once(mb):
    """Two handles run persistent steps on two streams at the same time, so the two
    launches compete for the SMs and neither can count on all its clusters being
    resident.  Work items are handed out in order, so both finish (no time-out) and
    each gives the bits of the same steps run alone."""
    sets = [synth.make_matrix_set(1, layers=[0]), synth.make_matrix_set(2, layers=[0])]
    alone, together = [], []
    for data in sets:
        W = [w.cuda().clone() for w in data["W"]]
        M = [m.cuda().clone() for m in data["M"]]
        run_steps(mb, "persistent", W, [g.cuda() for g in data["G"]], M, steps=3, lr=0.02)
        alone.append((W, M))
    hs = [handle(mb, "persistent") for _ in sets]
    streams = [torch.cuda.Stream() for _ in sets]
    try:
        state = []
        for data in sets:
            state.append(([w.cuda().clone() for w in data["W"]], [g.cuda() for g in data["G"]],
                          [m.cuda().clone() for m in data["M"]]))
        torch.cuda.synchronize()
        for _ in range(3):
            for h, st, (W, G, M) in zip(hs, streams, state):
                mb.muon_step(h, W, G, M, lr=0.02, stream=st)
        torch.cuda.synchronize()
        for h in hs:
            mb.muon_sync(h)
        together = [(W, M) for W, _, M in state]
    finally:
        for h in hs:
            mb.muon_destroy(h)
    for (wa, ma), (wt, mt) in zip(alone, together):
        for a, b in zip(wa + ma, wt + mt):
            assert torch.equal(a, b)
