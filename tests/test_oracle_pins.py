"""Pins of the CPU oracle to facts fixed outside itself (closed forms, library
routines, invariants, the pages' printed numbers).  CPU only.

Each pin is a function of the Newton-Schulz / step implementation it checks, so the
last tests can plant mistakes in a copy of the oracle and show that some pin fails.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle
from oracle import CUBIC, QUINTIC, newton_schulz
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- helpers (test side)

def scalar_map(x, coeffs):
    """Odd polynomial each Newton-Schulz step applies to every singular value:
    with X = U S V^T, X^T X = V S^2 V^T, so a X + X(b A + c A^2) = U (a S + b S^3 + c S^5) V^T."""
    x = np.asarray(x, dtype=np.float64)
    for a, b, c in coeffs:
        x = a * x + b * x ** 3 + c * x ** 5
    return x


def conditioned(rows, cols, seed, lo=0.1, hi=1.0):
    """Random full-rank matrix U diag(s) V^T with singular values in [lo, hi]."""
    rng = np.random.default_rng(seed)
    k = min(rows, cols)
    u, _ = np.linalg.qr(rng.standard_normal((rows, k)))
    v, _ = np.linalg.qr(rng.standard_normal((cols, k)))
    s = rng.uniform(lo, hi, size=k)
    return (u * s) @ v.T, s


def polar_svd(x):
    u, _, vt = np.linalg.svd(x, full_matrices=False)
    return u @ vt


def rel(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


# ---------------------------------------------------------------- pin functions

def pin_diagonal(ns):
    """A rectangular diagonal input stays diagonal, each entry mapped by the scalar
    polynomial (closed form)."""
    for rows, cols in [(5, 3), (3, 5), (4, 4)]:
        d = np.array([0.9, 0.5, 0.2, 0.05][:min(rows, cols)])
        x = np.zeros((rows, cols))
        x[np.arange(d.size), np.arange(d.size)] = d
        coeffs = [QUINTIC] * 5
        want = np.zeros_like(x)
        want[np.arange(d.size), np.arange(d.size)] = scalar_map(d, coeffs)
        got = ns(x, coeffs)
        assert np.allclose(got, want, rtol=1e-13, atol=1e-15), (rows, cols)


def pin_spectral_map(ns):
    """O = U diag(f5(s)) V^T with X0 = U diag(s) V^T (closed form of the iteration)."""
    for (rows, cols, seed) in [(24, 9, 1), (9, 24, 2), (17, 17, 3), (40, 40, 4), (64, 16, 5)]:
        x, _ = conditioned(rows, cols, seed, lo=0.02, hi=1.0)
        u, s, vt = np.linalg.svd(x, full_matrices=False)
        coeffs = [QUINTIC] * 5
        want = (u * scalar_map(s, coeffs)) @ vt
        got = ns(x, coeffs)
        assert rel(got, want) < 1e-11, (rows, cols, rel(got, want))
        sv_got = np.sort(np.linalg.svd(got, compute_uv=False))
        sv_want = np.sort(np.abs(scalar_map(s, coeffs)))
        assert np.allclose(sv_got, sv_want, rtol=1e-11, atol=1e-13)


# An invented per-step table whose rows differ (the pages give the triples per step but
# print none): each row's scalar map stays bounded on (0, 1.3].
TABLE_ROWS_DIFFER = [QUINTIC, tuple(0.9 * v for v in QUINTIC), CUBIC, (2.0, -1.5, 0.5), (3.0, -3.2, 1.2)]


def pin_spectral_map_table(ns):
    """With row k of a table used in step k, O = U diag(f_K(...f_1(s))) V^T: the steps'
    scalar maps compose in the table's order (closed form of the iteration)."""
    for (rows, cols, seed) in [(24, 9, 6), (9, 24, 7), (20, 20, 8)]:
        x, _ = conditioned(rows, cols, seed, lo=0.02, hi=1.0)
        u, s, vt = np.linalg.svd(x, full_matrices=False)
        want = (u * scalar_map(s, TABLE_ROWS_DIFFER)) @ vt
        got = ns(x, TABLE_ROWS_DIFFER)
        assert rel(got, want) < 1e-11, (rows, cols, rel(got, want))


def pin_polar(ns):
    """Cubic triple iterated to convergence = the SVD polar factor U V^T."""
    for (rows, cols, seed) in [(8, 5, 11), (5, 8, 12), (16, 16, 13), (12, 3, 14)]:
        x, s = conditioned(rows, cols, seed)
        # s <= 1, so no normalisation is needed for convergence of the cubic map
        prev = x
        for _ in range(100):
            cur = ns(prev, [CUBIC])
            if np.linalg.norm(cur - prev) < 1e-14:
                break
            prev = cur
        assert rel(cur, polar_svd(x)) < 1e-10, (rows, cols)


def pin_transpose(ns):
    """Tall and wide rules agree on transposed inputs: NS(X^T) = NS(X)^T."""
    rng = np.random.default_rng(21)
    for rows, cols in [(32, 8), (33, 17), (70, 70)]:
        x = rng.standard_normal((rows, cols))
        x /= np.linalg.norm(x)
        coeffs = [QUINTIC] * 5
        a = ns(x.T, coeffs)
        b = ns(x, coeffs).T
        assert rel(a, b) < 1e-13, (rows, cols)


PINS = [pin_diagonal, pin_spectral_map, pin_spectral_map_table, pin_polar, pin_transpose]


# ---------------------------------------------------------------- the pins on the oracle

@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_newton_schulz_pins(pin):
    pin(newton_schulz)


def test_orthogonal_fixed_point():
    """An orthogonal Q is a fixed point of the cubic step (1.5 Q - 0.5 Q Q^T Q = Q),
    and normalise-then-converge returns it."""
    rng = np.random.default_rng(31)
    for n in (4, 9, 16):
        q, _ = np.linalg.qr(rng.standard_normal((n, n)))
        assert rel(newton_schulz(q, [CUBIC]), q) < 1e-14
        x = oracle.frobenius_normalise(q, 0.0)
        for _ in range(100):
            x = newton_schulz(x, [CUBIC])
        assert rel(x, q) < 1e-10
    # rectangular: orthonormal columns / rows are fixed too
    q, _ = np.linalg.qr(rng.standard_normal((10, 4)))
    assert rel(newton_schulz(q, [CUBIC]), q) < 1e-14
    assert rel(newton_schulz(q.T, [CUBIC]), q.T) < 1e-14


def test_quintic_range_tiny_set():
    """With the quintic triple x5, normalised inputs whose singular values are all
    >= 2e-3 come out with singular values in [0.68, 1.21] (scalar map: max on (0,1]
    is 1.2024, min over [2e-3, 1] is 0.6818)."""
    grid = np.linspace(2e-3, 1.0, 200001)
    f5 = scalar_map(grid, [QUINTIC] * 5)
    assert 0.68 < f5.min() < 0.69 and 1.20 < f5.max() < 1.21
    data = synth.make_matrix_set(0)
    checked = 0
    for spec, g in zip(data["specs"], data["G"]):
        _, _, o = oracle.muon_step_matrix(np.zeros((spec.rows, spec.cols)), g.numpy(),
                                          np.zeros((spec.rows, spec.cols), np.float32),
                                          lr=0.02, mu=0.95, nesterov=True, eps=1e-7)
        _, u = oracle.nesterov_momentum_f32(g.numpy(), np.zeros((spec.rows, spec.cols), np.float32), 0.95, True)
        s0 = np.linalg.svd(oracle.frobenius_normalise(u, 1e-7), compute_uv=False)
        sv = np.linalg.svd(o, compute_uv=False)
        if s0.min() >= 2e-3:
            assert sv.min() >= 0.68 and sv.max() <= 1.21, spec
            checked += 1
        # at any input the output follows the scalar map
        assert np.allclose(np.sort(sv), np.sort(np.abs(scalar_map(s0, [QUINTIC] * 5))), rtol=1e-9, atol=1e-11)
    assert checked >= 3


# ---------------------------------------------------------------- momentum (float32 buffer)

def test_momentum_exact_small_cases():
    m = np.array([2.0, -4.0, 0.0, 1.5], np.float32)
    g = np.array([1.0, 1.0, -3.0, 0.25], np.float32)
    m_new, u = oracle.nesterov_momentum_f32(g, m, 0.5, True)
    assert np.array_equal(m_new, np.array([2.0, -1.0, -3.0, 1.0], np.float32))
    assert np.array_equal(u, np.array([2.0, 0.5, -4.5, 0.75]))
    m_new2, u2 = oracle.nesterov_momentum_f32(g, m, 0.5, False)
    assert np.array_equal(m_new2, m_new) and np.array_equal(u2, m_new.astype(np.float64))


def test_momentum_two_roundings_not_fused():
    """The buffer update rounds mu*M and then the sum (no fused multiply-add)."""
    rng = np.random.default_rng(41)
    mu32 = np.float32(0.95)
    m = rng.standard_normal(20000).astype(np.float32)
    g = rng.standard_normal(20000).astype(np.float32)
    m_new, _ = oracle.nesterov_momentum_f32(g, m, 0.95, True)
    two = np.float32(np.float32(mu32 * m) + g)
    fused = (np.float64(mu32) * m.astype(np.float64) + g.astype(np.float64)).astype(np.float32)
    assert np.array_equal(m_new, two)
    assert np.count_nonzero(m_new != fused) > 0  # the two readings are distinguishable here


def test_momentum_constant_gradient_closed_form():
    """Constant gradient g from M = 0: M_k = g (1 - mu^k)/(1 - mu), U_k = g + mu M_k."""
    mu = 0.9
    g = np.full(8, 0.125, np.float32)
    m = np.zeros(8, np.float32)
    for k in range(1, 30):
        m, u = oracle.nesterov_momentum_f32(g, m, mu, True)
        mk = 0.125 * (1 - np.float64(np.float32(mu)) ** k) / (1 - np.float64(np.float32(mu)))
        assert np.allclose(m, mk, rtol=1e-5)
        assert np.allclose(u, 0.125 + np.float64(np.float32(mu)) * mk, rtol=1e-5)


# ---------------------------------------------------------------- whole step

@pytest.mark.parametrize("rows,cols,scale", [(8, 2, 2.0), (2, 8, 1.0), (6, 6, 1.0), (12, 3, 2.0), (9, 4, 1.5)])
def test_step_with_converged_polar(rows, cols, scale):
    """With a converging coefficient table the step is W - lr*sqrt(max(1,r/c))*UV^T
    of U = G + mu*M_new (SVD polar factor; scale values worked by hand)."""
    g, _ = conditioned(rows, cols, 100 + rows * cols, lo=0.3, hi=1.0)
    rng = np.random.default_rng(7)
    w = rng.standard_normal((rows, cols))
    m = np.zeros((rows, cols), np.float32)
    assert oracle.update_scale(rows, cols) == pytest.approx(scale)
    w_new, m_new, o = oracle.muon_step_matrix(w, g.astype(np.float32), m, lr=0.1, mu=0.9,
                                              nesterov=True, coeffs=[CUBIC] * 80, eps=0.0)
    u = g.astype(np.float32).astype(np.float64) * (1 + np.float64(np.float32(0.9)))
    assert rel(o, polar_svd(u)) < 1e-10
    assert np.allclose(w_new, w - 0.1 * scale * polar_svd(u), atol=1e-10)
    assert np.array_equal(m_new, g.astype(np.float32))


def test_zero_gradient_and_scale_invariance():
    shape = (12, 7)
    z = np.zeros(shape, np.float32)
    w = np.ones(shape)
    w_new, m_new, o = oracle.muon_step_matrix(w, z, z, lr=0.02, mu=0.95, eps=1e-7)
    assert np.array_equal(o, np.zeros(shape)) and np.array_equal(w_new, w)
    assert np.array_equal(m_new, z)
    rng = np.random.default_rng(5)
    g = rng.standard_normal(shape).astype(np.float32)
    _, _, o1 = oracle.muon_step_matrix(w, g, z, lr=0.02, mu=0.95, eps=0.0)
    _, _, o2 = oracle.muon_step_matrix(w, np.float32(8.0) * g, z, lr=0.02, mu=0.95, eps=0.0)
    assert rel(o2, o1) < 1e-13
    _, _, o3 = oracle.muon_step_matrix(w, g, z, lr=0.02, mu=0.95, eps=1e-7)
    assert rel(o3, o1) < 1e-5


def test_brute_force_loops_match_tiny():
    """Pure-Python triple loops (no NumPy matmul) on 5x3 and 3x5, two quintic steps."""
    def mm(p, q):
        return [[sum(p[i][k] * q[k][j] for k in range(len(q))) for j in range(len(q[0]))]
                for i in range(len(p))]

    def tr(p):
        return [list(r) for r in zip(*p)]

    def axpy(a, x, b, y):
        return [[a * x[i][j] + b * y[i][j] for j in range(len(x[0]))] for i in range(len(x))]

    rng = np.random.default_rng(9)
    for rows, cols in [(5, 3), (3, 5)]:
        x0 = rng.standard_normal((rows, cols)) / 4
        x = x0.tolist()
        for a, b, c in [QUINTIC, QUINTIC]:
            if rows > cols:
                A = mm(tr(x), x)
                B = axpy(b, A, c, mm(A, A))
                x = axpy(a, x, 1.0, mm(x, B))
            else:
                A = mm(x, tr(x))
                B = axpy(b, A, c, mm(A, A))
                x = axpy(a, x, 1.0, mm(B, x))
        assert rel(newton_schulz(x0, [QUINTIC] * 2), np.array(x)) < 1e-14


# ---------------------------------------------------------------- the pages' printed numbers

def test_llama_shape_set_matches_printed_parameter_count():
    with open(os.path.join(GOLDEN, "little_lm_params.json")) as f:
        gold = json.load(f)
    specs = synth.config_shapes(4)
    assert len(specs) == 6 * gold["decoder_layers"] == 168
    total_m = sum(s.rows * s.cols for s in specs) / 1e6
    # the projections are all but the norm weights and scalars of the decoder layers
    assert total_m <= gold["decoder_layers_params_millions"]
    assert abs(total_m - gold["decoder_layers_params_millions"]) / gold["decoder_layers_params_millions"] < 1e-3
    # GQA: 24 query heads / 8 kv heads of 128 give the 3072 / 1024 projection widths
    assert 24 * 128 == 3072 and gold["kv_heads"] * 128 == 1024


# ---------------------------------------------------------------- planted mistakes

def _mutant(kind):
    def ns(x0, coeffs):
        x = np.array(x0, dtype=np.float64, copy=True)
        tall = x.shape[0] > x.shape[1]
        rows = list(coeffs)
        if kind == "reverse_rows":
            rows = rows[::-1]
        if kind == "first_row_only":
            rows = [rows[0]] * len(rows)
        for a, b, c in rows:
            if kind == "drop_c":
                c = 0.0
            if kind == "sign_b":
                b = -b
            gram = x.T @ x if tall else x @ x.T
            poly = b * gram + c * (gram @ gram)
            if kind == "swap_side" and not tall:
                x = a * x + x @ poly
            elif kind == "drop_a":
                x = x + (x @ poly if tall else poly @ x)
            else:
                x = a * x + (x @ poly if tall else poly @ x)
        return x
    return ns


@pytest.mark.parametrize("kind", ["drop_c", "sign_b", "swap_side", "drop_a", "reverse_rows", "first_row_only"])
def test_pins_catch_planted_mistakes(kind):
    bad = _mutant(kind)
    caught = 0
    for pin in PINS:
        try:
            pin(bad)
        except (AssertionError, ValueError):
            caught += 1
    assert caught >= 1, kind


# ---------------------------------------------------------------- options: lerp momentum, weight decay

def test_lerp_momentum_closed_form():
    """Interpolation form from M = 0 with a constant gradient: M_k = g (1 - mu^k),
    U_k = (1 - mu) g + mu M_k; exact small case with mu = 0.5."""
    mu = 0.75
    g = np.full(6, 0.5, np.float32)
    m = np.zeros(6, np.float32)
    for k in range(1, 25):
        m, u = oracle.nesterov_momentum_f32(g, m, mu, True, lerp=True)
        mk = 0.5 * (1 - 0.75 ** k)
        assert np.allclose(m, mk, rtol=1e-6)
        assert np.allclose(u, 0.25 * 0.5 + 0.75 * mk, rtol=1e-6)
    m2, u2 = oracle.nesterov_momentum_f32(np.array([1.0, -2.0], np.float32), np.array([4.0, 2.0], np.float32),
                                         0.5, True, lerp=True)
    assert np.array_equal(m2, np.array([2.5, 0.0], np.float32))
    assert np.array_equal(u2, np.array([1.75, -1.0]))


def test_weight_decay_and_cautious_mask_closed_form():
    """Diagonal gradient: O is diagonal with the scalar map's (positive) values and zero
    elsewhere, so the cautious mask (O * W >= 0) is false only where a diagonal entry
    of W is negative; the decayed weights are worked out by hand."""
    g = np.diag([0.8, 0.6, 0.3]).astype(np.float32)
    w = np.array([[0.5, -0.2, 0.1], [0.3, -0.4, -0.6], [-0.7, 0.2, 0.9]])
    z = np.zeros((3, 3), np.float32)
    coeffs = [QUINTIC] * 5
    w_plain, _, o = oracle.muon_step_matrix(w, g, z, lr=0.1, mu=0.0, coeffs=coeffs, eps=0.0)
    d = np.array([0.8, 0.6, 0.3]) / np.linalg.norm([0.8, 0.6, 0.3])
    od = scalar_map(d, coeffs)
    assert np.allclose(o, np.diag(od), atol=1e-15) and np.all(od > 0)
    # O is zero off the diagonal (mask true there), positive on it (mask = W >= 0)
    mask = np.ones((3, 3), bool)
    mask[1, 1] = False  # W[1,1] = -0.4 < 0 while O[1,1] > 0
    assert np.array_equal(oracle.cautious_mask(o, w), mask)
    w_cwd, _, _ = oracle.muon_step_matrix(w, g, z, lr=0.1, mu=0.0, coeffs=coeffs, eps=0.0, weight_decay=0.5,
                                          cautious=True)
    assert np.allclose(w_cwd, w - 0.1 * np.diag(od) - 0.05 * np.where(mask, w, 0.0), atol=1e-15)
    w_wd, _, _ = oracle.muon_step_matrix(w, g, z, lr=0.1, mu=0.0, coeffs=coeffs, eps=0.0, weight_decay=0.5)
    assert np.allclose(w_wd, w_plain - 0.05 * w, atol=1e-15)


# ---------------------------------------------------------------- NorMuon

@pytest.mark.parametrize("rows,cols", [(3, 5), (5, 3), (4, 4)])
def test_normuon_on_a_diagonal_input(rows, cols):
    """Diagonal O (entries d_i): one statistic per index of the shorter dimension,
    q_i = d_i^2 / L; from v = 0, v = (1-b2) q, so O' = d_i / (sqrt(1-b2) d_i/sqrt(L) + eps)
    is (nearly) the same for every i, and O'' has O's Frobenius norm."""
    k = min(rows, cols)
    L = max(rows, cols)
    d = np.array([0.9, 0.5, 0.25, 0.1][:k])
    o = np.zeros((rows, cols))
    o[np.arange(k), np.arange(k)] = d
    o2, v = oracle.normuon_rescale(o, np.zeros(k), 0.9, 1e-12)
    assert np.allclose(v, 0.1 * d ** 2 / L, rtol=1e-14)
    diag = o2[np.arange(k), np.arange(k)]
    assert np.allclose(diag, diag[0], rtol=1e-9)
    assert np.isclose(np.linalg.norm(o2), np.linalg.norm(o), rtol=1e-14)
    assert np.count_nonzero(o2) == k
    # second step with the same O: v = 0.9 v1 + 0.1 q = 0.19 q
    _, v2 = oracle.normuon_rescale(o, v, 0.9, 1e-12)
    assert np.allclose(v2, 0.19 * d ** 2 / L, rtol=1e-13)


def test_normuon_rows_vs_columns_by_aspect():
    rng = np.random.default_rng(77)
    o = rng.standard_normal((4, 9))
    _, v_wide = oracle.normuon_rescale(o, np.zeros(4), 0.0, 0.0)
    assert np.allclose(v_wide, np.mean(o ** 2, axis=1))
    _, v_tall = oracle.normuon_rescale(o.T, np.zeros(4), 0.0, 0.0)
    assert np.allclose(v_tall, np.mean(o ** 2, axis=1))
    # transposing the input transposes the output
    a, _ = oracle.normuon_rescale(o, np.full(4, 0.3), 0.5, 1e-6)
    b, _ = oracle.normuon_rescale(o.T, np.full(4, 0.3), 0.5, 1e-6)
    assert np.allclose(a, b.T, rtol=1e-14)


def test_normalisation_adds_eps_to_the_norm():
    """X0 = U / (||U||_F + eps): with ||U|| = 5 and eps = 1 the divisor is 6, not
    sqrt(25 + 1) (eps added to the squared norm) nor 5 (eps ignored)."""
    x0 = oracle.frobenius_normalise(np.array([[3.0, 4.0]]), 1.0)
    assert np.allclose(x0, [[0.5, 4.0 / 6.0]], rtol=0, atol=1e-15)


@pytest.mark.parametrize("tall", [False, True])
def test_step_rank_one_closed_form(tall):
    """Whole step on a rank-one gradient, closed form.  With M = 0 and Nesterov, M' = G and
    U = (1 + mu) G; X0 = U / (||U|| + eps) has the single singular value
    s = (1 + mu)||G|| / ((1 + mu)||G|| + eps) and the same singular vectors, so
    O = f5(s) G / ||G|| and W' = W - lr sqrt(max(1, r/c)) O."""
    u = np.array([1.0, 2.0, 2.0]) / 3.0            # unit vectors
    v = np.array([3.0, 4.0]) / 5.0
    g = 2.5 * np.outer(u, v)                         # 3 x 2 (tall) or 2 x 3 (wide), ||G|| = 2.5
    if not tall:
        g = g.T
    mu, eps, lr = 0.5, 0.25, 0.1
    w = np.full(g.shape, 0.125)
    w_new, m_new, o = oracle.muon_step_matrix(w, g.astype(np.float32), np.zeros(g.shape, np.float32), lr=lr,
                                              mu=mu, nesterov=True, eps=eps)
    s = (1 + mu) * 2.5 / ((1 + mu) * 2.5 + eps)
    f5 = scalar_map(np.array([s]), [QUINTIC] * 5)[0]
    # G is rounded to float32 on the way in; compare at float32 resolution
    assert np.allclose(o, f5 * g / 2.5, rtol=1e-6, atol=1e-7)
    scale = math.sqrt(max(1.0, g.shape[0] / g.shape[1]))
    assert np.allclose(w_new, w - lr * scale * o, rtol=0, atol=1e-15)
    assert np.array_equal(m_new, g.astype(np.float32))
