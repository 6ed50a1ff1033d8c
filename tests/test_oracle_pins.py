"""Pins of the fp64 oracle to facts fixed by the pages and by the mathematics.

None of these re-types the oracle's loop.  Newton-Schulz is checked against
its closed form on the singular values (every step is an odd matrix
polynomial, so U and V are kept and each singular value follows the scalar
map phi(x) = a x + b x^3 + c x^5); momentum against recurrences worked by
hand; the quintic against the band the README states; the classical cubic
against the polar factor from an SVD.
"""
import math

import numpy as np
import pytest

import oracle
from newton_schulz_11_b200 import inputs
from tests.conftest import load_golden

PAGE = load_golden("quintic_page.json")
QUINTIC5 = [tuple(PAGE["coeffs"])] * PAGE["steps"]


def scalar_map(x, coeffs):
    """phi_K o ... o phi_1 applied to an array of scalars."""
    y = np.asarray(x, np.float64).copy()
    for a, b, c in coeffs:
        y = a * y + b * y ** 3 + c * y ** 5
    return y


def closed_form_ns(G, coeffs, eps):
    """U diag(phi(sigma / (||G||_F + eps))) V^T from an fp64 SVD."""
    G = np.asarray(G, np.float64)
    U, s, Vt = np.linalg.svd(G, full_matrices=False)
    fro = math.sqrt(float(np.sum(s * s)))
    return (U * scalar_map(s / (fro + eps), coeffs)) @ Vt


def rel(a, b):
    return float(np.linalg.norm(np.asarray(a) - np.asarray(b)) / max(np.linalg.norm(np.asarray(b)), 1e-300))


def test_page_constants():
    assert tuple(oracle.QUINTIC) == tuple(PAGE["coeffs"])
    assert oracle.NS_EPS == PAGE["eps"]


# ---------------------------------------------------------------- momentum / Nesterov

def test_momentum_handworked_sequence():
    h = load_golden("momentum_handworked.json")["sequence"]
    m = np.array(h["m0"], np.float64)
    for g, m_exp, u_exp in zip(h["grads"], h["momentum"], h["nesterov_u"]):
        g = np.array(g, np.float64)
        m = oracle.momentum_update(m, g, h["beta"])
        assert np.array_equal(m, np.array(m_exp, np.float64))
        u = oracle.nesterov_input(g, m, h["beta"], True)
        assert np.array_equal(u, np.array(u_exp, np.float64))
        assert np.array_equal(oracle.nesterov_input(g, m, h["beta"], False), m)


def test_momentum_nonzero_start():
    h = load_golden("momentum_handworked.json")["nonzero_start"]
    m = oracle.momentum_update(np.array(h["m0"]), np.array(h["grad"]), h["beta"])
    assert np.array_equal(m, np.array(h["momentum"], np.float64))
    assert np.array_equal(oracle.nesterov_input(np.array(h["grad"]), m, h["beta"], True),
                          np.array(h["nesterov_u"], np.float64))
    assert np.array_equal(oracle.nesterov_input(np.array(h["grad"]), m, h["beta"], False),
                          np.array(h["plain_u"], np.float64))


def test_three_step_trajectory_is_geometric_sum():
    """From m0 = 0, three steps leave m = beta^2 g1 + beta g2 + g3 (unrolled recurrence)."""
    w = inputs.WORKLOADS["mlp-768x3072-bf16-3steps"]
    w = inputs.scaled_workload(w, [(16, 40)])
    g = [inputs.grad_np(w, s, 0).astype(np.float64) for s in range(3)]
    beta = 0.95
    m = np.zeros_like(g[0])
    for s in range(3):
        m = oracle.momentum_update(m, g[s], beta)
    expect = beta * beta * g[0] + beta * g[1] + g[2]
    assert rel(m, expect) < 1e-15


# ---------------------------------------------------------------- Newton-Schulz closed form

SHAPES = [(8, 8), (16, 40), (40, 16), (64, 24), (1, 7), (7, 1), (33, 33)]


@pytest.mark.parametrize("shape", SHAPES)
def test_ns_matches_svd_closed_form_quintic(shape):
    rng = np.random.default_rng(1234 + shape[0] * 100 + shape[1])
    G = rng.standard_normal(shape)
    G[: min(shape) // 2 or 1] *= 30.0  # uneven spectrum
    O = oracle.newton_schulz(G, QUINTIC5, 1e-7)
    assert O.shape == G.shape
    assert rel(O, closed_form_ns(G, QUINTIC5, 1e-7)) < 1e-10


@pytest.mark.parametrize("shape", [(12, 20), (20, 12), (9, 9)])
def test_ns_closed_form_any_table(shape):
    """Holds for any odd-quintic table, including per-iteration schedules."""
    rng = np.random.default_rng(99)
    G = rng.standard_normal(shape)
    table = [(2.1, -1.3, 0.4), (1.7, -0.9, 0.2), (3.0, -3.2, 1.1), (1.5, -0.5, 0.0)]
    assert rel(oracle.newton_schulz(G, table, 1e-7), closed_form_ns(G, table, 1e-7)) < 1e-10


def test_ns_rank_deficient_keeps_rank():
    rng = np.random.default_rng(5)
    G = rng.standard_normal((20, 3)) @ rng.standard_normal((3, 30))
    O = oracle.newton_schulz(G, QUINTIC5)
    s = np.linalg.svd(O, compute_uv=False)
    assert np.sum(s > 1e-8) == 3
    assert rel(O, closed_form_ns(G, QUINTIC5, 1e-7)) < 1e-10


def test_ns_eps_placement_tiny_matrix():
    """eps is added to the norm (not to its square): visible when ||G|| ~ eps."""
    G = np.array([[3e-8, 4e-8]])  # ||G|| = 5e-8, comparable to eps = 1e-7
    O = oracle.newton_schulz(G, QUINTIC5, 1e-7)
    x = 5e-8 / (5e-8 + 1e-7)
    expect = scalar_map(np.array([x]), QUINTIC5)[0] * np.array([[0.6, 0.8]])
    assert rel(O, expect) < 1e-12


def test_ns_tiny_bruteforce():
    """1x2 and 2x1 rank-one inputs: singular value 5, directions by hand."""
    x = 5.0 / (5.0 + 1e-7)
    f = scalar_map(np.array([x]), QUINTIC5)[0]
    assert rel(oracle.newton_schulz(np.array([[3.0, 4.0]]), QUINTIC5), f * np.array([[0.6, 0.8]])) < 1e-13
    assert rel(oracle.newton_schulz(np.array([[3.0], [4.0]]), QUINTIC5), f * np.array([[0.6], [0.8]])) < 1e-13
    # 1x1: sign(g) * phi^5(|g| / (|g| + eps))
    y = scalar_map(np.array([2.0 / (2.0 + 1e-7)]), QUINTIC5)[0]
    assert abs(oracle.newton_schulz(np.array([[-2.0]]), QUINTIC5)[0, 0] + y) < 1e-14


def test_ns_diagonal_by_hand():
    """diag(3, 4): singular values 3 and 4, norm 5, so O = diag(phi(0.6), phi(0.8)) up to eps."""
    G = np.diag([3.0, 4.0])
    O = oracle.newton_schulz(G, QUINTIC5)
    d = scalar_map(np.array([3.0, 4.0]) / (5.0 + 1e-7), QUINTIC5)
    assert np.allclose(O, np.diag(d), rtol=0, atol=1e-14)


# ---------------------------------------------------------------- polar limit and band

def test_cubic_newton_schulz_converges_to_polar_factor():
    """(1.5, -0.5, 0) is the classical Newton-Schulz iteration (Higham, Functions of
    Matrices, eq. 5.22, cited by the README): it converges to U V^T."""
    rng = np.random.default_rng(7)
    for shape in [(24, 40), (40, 24), (16, 16)]:
        U, _ = np.linalg.qr(rng.standard_normal((shape[0], min(shape))))
        V, _ = np.linalg.qr(rng.standard_normal((shape[1], min(shape))))
        s = np.linspace(0.05, 3.0, min(shape))
        G = (U * s) @ V.T
        O = oracle.newton_schulz(G, [(1.5, -0.5, 0.0)] * 60)
        assert rel(O, U @ V.T) < 1e-13


def test_quintic_band_after_five_steps():
    """Singular values of NS5(G) lie in the band that five applications of the page's
    quintic reach: computed here by dense sampling of the scalar map."""
    xs = np.linspace(0.0, 1.0, 400001)
    ys = scalar_map(xs, QUINTIC5)
    tau = xs[np.nonzero(ys < 0.68)[0].max() + 1]
    assert 1.4e-3 < tau < 1.6e-3
    hi = ys.max()
    assert 1.20 < hi < 1.21
    w = inputs.WORKLOADS["single-256x128-f32"]
    G = inputs.grad_np(w, 0, 0).astype(np.float64)
    O = oracle.newton_schulz(G, QUINTIC5)
    s_in = np.linalg.svd(G, compute_uv=False)
    x = s_in / (np.linalg.norm(G) + 1e-7)
    s_out = np.sort(np.linalg.svd(O, compute_uv=False))
    assert np.allclose(s_out, np.sort(scalar_map(x, QUINTIC5)), rtol=1e-10, atol=1e-12)
    band = scalar_map(x[x >= 1.6e-3], QUINTIC5)
    assert band.size > 0
    assert band.min() >= 0.68 and band.max() <= 1.21


def test_quintic_limit_band_matches_page():
    """Repeated application converges to [0.68, 1.13] as the README says."""
    xs = np.linspace(0.01, 1.0, 200001)
    ys = scalar_map(xs, [PAGE["coeffs"]] * 300)
    lo, hi = PAGE["limit_band_page"]
    assert abs(ys.min() - lo) < 0.005 and abs(ys.max() - hi) < 0.005


def test_workload_single_matrix_against_polar_factor():
    """The 256x128 fp32 workload: oracle NS equals its closed form and sits near U V^T."""
    w = inputs.WORKLOADS["single-256x128-f32"]
    g = inputs.grad_np(w, 0, 0).astype(np.float64)
    m = inputs.momentum_np(w, 0).astype(np.float64)
    Wt = inputs.weight_np(w, 0).astype(np.float64)
    W1, m1, O = oracle.muon_step(Wt, g, m, lr=w.lr, beta=w.beta, weight_decay=w.weight_decay,
                                 nesterov=True, coeffs=QUINTIC5)
    u = g + w.beta * (w.beta * m + g)
    assert rel(O, closed_form_ns(u, QUINTIC5, 1e-7)) < 1e-10
    U, s, Vt = np.linalg.svd(u, full_matrices=False)
    polar = U @ Vt
    # The quintic does not converge to 1: per-direction error is bounded by the band.
    cos = float(np.sum(O * polar) / (np.linalg.norm(O) * np.linalg.norm(polar)))
    assert cos > 0.9
    assert rel(W1, Wt - w.lr * math.sqrt(2.0) * O) < 1e-15


# ---------------------------------------------------------------- invariances

def test_ns_invariances():
    rng = np.random.default_rng(3)
    G = rng.standard_normal((18, 30))
    O = oracle.newton_schulz(G, QUINTIC5)
    # transpose
    assert rel(oracle.newton_schulz(G.T, QUINTIC5), O.T) < 1e-12
    # orthogonal equivariance
    Q, _ = np.linalg.qr(rng.standard_normal((18, 18)))
    R, _ = np.linalg.qr(rng.standard_normal((30, 30)))
    assert rel(oracle.newton_schulz(Q @ G @ R, QUINTIC5), Q @ O @ R) < 1e-11
    # positive scaling (up to eps)
    assert rel(oracle.newton_schulz(1000.0 * G, QUINTIC5), O) < 1e-8
    # zero maps to zero
    assert np.array_equal(oracle.newton_schulz(np.zeros((4, 6)), QUINTIC5), np.zeros((4, 6)))


# ---------------------------------------------------------------- update rule and scale

def test_shape_scale_values():
    for rows, cols, s in load_golden("shape_scale.json")["cases"]:
        assert abs(oracle.default_shape_scale(rows, cols) - s) < 1e-15


def test_decay_only_when_gradient_is_zero():
    h = load_golden("momentum_handworked.json")["decay_only"]
    W = np.array(h["W"], np.float64)
    W1, m1, O = oracle.muon_step(W, np.zeros_like(W), np.zeros_like(W), lr=h["lr"], beta=0.95,
                                 weight_decay=h["weight_decay"], nesterov=True, coeffs=QUINTIC5)
    assert np.array_equal(O, np.zeros_like(W))
    assert np.allclose(W1, np.array(h["W_new"]), rtol=0, atol=1e-15)


def test_update_moves_against_gradient_and_lr_zero_is_identity():
    rng = np.random.default_rng(11)
    W = rng.standard_normal((12, 20))
    g = rng.standard_normal((12, 20))
    W1, _, O = oracle.muon_step(W, g, np.zeros_like(g), lr=0.1, beta=0.9, weight_decay=0.0,
                                nesterov=False, coeffs=QUINTIC5)
    assert float(np.sum((W1 - W) * g)) < 0
    W0, _, _ = oracle.muon_step(W, g, np.zeros_like(g), lr=0.0, beta=0.9, weight_decay=0.3,
                                nesterov=True, coeffs=QUINTIC5)
    assert np.array_equal(W0, W)


def test_tall_scale_doubles_step():
    """3072x768-like tall shape: the orthogonalised step is scaled by 2 (shape rule)."""
    rng = np.random.default_rng(12)
    g = rng.standard_normal((64, 16))
    W = np.zeros((64, 16))
    W1, _, O = oracle.muon_step(W, g, np.zeros_like(g), lr=0.1, beta=0.0, weight_decay=0.0,
                                nesterov=False, coeffs=QUINTIC5)
    assert rel(-W1, 0.1 * 2.0 * O) < 1e-15
