"""Pins of the fp64 AdamW oracle (CPU): hand-worked recurrences, closed forms and
invariances that a dropped bias correction, a misplaced eps or decay, or a swapped beta
would break."""
import numpy as np
import pytest

from oracle import adamw_oracle as ao
from tests.conftest import load_golden


def test_moments_handworked():
    h = load_golden("adamw_handworked.json")
    m = np.zeros(3)
    v = np.zeros(3)
    for g, m_exp, v_exp in zip(h["grads"], h["m"], h["v"]):
        m, v = ao.adamw_moments(m, v, np.array(g), h["beta1"], h["beta2"])
        assert np.array_equal(m, np.array(m_exp))
        assert np.array_equal(v, np.array(v_exp))


def test_first_step_handworked():
    h = load_golden("adamw_handworked.json")
    f = h["first_step"]
    p1, m1, v1 = ao.adamw_step(np.array(f["p0"]), np.array(h["grads"][0]), np.zeros(3), np.zeros(3), lr=f["lr"],
                               beta1=h["beta1"], beta2=h["beta2"], eps=f["eps"],
                               weight_decay=f["weight_decay"], step=1)
    d = ao.adamw_direction(m1, v1, h["beta1"], h["beta2"], f["eps"], 1)
    assert np.allclose(d, f["direction"], rtol=0, atol=1e-15)
    assert np.allclose(p1, f["p1"], rtol=0, atol=1e-15)


@pytest.mark.parametrize("beta1,beta2,eps", [(0.9, 0.999, 1e-8), (0.8, 0.95, 1e-3), (0.5, 0.75, 0.25)])
def test_first_step_is_normalised_gradient(beta1, beta2, eps):
    # t = 1: m_hat = g and v_hat = g^2 exactly, so the direction is g / (|g| + eps)
    g = np.random.default_rng(3).standard_normal(50)
    _, m, v = ao.adamw_step(np.zeros(50), g, np.zeros(50), np.zeros(50), lr=1.0, beta1=beta1, beta2=beta2,
                            eps=eps, weight_decay=0.0, step=1)
    assert np.allclose(ao.adamw_direction(m, v, beta1, beta2, eps, 1), g / (np.abs(g) + eps), rtol=1e-13, atol=0)


def test_constant_gradient_gives_the_same_step_every_time():
    # with bias correction m_hat = g and v_hat = g^2 at every step for a constant g
    g = np.array([0.3, -2.0, 1e-3, 5.0])
    lr, eps = 0.01, 1e-8
    p = np.zeros(4)
    m = np.zeros(4)
    v = np.zeros(4)
    for t in range(1, 11):
        p_new, m, v = ao.adamw_step(p, g, m, v, lr=lr, beta1=0.9, beta2=0.999, eps=eps, weight_decay=0.0, step=t)
        assert np.allclose(p - p_new, lr * g / (np.abs(g) + eps), rtol=1e-12, atol=0)
        p = p_new


def test_decay_only_when_gradient_is_zero():
    p0 = np.array([1.0, -3.0, 0.5])
    p = p0.copy()
    m = np.zeros(3)
    v = np.zeros(3)
    for t in range(1, 4):
        p, m, v = ao.adamw_step(p, np.zeros(3), m, v, lr=0.1, beta1=0.9, beta2=0.999, eps=1e-8,
                                weight_decay=0.5, step=t)
    assert np.allclose(p, p0 * 0.95 ** 3, rtol=1e-15, atol=0)
    assert not m.any() and not v.any()


def test_direction_is_scale_invariant_without_eps():
    rng = np.random.default_rng(7)
    gs = [rng.standard_normal(20) for _ in range(4)]
    outs = []
    for c in (1.0, 1e3):
        m = np.zeros(20)
        v = np.zeros(20)
        for t, g in enumerate(gs, 1):
            m, v = ao.adamw_moments(m, v, c * g, 0.9, 0.99)
        outs.append(ao.adamw_direction(m, v, 0.9, 0.99, 0.0, len(gs)))
    assert np.allclose(outs[0], outs[1], rtol=1e-12, atol=0)


def test_eps_is_added_after_the_square_root():
    g = np.array([1e-12])
    _, m, v = ao.adamw_step(np.zeros(1), g, np.zeros(1), np.zeros(1), lr=1.0, beta1=0.9, beta2=0.999, eps=1e-8,
                            weight_decay=0.0, step=1)
    d = ao.adamw_direction(m, v, 0.9, 0.999, 1e-8, 1)
    assert np.allclose(d, 1e-12 / (1e-12 + 1e-8), rtol=1e-12)  # eps inside the root would give ~1e-8


def test_step_counts_from_one():
    with pytest.raises(ValueError):
        ao.adamw_step(np.zeros(1), np.zeros(1), np.zeros(1), np.zeros(1), lr=0.1, beta1=0.9, beta2=0.99,
                      eps=1e-8, weight_decay=0.0, step=0)
