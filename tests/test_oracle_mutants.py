"""Plant plausible mistakes in the oracle (on the CPU) and check that the pins catch each.

Each mutant swaps one step of the oracle for a wrong variant (a transposed
operand, a flipped sign, a dropped term, eps in the wrong place, a wrong
recurrence) and re-runs the closed-form and hand-worked checks against it.
"""
import math

import numpy as np
import pytest

import oracle
import oracle.muon_oracle as mo
from tests.conftest import load_golden
from tests.test_oracle_pins import QUINTIC5, closed_form_ns, rel


def _ns_pin_fails():
    rng = np.random.default_rng(2024)
    for shape in [(10, 10), (10, 18), (18, 10)]:
        G = rng.standard_normal(shape)
        G[:3] *= 20
        try:
            O = mo.newton_schulz(G, QUINTIC5, 1e-7)
        except ValueError:
            return True
        if O.shape != G.shape or rel(O, closed_form_ns(G, QUINTIC5, 1e-7)) > 1e-8:
            return True
    G = np.array([[3e-8, 4e-8]])
    x = 5e-8 / (5e-8 + 1e-7)
    y = x
    for a, b, c in QUINTIC5:
        y = a * y + b * y ** 3 + c * y ** 5
    return rel(mo.newton_schulz(G, QUINTIC5, 1e-7), y * np.array([[0.6, 0.8]])) > 1e-10


def _momentum_pin_fails():
    h = load_golden("momentum_handworked.json")["sequence"]
    m = np.array(h["m0"], np.float64)
    for g, m_exp, u_exp in zip(h["grads"], h["momentum"], h["nesterov_u"]):
        g = np.array(g, np.float64)
        m = mo.momentum_update(m, g, h["beta"])
        u = mo.nesterov_input(g, m, h["beta"], True)
        if not (np.array_equal(m, np.array(m_exp)) and np.array_equal(u, np.array(u_exp))):
            return True
    return False


def _update_pin_fails():
    h = load_golden("momentum_handworked.json")["decay_only"]
    W = np.array(h["W"], np.float64)
    W1, _, _ = mo.muon_step(W, np.zeros_like(W), np.zeros_like(W), lr=h["lr"], beta=0.95,
                            weight_decay=h["weight_decay"], nesterov=True, coeffs=QUINTIC5)
    if not np.allclose(W1, np.array(h["W_new"]), rtol=0, atol=1e-15):
        return True
    rng = np.random.default_rng(11)
    W = rng.standard_normal((12, 20))
    g = rng.standard_normal((12, 20))
    W1, _, _ = mo.muon_step(W, g, np.zeros_like(g), lr=0.1, beta=0.9, weight_decay=0.0,
                            nesterov=False, coeffs=QUINTIC5)
    return float(np.sum((W1 - W) * g)) >= 0


def _mut_gram(X):
    return X.T @ X


def _mut_poly_sign(A, b, c):
    return -b * A + c * (A @ A)


def _mut_poly_drop(A, b, c):
    return b * A


def _mut_apply_order(X, B, a):
    return a * X + X @ B if X.shape[0] == X.shape[1] else a * X + B @ X * 0.5


def _mut_apply_drop_a(X, B, a):
    return X + B @ X


def _mut_norm_sq_eps(u):
    u = np.asarray(u, np.float64)
    return float(np.sqrt(np.sum(u * u) + 1e-7)) - 1e-7


def _mut_momentum(m, g, beta):
    return beta * (np.asarray(m, np.float64) + np.asarray(g, np.float64))


def _mut_nesterov(g, m_new, beta, nesterov):
    return np.asarray(m_new, np.float64)


def _mut_update(W, O, lr, wd, s):
    return np.asarray(W) * (1 - wd) - lr * s * np.asarray(O)


def _mut_update_sign(W, O, lr, wd, s):
    return np.asarray(W) * (1 - lr * wd) + lr * s * np.asarray(O)


MUTANTS = [
    ("gram", _mut_gram, _ns_pin_fails),
    ("polynomial", _mut_poly_sign, _ns_pin_fails),
    ("polynomial", _mut_poly_drop, _ns_pin_fails),
    ("apply_step", _mut_apply_order, _ns_pin_fails),
    ("apply_step", _mut_apply_drop_a, _ns_pin_fails),
    ("frobenius_norm", _mut_norm_sq_eps, _ns_pin_fails),
    ("momentum_update", _mut_momentum, _momentum_pin_fails),
    ("nesterov_input", _mut_nesterov, _momentum_pin_fails),
    ("parameter_update", _mut_update, _update_pin_fails),
    ("parameter_update", _mut_update_sign, _update_pin_fails),
]


def test_unmutated_oracle_passes_every_detector():
    assert not _ns_pin_fails()
    assert not _momentum_pin_fails()
    assert not _update_pin_fails()


@pytest.mark.parametrize("name,mutant,detector", MUTANTS,
                         ids=[f"{n}-{m.__name__}" for n, m, _ in MUTANTS])
def test_planted_mistake_is_caught(monkeypatch, name, mutant, detector):
    monkeypatch.setattr(mo, name, mutant)
    with np.errstate(over="ignore", invalid="ignore"):  # a wrong iteration may diverge
        caught = detector()
    assert caught, f"mutant {mutant.__name__} of {name} slipped through the pins"


# ------------------------------------------------------------------ AdamW oracle

import oracle.adamw_oracle as ao  # noqa: E402


def _adamw_pins_fail():
    h = load_golden("adamw_handworked.json")
    m = np.zeros(3)
    v = np.zeros(3)
    for g, m_exp, v_exp in zip(h["grads"], h["m"], h["v"]):
        m, v = ao.adamw_moments(m, v, np.array(g), h["beta1"], h["beta2"])
        if not (np.array_equal(m, np.array(m_exp)) and np.array_equal(v, np.array(v_exp))):
            return True
    f = h["first_step"]
    p1, _, _ = ao.adamw_step(np.array(f["p0"]), np.array(h["grads"][0]), np.zeros(3), np.zeros(3), lr=f["lr"],
                             beta1=h["beta1"], beta2=h["beta2"], eps=f["eps"], weight_decay=f["weight_decay"],
                             step=1)
    if not np.allclose(p1, f["p1"], rtol=0, atol=1e-15):
        return True
    g = np.array([0.3, -2.0, 1e-3, 5.0])
    p = np.zeros(4)
    m = np.zeros(4)
    v = np.zeros(4)
    for t in range(1, 6):
        p_new, m, v = ao.adamw_step(p, g, m, v, lr=0.01, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.0, step=t)
        if not np.allclose(p - p_new, 0.01 * g / (np.abs(g) + 1e-8), rtol=1e-12, atol=0):
            return True
        p = p_new
    p0 = np.array([1.0, -3.0, 0.5])
    p, _, _ = ao.adamw_step(p0, np.zeros(3), np.zeros(3), np.zeros(3), lr=0.1, beta1=0.9, beta2=0.999, eps=1e-8,
                            weight_decay=0.5, step=1)
    if not np.allclose(p, 0.95 * p0, rtol=1e-15, atol=0):
        return True
    _, m, v = ao.adamw_step(np.zeros(1), np.array([1e-12]), np.zeros(1), np.zeros(1), lr=1.0, beta1=0.9,
                            beta2=0.999, eps=1e-8, weight_decay=0.0, step=1)
    return not np.allclose(ao.adamw_direction(m, v, 0.9, 0.999, 1e-8, 1), 1e-12 / (1e-12 + 1e-8), rtol=1e-12)


def _mut_adam_swapped_betas(m, v, g, beta1, beta2):
    g = np.asarray(g, np.float64)
    return beta2 * m + (1 - beta2) * g, beta1 * v + (1 - beta1) * g * g


def _mut_adam_abs_second_moment(m, v, g, beta1, beta2):
    g = np.asarray(g, np.float64)
    return beta1 * m + (1 - beta1) * g, beta2 * v + (1 - beta2) * np.abs(g)


def _mut_adam_no_bias_correction(m, v, beta1, beta2, eps, step):
    return m / (np.sqrt(v) + eps)


def _mut_adam_eps_in_root(m, v, beta1, beta2, eps, step):
    return (m / (1 - beta1 ** step)) / np.sqrt(v / (1 - beta2 ** step) + eps)


def _mut_adam_decay_new_p(p, g, m, v, *, lr, beta1, beta2, eps, weight_decay, step):
    m1, v1 = ao.adamw_moments(m, v, g, beta1, beta2)
    return (p - lr * ao.adamw_direction(m1, v1, beta1, beta2, eps, step)) * (1 - lr * weight_decay), m1, v1


def _mut_adam_decay_without_lr(p, g, m, v, *, lr, beta1, beta2, eps, weight_decay, step):
    m1, v1 = ao.adamw_moments(m, v, g, beta1, beta2)
    return p * (1 - weight_decay) - lr * ao.adamw_direction(m1, v1, beta1, beta2, eps, step), m1, v1


ADAMW_MUTANTS = [
    ("adamw_moments", _mut_adam_swapped_betas),
    ("adamw_moments", _mut_adam_abs_second_moment),
    ("adamw_direction", _mut_adam_no_bias_correction),
    ("adamw_direction", _mut_adam_eps_in_root),
    ("adamw_step", _mut_adam_decay_new_p),
    ("adamw_step", _mut_adam_decay_without_lr),
]


def test_unmutated_adamw_oracle_passes_its_pins():
    assert not _adamw_pins_fail()


@pytest.mark.parametrize("name,mutant", ADAMW_MUTANTS, ids=[f"{n}-{m.__name__}" for n, m in ADAMW_MUTANTS])
def test_planted_adamw_mistake_is_caught(monkeypatch, name, mutant):
    monkeypatch.setattr(ao, name, mutant)
    assert _adamw_pins_fail(), f"mutant {mutant.__name__} of {name} slipped through the pins"
