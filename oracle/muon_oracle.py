"""Plain fp64 CPU oracle for the Muon optimizer step.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this module:
only the tests, the smoke check and the CPU-baseline leg of the benchmark
call it.  It shares no code with the CUDA library; the two meet only through
the seeded inputs both are fed.

Everything is float64 numpy with no bf16 rounding anywhere, written to be
checked against the pages by eye:

* Momentum and update rule -- "14 -- modded-nanogpt: the Speedrun Community",
  section 3 "Muon -- the optimizer that started the modern speedrun era",
  the ``muon_step`` pseudocode under "The one-line version": the buffer is
  ``beta * momentum + grad``, it is orthogonalised with five Newton-Schulz
  iterations, and the parameter moves by ``-lr`` times the result.
* Nesterov -- "NanoGPT Speedrun" (README mirror), the list of practices after
  the Newton-Schulz listing: Nesterov momentum is used inside the update and
  the orthogonalisation is applied after the momentum.  The page's own
  formula for the full update was lost, so the reading taken is
  ``u = g + beta * m_new`` with ``m_new = beta * m + g`` (plain momentum
  gives ``u = m_new``).
* Newton-Schulz -- "NanoGPT Speedrun" (README mirror), the
  ``zeroth_power_via_newtonschulz5`` listing under "Muon is defined as
  follows": divide by the Frobenius norm plus eps, put the short side on
  the rows, iterate ``A = X X^T``, ``B = b A + c A A``, ``X = a X + B X``
  with the quintic coefficients (3.4445, -4.7750, 2.0315), undo the
  transpose.  The table form (one (a, b, c) row per iteration) also covers
  the per-iteration schedules named on the same page ("Polar Express
  implementation in Muon").
* Weight decay and shape scale -- the record titles on the same page name
  "standard weight decay" and "Muon custom sizing" without formulas; the
  reading is decoupled decay ``W (1 - lr wd)`` taken from the old W and a
  per-matrix factor ``sqrt(max(1, rows / cols))`` on the orthogonalised
  update.

Pinned (tests/test_oracle_pins.py) by: the SVD closed form of the iteration,
the classical cubic iteration's convergence to the polar factor, the band
the page states for the quintic, hand-worked momentum recurrences, exact
invariances and tiny hand-checkable inputs.
"""
from __future__ import annotations

import math
from typing import Optional, Sequence, Tuple

import numpy as np

# "NanoGPT Speedrun", zeroth_power_via_newtonschulz5 listing: (a, b, c) and eps.
QUINTIC = (3.4445, -4.7750, 2.0315)
NS_EPS = 1e-7


def momentum_update(m: np.ndarray, g: np.ndarray, beta: float) -> np.ndarray:
    """m <- beta * m + g  ("14 -- modded-nanogpt", section 3, muon_step pseudocode)."""
    return beta * np.asarray(m, np.float64) + np.asarray(g, np.float64)


def nesterov_input(g: np.ndarray, m_new: np.ndarray, beta: float, nesterov: bool) -> np.ndarray:
    """The matrix handed to Newton-Schulz ("NanoGPT Speedrun", list of practices).

    Nesterov: u = g + beta * m_new; otherwise u = m_new.
    """
    g = np.asarray(g, np.float64)
    m_new = np.asarray(m_new, np.float64)
    return g + beta * m_new if nesterov else m_new


def frobenius_norm(u: np.ndarray) -> float:
    """sqrt of the sum of squares: the ``G.norm()`` of the listing."""
    u = np.asarray(u, np.float64)
    return float(np.sqrt(np.sum(u * u)))


def gram(X: np.ndarray) -> np.ndarray:
    """A = X X^T (listing, first line of the loop body)."""
    return X @ X.T


def polynomial(A: np.ndarray, b: float, c: float) -> np.ndarray:
    """B = b A + c A A (listing, second line of the loop body)."""
    return b * A + c * (A @ A)


def apply_step(X: np.ndarray, B: np.ndarray, a: float) -> np.ndarray:
    """X <- a X + B X (listing, third line of the loop body)."""
    return a * X + B @ X


def newton_schulz(G: np.ndarray, coeffs: Sequence[Sequence[float]], eps: float = NS_EPS) -> np.ndarray:
    """zeroth_power_via_newtonschulz5 in fp64 with a per-iteration coefficient table.

    ``coeffs`` holds one (a, b, c) row per iteration; five rows of QUINTIC is
    the page's default.  The transpose rule follows the listing: only a
    matrix with more rows than columns is transposed.
    """
    G = np.asarray(G, np.float64)
    if G.ndim != 2:
        raise ValueError("Newton-Schulz is defined for 2-D matrices only")
    X = G / (frobenius_norm(G) + eps)
    tall = G.shape[0] > G.shape[1]
    if tall:
        X = X.T
    for a, b, c in coeffs:
        A = gram(X)
        B = polynomial(A, b, c)
        X = apply_step(X, B, a)
    if tall:
        X = X.T
    return X


def default_shape_scale(rows: int, cols: int) -> float:
    """sqrt(max(1, rows / cols)): 1 for wide and square matrices, > 1 for tall ones."""
    return math.sqrt(max(1.0, rows / cols))


def parameter_update(W: np.ndarray, O: np.ndarray, lr: float, weight_decay: float,
                     shape_scale: float) -> np.ndarray:
    """W <- W (1 - lr wd) - lr * shape_scale * O  (decoupled decay from the old W)."""
    W = np.asarray(W, np.float64)
    O = np.asarray(O, np.float64)
    return W * (1.0 - lr * weight_decay) - (lr * shape_scale) * O


def muon_step(W: np.ndarray, g: np.ndarray, m: np.ndarray, *, lr: float, beta: float,
              weight_decay: float, nesterov: bool, coeffs: Sequence[Sequence[float]],
              shape_scale: Optional[float] = None, eps: float = NS_EPS
              ) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """One Muon step on one matrix.  Returns (W_new, m_new, O), all fp64.

    Order of operations as on the pages: momentum, Nesterov input,
    Newton-Schulz on that input, then the parameter update.
    """
    rows, cols = np.shape(g)
    m_new = momentum_update(m, g, beta)
    u = nesterov_input(g, m_new, beta, nesterov)
    O = newton_schulz(u, coeffs, eps)
    scale = default_shape_scale(rows, cols) if shape_scale is None else float(shape_scale)
    W_new = parameter_update(W, O, lr, weight_decay, scale)
    return W_new, m_new, O

