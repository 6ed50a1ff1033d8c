"""Per-iteration Newton-Schulz coefficient tables.

The README's technique list names a "Polar Express implementation in Muon" (and the
GPT-2-medium track "tuned Muon Newton-Schulz coefficients") without printing the
values.  The schedule shipped here is derived in this file, in float64, by the
greedy rule that name refers to (Amsel, Persson, Musco, Gower, "The Polar Express",
2025): at step k, with every normalised singular value known to lie in [lo_k, hi_k],
take the odd quintic p(x) = a x + b x^3 + c x^5 that minimises
max |1 - p(x)| over [lo_k, hi_k] (a linear program on a dense grid), then move to
the interval p maps [lo_k, hi_k] onto.  Every step but the last is evaluated at
x / 1.01, so that singular values pushed slightly above hi_k by rounding are not
amplified.  Starting interval: [1e-3, 1].

    python -m newton_schulz_11_b200.schedules     # re-derives and rewrites data/polar5.json

The table is an input of the step like the fixed quintic: the CUDA path and the
oracle both take it as given.
"""
from __future__ import annotations

import json
import os
from typing import List, Tuple

import numpy as np

DATA = os.path.join(os.path.dirname(os.path.abspath(__file__)), "data")

Row = Tuple[float, float, float]


def _grid(lo: float, hi: float, n: int = 3001) -> np.ndarray:
    return np.unique(np.concatenate([np.geomspace(lo, hi, n), np.linspace(lo, hi, n)]))


def poly(row: Row, x: np.ndarray) -> np.ndarray:
    a, b, c = row
    return a * x + b * x ** 3 + c * x ** 5


def minimax_odd_quintic(lo: float, hi: float) -> Tuple[Row, float]:
    """argmin over (a, b, c) of max_{x in [lo, hi]} |1 - (a x + b x^3 + c x^5)|."""
    from scipy.optimize import linprog

    x = _grid(lo, hi)
    V = np.stack([x, x ** 3, x ** 5], axis=1)
    ones = np.ones((len(x), 1))
    # variables (a, b, c, t): minimise t with  p(x) - 1 <= t  and  1 - p(x) <= t
    A_ub = np.vstack([np.hstack([V, -ones]), np.hstack([-V, -ones])])
    b_ub = np.concatenate([np.ones(len(x)), -np.ones(len(x))])
    res = linprog(c=[0, 0, 0, 1], A_ub=A_ub, b_ub=b_ub, bounds=[(None, None)] * 3 + [(0, None)],
                  method="highs")
    if not res.success:
        raise RuntimeError(f"minimax LP failed on [{lo}, {hi}]: {res.message}")
    a, b, c, t = res.x
    return (float(a), float(b), float(c)), float(t)


def derive(steps: int = 5, lo: float = 1e-3, hi: float = 1.0, safety: float = 1.01) -> List[Row]:
    table: List[Row] = []
    for k in range(steps):
        (a, b, c), _ = minimax_odd_quintic(lo, hi)
        if k + 1 < steps:
            a, b, c = a / safety, b / safety ** 3, c / safety ** 5
        row = (a, b, c)
        x = _grid(lo, hi)
        y = poly(row, x)
        lo, hi = float(y.min()), float(y.max())
        table.append(row)
    return table


def image_of_interval(table: List[Row], lo: float = 1e-3, hi: float = 1.0, n: int = 200001) -> Tuple[float, float]:
    """Range of the composed scalar map over [lo, hi] (dense sampling)."""
    x = np.linspace(lo, hi, n)
    for row in table:
        x = poly(row, x)
    return float(x.min()), float(x.max())


def load(name: str) -> List[Row]:
    with open(os.path.join(DATA, f"{name}.json")) as f:
        doc = json.load(f)
    return [tuple(float(v) for v in r) for r in doc["rows"]]


def write_polar5() -> str:
    rows = derive()
    lo, hi = image_of_interval(rows)
    doc = {
        "name": "polar5",
        "derivation": "greedy minimax odd quintic per step on the tracked interval, start [1e-3, 1], "
                      "safety 1.01 on all but the last step (newton_schulz_11_b200/schedules.py)",
        "rows": [list(r) for r in rows],
        "image_of_1e-3_to_1": [lo, hi],
    }
    os.makedirs(DATA, exist_ok=True)
    path = os.path.join(DATA, "polar5.json")
    with open(path, "w") as f:
        json.dump(doc, f, indent=1)
        f.write("\n")
    return path


if __name__ == "__main__":
    print(write_polar5())
    for r in load("polar5"):
        print(r)
    print("image of [1e-3, 1]:", image_of_interval(load("polar5")))
