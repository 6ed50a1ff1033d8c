"""The derived per-iteration (Polar-Express-style) table: reproducible and doing its job."""
import numpy as np
import pytest

import oracle
from newton_schulz_11_b200 import schedules


def test_table_is_reproducible_from_its_derivation():
    pytest.importorskip("scipy")
    stored = np.array(schedules.load("polar5"))
    again = np.array(schedules.derive())
    assert stored.shape == (5, 3)
    assert np.allclose(stored, again, rtol=1e-6, atol=1e-6)


def test_table_maps_the_start_interval_close_to_one():
    lo, hi = schedules.image_of_interval(schedules.load("polar5"))
    assert 0.85 < lo < 1.0 < hi < 1.15
    # tighter than five applications of the fixed quintic, which reach [0.68, 1.21]
    qlo, qhi = schedules.image_of_interval([oracle.QUINTIC] * 5, lo=1.6e-3)
    assert qlo < lo and qhi > hi


def test_oracle_with_table_lands_in_band():
    table = schedules.load("polar5")
    rng = np.random.default_rng(4)
    G = rng.standard_normal((48, 80))
    G[:4] *= 25
    O = oracle.newton_schulz(G, table)
    s_in = np.linalg.svd(G, compute_uv=False) / (np.linalg.norm(G) + 1e-7)
    s_out = np.linalg.svd(O, compute_uv=False)
    lo, hi = schedules.image_of_interval(table)
    keep = np.sort(s_out[s_in >= 1e-3])
    assert keep.min() >= lo - 1e-9 and keep.max() <= hi + 1e-9
