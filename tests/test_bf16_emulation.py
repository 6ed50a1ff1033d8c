"""Why two GPU parity cases carry tolerances other than 2e-2, shown on the CPU.

tests/bf16_emulation.py models the CUDA path's rounding points (bf16 tensor-core operands
with fp32 accumulation, A and B stored in bf16, X carried as a bf16 hi plus an 8-bit
residual).  Against the fp64 oracle the model shows:

  * on the workloads' shapes the bf16 path sits one order of magnitude below the 2e-2 bar;
  * on rank-1 inputs (one side of the matrix is 1) most inputs exceed 2e-2 whatever the
    kernel does: Newton-Schulz is then a scalar recurrence x <- x (a + B) with
    B = b x^2 + c x^4 ~ -2.74 held in bf16 (half an ulp there is 0.0078, against a + B ~ 0.70),
    so one rounding of B moves the result by about 1.1% and five steps compound it;
  * the per-iteration polar5 table (first row a = 8.4, b = -24.4, c = 17.7) on the small,
    ill-conditioned 72 x 40 matrix exceeds 2e-2 as well, while the quintic does not.

The GPU tests use TOL_RANK1 for the rank-1 family and keep polar5 off the 72 x 40 matrix;
every other case keeps the 2e-2 bar.
"""
import numpy as np
import pytest

import oracle
from newton_schulz_11_b200 import inputs, schedules
from tests import bf16_emulation as em

TOL_O = 2e-2
TOL_RANK1 = 0.15  # the GPU parity tests' bound for the rank-1 family
QUINTIC5 = [oracle.QUINTIC] * 5


def rel_fro(a, b):
    return float(np.linalg.norm(np.asarray(a) - b) / np.linalg.norm(b))


def model_err(G, table):
    return rel_fro(em.newton_schulz(G, table), oracle.newton_schulz(np.asarray(G, np.float64), table))


def test_model_rounding_primitives():
    """bf16 rounding agrees with torch's conversion (ties to even included); the carried
    value of x keeps 15 significant bits, is exact when x has at most 15, and the residual
    never needs more than +-64 units of 2^9 ulps."""
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(5)
    x = (rng.standard_normal(20000) * np.exp2(rng.integers(-30, 30, 20000))).astype(np.float32)
    ties = (np.arange(1, 2001, dtype=np.float64) * 2.0 ** -8 + 2.0 ** -9 + 1.0).astype(np.float32)  # halfway
    for v in (x, ties, -ties):
        want = torch.from_numpy(v).to(torch.bfloat16).to(torch.float64).numpy()
        assert np.array_equal(em.bf16(v), want)
    hi, carried = em.carry(x)
    xd = x.astype(np.float64)
    assert np.all(np.abs(carried - xd) <= np.abs(xd) * 2.0 ** -15 + 1e-300)
    d = em._bits(carried) - em._bits(hi)
    assert np.all(d % 512 == 0) and np.all(np.abs(d // 512) <= 64)
    exact15 = np.float32(1.0) + np.arange(64, dtype=np.float32) * np.float32(2.0 ** -14)
    assert np.array_equal(em.carry(exact15)[1], exact15.astype(np.float64))


def test_model_is_exact_on_a_diagonal_of_powers_of_two():
    """Powers of two survive every rounding point, so on diag(1, 2^-1, ..., 2^-k) only the
    coefficients' fp32 rounding and the polynomial's bf16 rounding remain: the model must
    then follow the oracle to bf16 accuracy."""
    G = np.diag(np.exp2(-np.arange(6.0))).astype(np.float32)
    assert model_err(G, QUINTIC5) < 2e-2


def test_rank1_inputs_exceed_the_bar_for_any_bf16_operand_path():
    rng = np.random.default_rng(7)
    errs = []
    for _ in range(10000):
        n = int(rng.integers(1, 400))
        shape = (1, n) if rng.integers(2) else (n, 1)
        errs.append(model_err(rng.standard_normal(shape).astype(np.float32), QUINTIC5))
    errs = np.array(errs)
    print(f"rank-1, 10^4 inputs: max {errs.max():.4f}, median {np.median(errs):.4f}, "
          f"above 2e-2: {np.mean(errs > TOL_O):.2f}")
    assert np.mean(errs > TOL_O) > 0.5       # most rank-1 inputs miss the 2e-2 bar
    assert 0.06 < errs.max() < TOL_RANK1     # the worst case stays inside the GPU test's bound
    # the GPU test's own cases (same seeds)
    for shape in [(1, 24), (24, 1), (1, 1), (1, 300), (300, 1)]:
        G = np.random.default_rng(shape[0] * 7 + shape[1]).standard_normal(shape).astype(np.float32)
        assert model_err(G, QUINTIC5) < TOL_RANK1


def test_polar5_misses_the_bar_on_72x40_but_not_the_quintic():
    shapes = [(1088, 1088), (256, 128), (128, 384), (200, 136), (72, 40), (100, 37)]
    w = inputs.scaled_workload(inputs.WORKLOADS["gpt2-medium-144-matrices"], shapes)
    G = inputs.grad_np(w, 0, 4)  # the 72 x 40 matrix of the GPU test's mixed wave
    e_polar = model_err(G, schedules.load("polar5"))
    e_quintic = model_err(G, QUINTIC5)
    print(f"72 x 40: polar5 {e_polar:.3e}, quintic {e_quintic:.3e}")
    assert 2.5e-2 < e_polar < 4e-2
    assert e_quintic < 1e-2
    for i in (1, 2, 3):  # both sides >= 128: polar5 keeps the bar
        assert model_err(inputs.grad_np(w, 0, i), schedules.load("polar5")) < TOL_O / 2


def test_workload_shapes_sit_far_below_the_bar():
    w = inputs.WORKLOADS["single-256x128-f32"]
    g, m = inputs.grad_np(w, 0, 0), inputs.momentum_np(w, 0)
    u = oracle.nesterov_input(g, oracle.momentum_update(m.astype(np.float64), g, w.beta), w.beta, True)
    assert model_err(u.astype(np.float32), QUINTIC5) < 5e-3
    w = inputs.WORKLOADS["gpt2-124m-72-matrices"]
    for i in (0, 4, 5):  # 768 x 768, 768 x 3072, 3072 x 768
        e = model_err(inputs.grad_np(w, 1, i), QUINTIC5)
        print(f"{w.shapes[i]}: {e:.3e}")
        assert e < 2e-3
