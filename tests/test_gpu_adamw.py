"""AdamW kernel against the fp64 oracle on the same seeded inputs (GPU, through the C ABI).

Tolerances, from the fp32 arithmetic of one step (each side continues from the GPU's
previous m, v, p, so rounding does not accumulate):
  m, v   per element, four roundings of 2^-24 of the magnitudes of the two terms
         (beta m and (1 - beta) g, or beta v and (1 - beta) g^2) -- relative to m itself
         this is unbounded where the terms cancel, so the bound is on the terms
  p fp32 1e-6 relative (Frobenius)
  p bf16 one bf16 ulp of the fp64 result plus the fp32 evaluation error of
         p (1 - lr wd) - step m / denom (two roundings of 2^-24 of the operands)"""
import numpy as np
import pytest

from oracle import adamw_oracle as ao
from tests.gpu_util import require_gpu, torch

pytestmark = pytest.mark.gpu

# the C ABI takes fp32 hyperparameters: the oracle gets the same (fp32-rounded) values,
# e.g. beta1 = fp32(0.9), whose 1 - beta1 differs from 0.1 by 2.4e-7 relative
HYPER = {k: float(np.float32(v)) for k, v in dict(lr=1e-3, beta1=0.9, beta2=0.95, eps=1e-8,
                                                   weight_decay=0.1).items()}


def bf16_round(x):
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16).float().numpy().astype(np.float64)


def bf16_ulp(x):
    x = np.abs(np.asarray(x, np.float64))
    e = np.floor(np.log2(np.maximum(x, 2.0 ** -126)))
    return 2.0 ** (e - 7)


def run_case(sizes, dtype, steps, offset=0, seed=0):
    require_gpu()
    from newton_schulz_11_b200 import api

    rng = np.random.default_rng(seed)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    P, G, M, V = [], [], [], []
    P_ref, M_ref, V_ref = [], [], []
    for n in sizes:
        p0 = (0.02 * rng.standard_normal(n)).astype(np.float32)
        if dtype == "bf16":
            p0 = bf16_round(p0).astype(np.float32)
        # a view starting `offset` elements into a buffer: 0 keeps the 32-byte alignment of
        # the allocation (256-bit path), 4 leaves 16 bytes (128-bit path), 1 none (scalar)
        buf = torch.zeros(n + offset, dtype=tdt, device="cuda")
        P.append(buf[offset:])
        P[-1].copy_(torch.from_numpy(p0).to(tdt))
        M.append(torch.zeros(n + offset, device="cuda")[offset:])
        V.append(torch.zeros(n + offset, device="cuda")[offset:])
        P_ref.append(p0.astype(np.float64))
        M_ref.append(np.zeros(n))
        V_ref.append(np.zeros(n))
    for t in range(1, steps + 1):
        G = []
        gs = []
        for n in sizes:
            g = (1e-2 * rng.standard_normal(n)).astype(np.float32)
            g[::7] *= 50  # a spread of magnitudes
            gs.append(g)
            G.append(torch.from_numpy(g).cuda())
        p_in = [x.copy() for x in P_ref]
        m_prev = [x.copy() for x in M_ref]
        v_prev = [x.copy() for x in V_ref]
        if dtype == "bf16":
            p_in = [p.float().cpu().numpy().astype(np.float64) for p in P]
        api.adamw_step(P, G, M, V, lr=HYPER["lr"], step=t, betas=(HYPER["beta1"], HYPER["beta2"]),
                       eps=HYPER["eps"], weight_decay=HYPER["weight_decay"])
        torch.cuda.synchronize()
        for i in range(len(sizes)):
            p_new, M_ref[i], V_ref[i] = ao.adamw_step(p_in[i], gs[i].astype(np.float64), M_ref[i], V_ref[i],
                                                      step=t, **HYPER)
            m_gpu = M[i].double().cpu().numpy()
            v_gpu = V[i].double().cpu().numpy()
            p_gpu = P[i].double().cpu().numpy()
            g64 = gs[i].astype(np.float64)
            b1, b2 = HYPER["beta1"], HYPER["beta2"]
            tol_m = 4 * 2.0 ** -24 * (b1 * np.abs(m_prev[i]) + (1 - b1) * np.abs(g64)) + 1e-30
            tol_v = 4 * 2.0 ** -24 * (b2 * v_prev[i] + (1 - b2) * g64 * g64) + 1e-30
            assert (np.abs(m_gpu - M_ref[i]) <= tol_m).all(), (i, t)
            assert (np.abs(v_gpu - V_ref[i]) <= tol_v).all(), (i, t)
            if dtype == "f32":
                assert np.linalg.norm(p_gpu - p_new) <= 1e-6 * np.linalg.norm(p_new), (i, t)
                P_ref[i] = p_gpu  # continue from the GPU's parameter
            else:
                d = np.abs(p_gpu - p_new)
                step_size = HYPER["lr"] / (1 - HYPER["beta1"] ** t)
                bound = bf16_ulp(p_new) + 2.0 ** -23 * (np.abs(p_in[i]) + step_size * 1.01)
                assert (d <= bound).all(), (i, t, d.max())
            # the moments continue from the GPU's values, so rounding does not accumulate
            M_ref[i], V_ref[i] = m_gpu, v_gpu


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_adamw_matches_oracle_over_three_steps(dtype):
    run_case([1, 3, 4, 17, 16384, 16385, 100003], dtype, steps=3)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_adamw_unaligned_views_take_the_scalar_path(dtype):
    run_case([5, 4099, 70001], dtype, steps=2, offset=1, seed=1)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_adamw_16_byte_views_take_the_128_bit_path(dtype):
    run_case([5, 4099, 70001], dtype, steps=2, offset=4, seed=3)


def test_adamw_many_tensors_split_over_launches():
    # more than one launch's worth of tensors (128 per launch)
    run_case([7 + (i % 5) for i in range(300)], "f32", steps=2, seed=2)
