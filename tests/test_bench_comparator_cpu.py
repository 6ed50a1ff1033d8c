"""bench.py's plain-PyTorch comparator, run on the CPU: it must take the same step as the
oracle -- momentum to fp32 rounding, and the parameter change within the accuracy of an X
kept in bf16 (about 3% on these Gaussian inputs; a tall matrix's shape scale of sqrt(2)
left out would show as about 40%)."""
import dataclasses
import os
import sys

import numpy as np
import pytest

import oracle

torch = pytest.importorskip("torch")
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_torch_comparator_takes_the_oracles_step():
    sys.path.insert(0, ROOT)
    import bench
    from newton_schulz_11_b200 import inputs

    base = inputs.WORKLOADS["gpt2-124m-72-matrices"]
    w = dataclasses.replace(base, shapes=((48, 48), (48, 96), (96, 48), (48, 96)), name="small",
                            param_dtype="f32", weight_decay=0.1)
    rng = np.random.default_rng(3)
    gs = [rng.standard_normal(s).astype(np.float32) for s in w.shapes]
    ms = [rng.standard_normal(s).astype(np.float32) for s in w.shapes]
    Ws = [(0.02 * rng.standard_normal(s)).astype(np.float32) for s in w.shapes]
    coeffs = bench.load_coeffs(w)
    step, cls = bench.torch_comparator_step(w, [torch.from_numpy(x) for x in gs], [torch.from_numpy(x) for x in ms],
                                            [torch.from_numpy(x.copy()) for x in Ws], coeffs)
    step()
    # classes in order of first appearance: (48, 48): [0]; (48, 96): [1, 3]; (96, 48): [2]
    order = [[0], [1, 3], [2]]
    for (g_t, m_t, p_t, tall, scale), idx in zip(cls, order):
        for k, i in enumerate(idx):
            rows, cols = w.shapes[i]
            assert tall == (rows > cols)
            m_ref = oracle.momentum_update(ms[i].astype(np.float64), gs[i], w.beta)
            np.testing.assert_allclose(m_t[k].numpy(), m_ref, rtol=1e-6, atol=1e-6)
            u = oracle.nesterov_input(gs[i], m_ref, w.beta, w.nesterov)
            O = oracle.newton_schulz(u, coeffs)
            W_ref = oracle.parameter_update(Ws[i].astype(np.float64), O, w.lr, w.weight_decay,
                                        oracle.default_shape_scale(rows, cols))
            dW, dW_ref = p_t[k].numpy().astype(np.float64) - Ws[i], W_ref - Ws[i]
            err = np.linalg.norm(dW - dW_ref) / np.linalg.norm(dW_ref)
            print(w.shapes[i], f"{err:.3e}")
            assert err < 0.1, (w.shapes[i], err)
