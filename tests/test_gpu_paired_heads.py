"""Per-head and paired-head Muon: Q/K/V projections split into blocks of whole heads,
each block orthogonalised as its own matrix (strided views, no copies).

The pages name paired-head attention and a paired-head Muon record without a formula;
the reading taken is that every block of `heads_per_block` heads (rows of a Q/K/V
projection, columns of the output projection) is its own Newton-Schulz problem.  Parity:
the oracle applied to each block on its own; a grouped call over all blocks of several
matrices equals one call per block, bit for bit."""
import numpy as np
import pytest

import oracle
from newton_schulz_11_b200 import inputs
from tests.gpu_util import bf16_ulp, rel_fro, require_gpu, to_np, torch

pytestmark = pytest.mark.gpu
QUINTIC5 = [oracle.QUINTIC] * 5
D, HEAD = 768, 64


def _weights(seed):
    w = inputs.scaled_workload(inputs.WORKLOADS["gpt2-124m-72-matrices"], [(D, D)] * 3)
    W = [torch.from_numpy(inputs.weight_np(w, i)).cuda().to(torch.bfloat16) for i in range(3)]
    G = [torch.from_numpy(inputs.grad_np(w, 1 + seed, i)).cuda() for i in range(3)]
    M = [torch.from_numpy(inputs.grad_np(w, 0, i)).cuda() for i in range(3)]
    return W, G, M


@pytest.mark.parametrize("heads_per_block", [1, 2])
def test_head_blocks_match_the_oracle_per_block(heads_per_block):
    require_gpu()
    from newton_schulz_11_b200 import api

    W, G, M = _weights(0)
    W_in = [to_np(w.float()) for w in W]
    M_in = [to_np(m) for m in M]
    blocks = []  # (param view, grad view, momentum view, dim)
    for i, dim in enumerate((0, 0, 1)):  # Q and K split by rows, the output projection by columns
        for p, g, m in zip(api.head_blocks(W[i], HEAD, heads_per_block, dim),
                           api.head_blocks(G[i], HEAD, heads_per_block, dim),
                           api.head_blocks(M[i], HEAD, heads_per_block, dim)):
            blocks.append((p, g, m, dim))
    outs = [torch.empty(g.shape, device="cuda") for _, g, _, _ in blocks]
    api.muon_step([b[0] for b in blocks], [b[1] for b in blocks], [b[2] for b in blocks], lr=0.02,
                  weight_decay=0.01, outs=outs)
    torch.cuda.synchronize()
    size = HEAD * heads_per_block
    k = 0
    for i, dim in enumerate((0, 0, 1)):
        for j in range(D // size):
            sl = (slice(j * size, (j + 1) * size), slice(None)) if dim == 0 else (slice(None), slice(j * size, (j + 1) * size))
            g = to_np(G[i])[sl].astype(np.float64)
            _, m_ref, O_ref = oracle.muon_step(W_in[i][sl].astype(np.float64), g, M_in[i][sl].astype(np.float64),
                                               lr=0.02, beta=0.95, weight_decay=0.01, nesterov=True, coeffs=QUINTIC5)
            O_gpu = to_np(outs[k])
            assert rel_fro(O_gpu, O_ref) <= 2e-2, (i, j)
            assert rel_fro(to_np(M[i])[sl], m_ref) <= 1e-6, (i, j)
            # W of the block: within one bf16 ulp of the oracle's update of the GPU's own O,
            # plus the fp32 evaluation error (see check_bf16_update in the parity tests)
            r, c = O_gpu.shape
            scale = oracle.default_shape_scale(r, c)
            W_exp = oracle.parameter_update(W_in[i][sl].astype(np.float64), O_gpu, 0.02, 0.01, scale)
            bound = bf16_ulp(W_exp) + 2.0 ** -23 * (np.abs(W_in[i][sl]) + 0.02 * scale * np.abs(O_gpu))
            assert (np.abs(to_np(W[i].float())[sl] - W_exp) <= bound).all(), (i, j)
            k += 1


def test_grouped_blocks_equal_one_call_per_block():
    require_gpu()
    from newton_schulz_11_b200 import api

    W1, G, M1 = _weights(1)
    W2 = [w.clone() for w in W1]
    M2 = [m.clone() for m in M1]
    def blocks(W, M):
        out = []
        for i, dim in enumerate((0, 0, 1)):
            out += list(zip(api.head_blocks(W[i], HEAD, 2, dim), api.head_blocks(G[i], HEAD, 2, dim),
                            api.head_blocks(M[i], HEAD, 2, dim)))
        return out
    b1 = blocks(W1, M1)
    api.muon_step([b[0] for b in b1], [b[1] for b in b1], [b[2] for b in b1], lr=0.02)
    for p, g, m in blocks(W2, M2):
        api.muon_step([p], [g], [m], lr=0.02)
    torch.cuda.synchronize()
    for a, b in zip(W1 + M1, W2 + M2):
        assert torch.equal(a, b)
