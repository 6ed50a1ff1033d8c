"""Data-parallel sharded Muon on two gloo ranks (CPU).  The local step is the fp64 oracle
applied to the owned matrices, so what is tested is the host logic: the owner assignment,
the per-owner broadcast plan, and that every rank ends with the parameters a single
process computes, while each momentum buffer changes only on its owner."""
import json
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SHAPES = [(48, 32), (32, 80), (64, 64), (16, 24), (40, 40), (24, 56), (8, 8)]
HYPER = dict(lr=0.02, beta=0.95, weight_decay=0.01, nesterov=True)


def _inputs():
    rng = np.random.default_rng(0)
    W = [rng.standard_normal(s).astype(np.float32) * 0.02 for s in SHAPES]
    G = [rng.standard_normal(s).astype(np.float32) for s in SHAPES]
    M = [rng.standard_normal(s).astype(np.float32) for s in SHAPES]
    return W, G, M


def test_lpt_partition_balances_and_is_deterministic():
    sys.path.insert(0, ROOT)
    from newton_schulz_11_b200.distributed import ns_flops, partition_lpt

    costs = [ns_flops(*s) for s in SHAPES]
    own = partition_lpt(costs, 3)
    assert own == partition_lpt(costs, 3)
    loads = [sum(c for c, o in zip(costs, own) if o == r) for r in range(3)]
    assert max(loads) <= sum(costs) / 3 + max(costs)  # the LPT bound
    assert partition_lpt(costs, 1) == [0] * len(costs)
    assert sorted(set(partition_lpt([1.0] * 5, 5))) == [0, 1, 2, 3, 4]


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch.distributed as dist

    import oracle
    from newton_schulz_11_b200.distributed import ShardedMuon

    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        W, G, M = _inputs()
        params = [torch.from_numpy(w.copy()) for w in W]
        grads = [torch.from_numpy(g) for g in G]
        moms = [torch.from_numpy(m.copy()) for m in M]

        def local_step(idx):
            for i in idx:
                W1, m1, _ = oracle.muon_step(params[i].double().numpy(), grads[i].double().numpy(),
                                             moms[i].double().numpy(), coeffs=[oracle.QUINTIC] * 5, **HYPER)
                params[i].copy_(torch.from_numpy(W1))
                moms[i].copy_(torch.from_numpy(m1))

        step = ShardedMuon(params, grads, moms, local_step=local_step)
        step()
        step()
        res = {"owners": step.owners, "params": [p.tolist() for p in params],
               "mom_changed": [bool((m.numpy() != m0).any()) for m, m0 in zip(moms, M)]}
    finally:
        dist.destroy_process_group()
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump(res, f)


@pytest.mark.parametrize("world", [2, 3])
def test_sharded_step_matches_single_process(tmp_path, world):
    sys.path.insert(0, ROOT)
    import oracle

    port = _free_port()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, str(tmp_path))) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=240)
    for p in procs:
        if p.is_alive():
            p.kill()
            pytest.fail("a rank did not finish")
        assert p.exitcode == 0
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    # single-process reference: two steps of every matrix
    W, G, M = _inputs()
    for i in range(len(SHAPES)):
        w, m = W[i].astype(np.float64), M[i].astype(np.float64)
        for _ in range(2):
            w, m, _ = oracle.muon_step(np.float32(w).astype(np.float64), G[i].astype(np.float64),
                                       np.float32(m).astype(np.float64), coeffs=[oracle.QUINTIC] * 5, **HYPER)
        for r in range(world):
            assert np.allclose(np.array(res[r]["params"][i]), np.float32(w), rtol=0, atol=1e-6), (i, r)
    owners = res[0]["owners"]
    assert all(x["owners"] == owners for x in res)
    assert set(owners) == set(range(world))
    for r in range(world):
        for i, o in enumerate(owners):
            assert res[r]["mom_changed"][i] == (o == r)
