"""Data-parallel sharded Muon on gloo ranks (CPU).  The local step is the fp64 oracle
applied to the owned matrices, so what is tested is the host logic: the owner and wave
assignment, the gradient reduction onto the owners, the per-owner broadcast plan, and that
every rank ends with the parameters a single process computes, while each momentum buffer
changes only on its owner and the caller's gradients are never written."""
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


def _local_grads(G, rank, world):
    """Rank-local gradients whose mean over the ranks is G (up to fp32 rounding)."""
    rng = np.random.default_rng(100 + rank)
    return [(g + np.float32(rank - (world - 1) / 2) * rng.standard_normal(g.shape).astype(np.float32)
             * np.float32(0.5)).astype(np.float32) if world > 1 else g for g in G]


def test_wave_assignment_balances_each_owner():
    sys.path.insert(0, ROOT)
    from newton_schulz_11_b200.distributed import assign_waves, ns_flops, partition_lpt

    costs = [ns_flops(*s) for s in SHAPES]
    own = partition_lpt(costs, 2)
    wave = assign_waves(costs, own, 2)
    for r in range(2):
        mine = sorted((i for i in range(len(SHAPES)) if own[i] == r), key=lambda k: (-costs[k], k))
        assert [wave[i] for i in mine] == [k % 2 for k in range(len(mine))]
    assert assign_waves(costs, own, 1) == [0] * len(SHAPES)
    with pytest.raises(ValueError):
        assign_waves(costs, own, 0)


def _rank_main(rank, world, port, out_dir, reduce_grads=False, waves=1):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch.distributed as dist

    import oracle
    from newton_schulz_11_b200.distributed import ShardedMuon

    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        W, G, M = _inputs()
        if reduce_grads:
            G = _local_grads(G, rank, world)
        params = [torch.from_numpy(w.copy()) for w in W]
        grads = [torch.from_numpy(g.copy()) for g in G]
        moms = [torch.from_numpy(m.copy()) for m in M]
        calls = []

        def local_step(idx, gs):
            calls.append(list(idx))
            for i, g in zip(idx, gs):
                W1, m1, _ = oracle.muon_step(params[i].double().numpy(), g.double().numpy(),
                                             moms[i].double().numpy(), coeffs=[oracle.QUINTIC] * 5, **HYPER)
                params[i].copy_(torch.from_numpy(W1))
                moms[i].copy_(torch.from_numpy(m1))

        step = ShardedMuon(params, grads, moms, local_step=local_step, reduce_grads=reduce_grads, waves=waves)
        step()
        step()
        res = {"owners": step.owners, "waves": step.wave_of, "calls": calls, "params": [p.tolist() for p in params],
               "mom_changed": [bool((m.numpy() != m0).any()) for m, m0 in zip(moms, M)],
               "grads_kept": all(bool((g.numpy() == g0).all()) for g, g0 in zip(grads, G))}
    finally:
        dist.destroy_process_group()
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump(res, f)


@pytest.mark.parametrize("world,reduce_grads,waves", [(2, False, 1), (3, False, 1), (2, True, 1), (3, True, 2),
                                                      (2, False, 3)])
def test_sharded_step_matches_single_process(tmp_path, world, reduce_grads, waves):
    sys.path.insert(0, ROOT)
    import oracle

    port = _free_port()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, str(tmp_path), reduce_grads, waves))
             for r in range(world)]
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
    # single-process reference: two steps of every matrix, on the mean of the ranks' gradients
    W, G, M = _inputs()
    if reduce_grads:
        local = [_local_grads(G, r, world) for r in range(world)]
        G = [np.mean([np.float64(lg[i]) for lg in local], axis=0) for i in range(len(SHAPES))]
    for i in range(len(SHAPES)):
        w, m = W[i].astype(np.float64), M[i].astype(np.float64)
        for _ in range(2):
            w, m, _ = oracle.muon_step(np.float32(w).astype(np.float64), np.asarray(G[i], np.float64),
                                       np.float32(m).astype(np.float64), coeffs=[oracle.QUINTIC] * 5, **HYPER)
        for r in range(world):
            assert np.allclose(np.array(res[r]["params"][i]), np.float32(w), rtol=0, atol=1e-6), (i, r)
    owners = res[0]["owners"]
    assert all(x["owners"] == owners for x in res)
    assert set(owners) == set(range(world))
    for r in range(world):
        assert res[r]["grads_kept"]
        for i, o in enumerate(owners):
            assert res[r]["mom_changed"][i] == (o == r)
        # each owned wave stepped once per call, waves in order
        mine = [[i for i in range(len(SHAPES)) if owners[i] == r and res[r]["waves"][i] == j]
                for j in range(max(res[r]["waves"]) + 1)]
        assert res[r]["calls"] == [c for c in mine if c] * 2


def test_flat_buffers_keep_views_aligned_and_disjoint():
    sys.path.insert(0, ROOT)
    from newton_schulz_11_b200.distributed import _PAD, _Flat

    shapes = [(3, 5), (8, 8), (1, 1), (16, 24)]
    for dtype in (torch.float32, torch.bfloat16):
        f = _Flat(shapes, dtype, torch.device("cpu"))
        base = f.buf.data_ptr()
        spans = []
        for v, (r, c) in zip(f.views, shapes):
            assert tuple(v.shape) == (r, c) and v.is_contiguous()
            off = (v.data_ptr() - base) // f.buf.element_size()
            assert off % _PAD == 0
            spans.append((off, off + r * c))
        spans.sort()
        assert all(a[1] <= b[0] for a, b in zip(spans, spans[1:]))
        src = [torch.randn(s).to(dtype) for s in shapes]
        f.pack(src)
        dst = [torch.empty(s, dtype=dtype) for s in shapes]
        f.unpack(dst)
        assert all(torch.equal(a, b) for a, b in zip(src, dst))
