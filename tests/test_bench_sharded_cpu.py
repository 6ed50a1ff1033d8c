"""bench.py's sharded mode (the default under torchrun), driven end to end on two gloo ranks.

The bench's own pieces run as on GPUs -- parallel_mode, make_step (ShardedMuon with the
gradients averaged onto each matrix's owner and the parameters broadcast back),
time_steps (barrier, timed steps, max over ranks) and base_line -- with the fp64 oracle as
the local step on the owned matrices, on a GPT-2-shaped set scaled down.  Every rank must
end with the parameters one process computes from the mean gradient, both ranks must see
the same step time, and the line must describe a strong-scaling sharded run.
"""
import dataclasses
import json
import os
import socket
import sys
import types

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
WORLD = 2
STEPS, WARMUP = 2, 1


def _workload():
    sys.path.insert(0, ROOT)
    from newton_schulz_11_b200 import inputs

    base = inputs.WORKLOADS["gpt2-124m-72-matrices"]
    shapes = [(64, 64)] * 4 + [(64, 256), (256, 64)]
    return dataclasses.replace(base, shapes=tuple(shapes * 2), name="gpt2-shaped-2x64", param_dtype="f32")


def _local_grads(w, rank):
    """Rank-local gradients whose mean over the ranks is the workload's gradient."""
    from newton_schulz_11_b200 import inputs

    rng = np.random.default_rng(50 + rank)
    out = []
    for i in range(len(w.shapes)):
        g = inputs.grad_np(w, 1, i)
        noise = rng.standard_normal(g.shape).astype(np.float32) * np.float32(1e-3)
        out.append((g + np.float32(rank - (WORLD - 1) / 2) * 2 * noise).astype(np.float32))
    return out


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, port, out_dir):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(WORLD),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    import torch.distributed as dist

    import bench
    import oracle
    from newton_schulz_11_b200 import inputs

    args = types.SimpleNamespace(steps=STEPS, warmup=WARMUP, parallel="auto", waves=2)
    world, r, _ = bench.dist_setup(args, backend="gloo")
    try:
        w = _workload()
        ps = [torch.from_numpy(inputs.weight_np(w, i)) for i in range(len(w.shapes))]
        gs = [torch.from_numpy(g) for g in _local_grads(w, r)]
        ms = [torch.from_numpy(inputs.momentum_np(w, i)) for i in range(len(w.shapes))]
        coeffs = bench.load_coeffs(w)

        def local_step(idx, grads):
            for i, g in zip(idx, grads):
                W1, m1, _ = oracle.muon_step(ps[i].double().numpy(), g.double().numpy(), ms[i].double().numpy(),
                                             lr=w.lr, beta=w.beta, weight_decay=w.weight_decay,
                                             nesterov=w.nesterov, coeffs=coeffs)
                ps[i].copy_(torch.from_numpy(W1))
                ms[i].copy_(torch.from_numpy(m1))

        mode = bench.parallel_mode(args, world)
        step, owned = bench.make_step(w, ps, gs, ms, mode=mode, world=world, waves=args.waves,
                                      local_step=local_step)
        for _ in range(args.warmup):
            step()
        ms_step = bench.time_steps(step, args.steps, world, "cpu")
        line = bench.base_line(w, world, mode, ms_step, args)
        res = {"line": line, "owned": owned, "ms_step": ms_step, "params": [p.tolist() for p in ps]}
    finally:
        dist.destroy_process_group()
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump(res, f)


def test_bench_sharded_mode_on_two_gloo_ranks(tmp_path):
    sys.path.insert(0, ROOT)
    import bench
    import oracle
    from newton_schulz_11_b200 import inputs

    port = _free_port()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_rank_main, args=(r, port, str(tmp_path))) for r in range(WORLD)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
    for p in procs:
        if p.is_alive():
            p.kill()
            pytest.fail("a rank did not finish")
        assert p.exitcode == 0
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(WORLD)]

    w = _workload()
    # the owners split the matrices, and both ranks timed the same (max over ranks) step
    assert sorted(res[0]["owned"] + res[1]["owned"]) == list(range(len(w.shapes)))
    assert res[0]["owned"] and res[1]["owned"]
    assert res[0]["ms_step"] == res[1]["ms_step"] > 0
    line = res[0]["line"]
    assert line["n_gpus"] == WORLD and line["scaling"] == "strong" and line["value"] > 0
    assert line["config"] == bench.config_of(w, WORLD, "sharded")
    assert line["config"]["parallelism"] == "sharded"

    # one process, the mean gradient, warm-up + timed steps
    local = [_local_grads(w, r) for r in range(WORLD)]
    coeffs = bench.load_coeffs(w)
    for i in range(len(w.shapes)):
        g = np.mean([np.float64(lg[i]) for lg in local], axis=0)
        W, m = inputs.weight_np(w, i).astype(np.float64), inputs.momentum_np(w, i).astype(np.float64)
        for _ in range(WARMUP + STEPS):
            W, m, _ = oracle.muon_step(np.float32(W).astype(np.float64), np.float32(g).astype(np.float64),
                                       np.float32(m).astype(np.float64), lr=w.lr, beta=w.beta,
                                       weight_decay=w.weight_decay, nesterov=w.nesterov, coeffs=coeffs)
        for r in range(WORLD):
            got = np.array(res[r]["params"][i])
            assert np.allclose(got, np.float32(W), rtol=0, atol=1e-6), (i, r, np.abs(got - W).max())
