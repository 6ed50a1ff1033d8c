"""The N > 1 path of bench.py, run as two gloo ranks on the CPU.

On GPUs the same code runs one process per GPU over NCCL.  Each rank times its own
replica of the workload (weak scaling, no data-path collective); the ranks meet only
at the barriers around the timed region and in the max over ranks of the step time.
Here rank r reports r + 1 as its time, so every rank must see the max (= world size),
and only rank 0 of the reference arm prints a line.
"""
import contextlib
import io
import json
import os
import socket
import sys
import types

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
WORLD = 2


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

    args = types.SimpleNamespace(workload="single-256x128-f32", steps=2, warmup=1)
    world, r, local = bench.dist_setup(args, backend="gloo")
    result = {"world": world, "rank": r, "local": local}
    try:
        bench.barrier(world)
        result["max"] = bench.dist_max(float(r + 1), world)
        bench.barrier(world)
        buf = io.StringIO()
        with contextlib.redirect_stdout(buf):
            bench.run_reference(args, world, r)
        result["printed"] = buf.getvalue()
        bench.barrier(world)
    finally:
        dist.destroy_process_group()
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump(result, f)


def test_two_gloo_ranks_share_the_max_and_only_rank0_prints(tmp_path):
    port = _free_port()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_rank_main, args=(r, port, str(tmp_path))) for r in range(WORLD)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=240)
    for p in procs:
        if p.is_alive():
            p.kill()
            pytest.fail("a rank did not finish")
        assert p.exitcode == 0
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(WORLD)]
    for r, x in enumerate(res):
        assert (x["world"], x["rank"], x["local"]) == (WORLD, r, r)
        assert x["max"] == float(WORLD)
    line = json.loads(res[0]["printed"])
    assert line["impl"] == "reference" and line["n_gpus"] == WORLD and line["value"] > 0
    assert res[1]["printed"] == ""
