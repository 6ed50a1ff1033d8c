"""bench.py's step constructions on one GPU: the sharded mode (ShardedMuon over two waves of
the owned matrices; on one rank it owns every matrix and runs no collective) must give
exactly the plain grouped step's parameters and momentum."""
import os
import sys

import pytest

from tests.gpu_util import require_gpu, torch

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_sharded_mode_on_one_rank_equals_the_plain_step():
    require_gpu()
    sys.path.insert(0, ROOT)
    import bench
    from newton_schulz_11_b200 import api, inputs

    w = inputs.scaled_workload(inputs.WORKLOADS["gpt2-124m-72-matrices"],
                               [(256, 256)] * 4 + [(256, 1024), (1024, 256)] * 2, name="gpt2-shaped-256")
    dev = torch.device("cuda", torch.cuda.current_device())
    runs = {}
    for mode in ("single", "sharded"):
        _, (gs, ms, ps), _ = bench.flat_workload(w, dev, inputs.first_step_index(w))
        step, owned = bench.make_step(w, ps, gs, ms, mode=mode, world=1, waves=2, workspace=api.Workspace(dev))
        assert owned == list(range(len(w.shapes)))
        for _ in range(3):
            step()
        torch.cuda.synchronize()
        runs[mode] = ([p.clone() for p in ps], [m.clone() for m in ms])
    for a, b in zip(runs["single"][0] + runs["single"][1], runs["sharded"][0] + runs["sharded"][1]):
        assert torch.equal(a, b)
