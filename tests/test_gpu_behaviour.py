"""Behaviour of the CUDA path beyond single-call parity: determinism, waves, strided
views, NaN isolation between matrices, no-op on invalid calls, state round trip."""
import numpy as np
import pytest

import oracle
from newton_schulz_11_b200 import inputs
from tests.gpu_util import rel_fro, require_gpu, to_np, torch

pytestmark = pytest.mark.gpu
QUINTIC5 = [oracle.QUINTIC] * 5


def _set(shapes, seed=0, dtype=torch.bfloat16):
    w = inputs.scaled_workload(inputs.WORKLOADS["gpt2-124m-72-matrices"], shapes)
    Ws = [torch.from_numpy(inputs.weight_np(w, i)).cuda().to(dtype) for i in range(len(shapes))]
    gs = [torch.from_numpy(inputs.grad_np(w, 1 + seed, i)).cuda() for i in range(len(shapes))]
    ms = [torch.from_numpy(inputs.grad_np(w, 0, i)).cuda() for i in range(len(shapes))]
    return Ws, gs, ms


def _clone(ts):
    return [t.clone() for t in ts]


SHAPES = [(256, 128), (128, 384), (256, 128), (192, 192), (136, 200)]


def test_bitwise_deterministic():
    require_gpu()
    from newton_schulz_11_b200 import api

    Ws, gs, ms = _set(SHAPES)
    W1, m1 = _clone(Ws), _clone(ms)
    W2, m2 = _clone(Ws), _clone(ms)
    O1 = [torch.empty_like(g) for g in gs]
    O2 = [torch.empty_like(g) for g in gs]
    api.muon_step(W1, gs, m1, lr=0.02, outs=O1)
    api.muon_step(W2, gs, m2, lr=0.02, outs=O2)
    for a, b in zip(O1 + W1 + m1, O2 + W2 + m2):
        assert torch.equal(a, b)


def test_concurrent_steps_on_two_streams_match_sequential_ones():
    """Two grouped steps issued on two streams at once, each with its own workspace and
    matrices (one set of shapes shared, so the library's per-signature plans and launch
    state are exercised from both), give bit-identical results to the same steps run one
    after the other."""
    require_gpu()
    from newton_schulz_11_b200 import api

    dev = torch.device("cuda", torch.cuda.current_device())
    sets = [_set(SHAPES, seed=0), _set(SHAPES[:3] + [(512, 256)], seed=1)]
    runs = []
    for concurrent in (False, True):
        state = [(_clone(W), g, _clone(m), [torch.empty_like(x) for x in g]) for W, g, m in sets]
        wss = [api.Workspace(dev), api.Workspace(dev)]
        streams = [torch.cuda.Stream(dev), torch.cuda.Stream(dev)]
        torch.cuda.synchronize()
        for k, ((W, g, m, O), ws) in enumerate(zip(state, wss)):
            s = streams[k] if concurrent else torch.cuda.current_stream(dev)
            with torch.cuda.stream(s):
                for _ in range(3):
                    api.muon_step(W, g, m, lr=0.02, outs=O, workspace=ws)
        torch.cuda.synchronize()
        for ws in wss:
            assert api.device_status(ws)[0] == 0
        runs.append([t for W, _, m, O in state for t in W + m + O])
    for a, b in zip(*runs):
        assert torch.equal(a, b)


def test_waves_give_identical_results():
    """A workspace that fits one matrix at a time gives bit-identical results."""
    require_gpu()
    from newton_schulz_11_b200 import api

    Ws, gs, ms = _set(SHAPES)
    W1, m1, W2, m2 = _clone(Ws), _clone(ms), _clone(Ws), _clone(ms)
    O1 = [torch.empty_like(g) for g in gs]
    O2 = [torch.empty_like(g) for g in gs]
    api.muon_step(W1, gs, m1, lr=0.02, outs=O1)
    one = max(api.workspace_size([tuple(g.shape)]) for g in gs)
    ws = api.Workspace(gs[0].device)
    api.muon_step(W2, gs, m2, lr=0.02, outs=O2, workspace=ws, workspace_bytes=one)
    assert api.scratch_view([tuple(g.shape) for g in gs], len(gs) - 1, one).wave == len(gs) - 1
    for a, b in zip(O1 + W1 + m1, O2 + W2 + m2):
        assert torch.equal(a, b)


def test_strided_views_match_contiguous():
    """Parameters, grads and momentum given as column blocks of wider buffers (ld > cols)."""
    require_gpu()
    from newton_schulz_11_b200 import api

    Ws, gs, ms = _set([(192, 128), (128, 256)], dtype=torch.float32)
    bigW = [torch.zeros(W.shape[0], W.shape[1] + 40, device="cuda") for W in Ws]
    bigg = [torch.zeros(g.shape[0], g.shape[1] + 24, device="cuda") for g in gs]
    bigm = [torch.zeros(m.shape[0], m.shape[1] + 8, device="cuda") for m in ms]
    vW = [b[:, 8: 8 + W.shape[1]] for b, W in zip(bigW, Ws)]
    vg = [b[:, 4: 4 + g.shape[1]] for b, g in zip(bigg, gs)]
    vm = [b[:, : m.shape[1]] for b, m in zip(bigm, ms)]
    for v, t in zip(vW + vg + vm, Ws + gs + ms):
        v.copy_(t)
    Wc, mc = _clone(Ws), _clone(ms)
    api.muon_step(Wc, gs, mc, lr=0.02, weight_decay=0.1)
    api.muon_step(vW, vg, vm, lr=0.02, weight_decay=0.1)
    for a, b in zip(vW + vm, Wc + mc):
        assert torch.equal(a, b)
    # bytes outside the views untouched
    for b, W in zip(bigW, Ws):
        assert torch.count_nonzero(b[:, :8]).item() == 0 and torch.count_nonzero(b[:, 8 + W.shape[1]:]).item() == 0


def test_nan_stays_in_its_matrix_and_is_reported():
    """A NaN in one gradient propagates into that matrix's results only, and the
    elementwise pass reports it: MUON_ERR_NONFINITE with the matrix's index, and the count
    of non-finite u (u = g + beta (beta m + g) is non-finite exactly where g or m is)."""
    require_gpu()
    from newton_schulz_11_b200 import _lib, api

    Ws, gs, ms = _set([(128, 128), (128, 256), (200, 72)], dtype=torch.float32)
    ws = api.Workspace(gs[0].device)
    O = [torch.empty_like(g) for g in gs]
    api.muon_step(Ws, gs, ms, lr=0.02, outs=O, workspace=ws)
    assert api.device_status(ws) == (_lib.MUON_OK, 0)
    assert api.nonfinite_count(ws) == 0
    gs[1][3, 5] = float("nan")
    gs[1][100, 7] = float("inf")
    ms[1][0, 255] = float("-inf")
    api.muon_step(Ws, gs, ms, lr=0.02, outs=O, workspace=ws)
    assert torch.isnan(O[1]).any()
    for i in (0, 2):
        assert torch.isfinite(O[i]).all() and torch.isfinite(Ws[i]).all() and torch.isfinite(ms[i]).all()
    assert api.device_status(ws) == (_lib.MUON_ERR_NONFINITE, 1)
    assert api.nonfinite_count(ws) == 3
    # sticky until cleared; Newton-Schulz alone checks its input G the same way
    api.clear_device_status(ws)
    assert api.device_status(ws) == (_lib.MUON_OK, 0) and api.nonfinite_count(ws) == 0
    G = [torch.randn(96, 64, device="cuda"), torch.randn(64, 64, device="cuda")]
    G[1][7, 7] = float("nan")
    api.newton_schulz(G, workspace=ws)
    assert api.device_status(ws) == (_lib.MUON_ERR_NONFINITE, 1)
    assert api.nonfinite_count(ws) == 1


def test_checkpoint_round_trip_is_bit_identical():
    """3 steps == 2 steps, save/load of params and momentum, 1 step."""
    require_gpu()
    from newton_schulz_11_b200 import api

    Ws, gs, ms = _set([(256, 128), (128, 256)])
    WA, mA = _clone(Ws), _clone(ms)
    for _ in range(3):
        api.muon_step(WA, gs, mA, lr=0.02, weight_decay=0.01)
    WB, mB = _clone(Ws), _clone(ms)
    for _ in range(2):
        api.muon_step(WB, gs, mB, lr=0.02, weight_decay=0.01)
    saved = [t.cpu() for t in WB + mB]
    WC = [t.cuda() for t in saved[:2]]
    mC = [t.cuda() for t in saved[2:]]
    api.muon_step(WC, gs, mC, lr=0.02, weight_decay=0.01)
    for a, b in zip(WA + mA, WC + mC):
        assert torch.equal(a, b)


def test_invalid_call_touches_nothing():
    require_gpu()
    from newton_schulz_11_b200 import api, _lib

    Ws, gs, ms = _set([(64, 64)], dtype=torch.float32)
    W0, m0 = _clone(Ws), _clone(ms)
    with pytest.raises(_lib.MuonError):
        api.muon_step(Ws, gs, ms, lr=0.02, beta=2.0)
    torch.cuda.synchronize()
    assert torch.equal(Ws[0], W0[0]) and torch.equal(ms[0], m0[0])


def test_device_status_stays_ok():
    require_gpu()
    from newton_schulz_11_b200 import api, _lib

    Ws, gs, ms = _set(SHAPES)
    ws = api.Workspace(gs[0].device)
    api.muon_step(Ws, gs, ms, lr=0.02, workspace=ws)
    assert api.device_status(ws) == (_lib.MUON_OK, 0)


def test_prepared_calls_match_one_shot_calls():
    """PreparedMuonStep / PreparedAdamW reuse their descriptors; results are bit-identical
    to the one-shot calls, over consecutive steps."""
    require_gpu()
    from newton_schulz_11_b200 import api

    Ws, gs, ms = _set(SHAPES)
    W1, m1 = _clone(Ws), _clone(ms)
    W2, m2 = _clone(Ws), _clone(ms)
    prep = api.PreparedMuonStep(W2, gs, m2, lr=0.02, weight_decay=0.01)
    for _ in range(2):
        api.muon_step(W1, gs, m1, lr=0.02, weight_decay=0.01)
        prep()
    for a, b in zip(W1 + m1, W2 + m2):
        assert torch.equal(a, b)

    g = [torch.randn(n, device="cuda") for n in (5, 4096, 70001)]
    p1 = [torch.randn(x.numel(), device="cuda").to(torch.bfloat16) for x in g]
    p2 = _clone(p1)
    st1 = [[torch.zeros_like(x) for x in g] for _ in range(2)]
    st2 = [[torch.zeros_like(x) for x in g] for _ in range(2)]
    prep_a = api.PreparedAdamW(p2, g, st2[0], st2[1], lr=1e-3, betas=(0.9, 0.95), weight_decay=0.1)
    for t in (1, 2, 3):
        api.adamw_step(p1, g, st1[0], st1[1], lr=1e-3, step=t, betas=(0.9, 0.95), weight_decay=0.1)
        prep_a(t)
    for a, b in zip(p1 + st1[0] + st1[1], p2 + st2[0] + st2[1]):
        assert torch.equal(a, b)


@pytest.mark.parametrize("waves", [1, 2])
def test_sharded_muon_on_one_rank_is_the_plain_step(waves):
    """Without a process group (one rank) the sharded step owns every matrix and runs the
    library's grouped step, one prepared step per wave: bit-identical to muon_step."""
    require_gpu()
    from newton_schulz_11_b200 import api
    from newton_schulz_11_b200.distributed import ShardedMuon

    Ws, gs, ms = _set(SHAPES)
    W1, m1 = _clone(Ws), _clone(ms)
    W2, m2 = _clone(Ws), _clone(ms)
    api.muon_step(W1, gs, m1, lr=0.02, weight_decay=0.01)
    sh = ShardedMuon(W2, gs, m2, lr=0.02, weight_decay=0.01, waves=waves)
    assert sh.waves == waves and sorted(i for w in sh.wave_idx for i in w) == list(range(len(gs)))
    sh()
    for a, b in zip(W1 + m1, W2 + m2):
        assert torch.equal(a, b)


def test_prepared_step_survives_workspace_growth():
    """A prepared step keeps the buffer it was prepared on: growing the shared workspace for a
    larger step afterwards (which drops the old buffer) leaves the first step's results
    bit-identical to the plain call, and its status word readable."""
    require_gpu()
    from newton_schulz_11_b200 import _lib, api

    Ws, gs, ms = _set(SHAPES[:2])
    W1, m1, W2, m2 = _clone(Ws), _clone(ms), _clone(Ws), _clone(ms)
    ws = api.Workspace(gs[0].device)
    small = api.PreparedMuonStep(W2, gs, m2, lr=0.02, workspace=ws)
    before = ws.nbytes
    BW, bg, bm = _set([(1024, 2048)], seed=3)
    big = api.PreparedMuonStep(BW, bg, bm, lr=0.02, workspace=ws)
    assert ws.nbytes > before
    # reuse the freed memory for something else before the small step runs again
    junk = [torch.full((before // 4,), float("nan"), device=gs[0].device) for _ in range(2)]
    for _ in range(2):
        api.muon_step(W1, gs, m1, lr=0.02)
        small()
        big()
    torch.cuda.synchronize()
    del junk
    for a, b in zip(W1 + m1, W2 + m2):
        assert torch.equal(a, b)
    assert small.device_status() == (_lib.MUON_OK, 0)
    assert big.device_status() == (_lib.MUON_OK, 0)


def test_step_replays_from_a_cuda_graph():
    """A step is kernel launches only (parameters by value, no host copies or syncs), so it
    can be captured in a CUDA graph; each replay equals an eager step bit for bit."""
    require_gpu()
    from newton_schulz_11_b200 import _lib, api

    Ws, gs, ms = _set(SHAPES)
    W1, m1, W2, m2 = _clone(Ws), _clone(ms), _clone(Ws), _clone(ms)
    eager = api.PreparedMuonStep(W1, gs, m1, lr=0.02, weight_decay=0.01)
    graphed = api.PreparedMuonStep(W2, gs, m2, lr=0.02, weight_decay=0.01)
    eager()
    graphed()  # the first call builds and caches the host-side plan
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        graphed()
    for _ in range(3):
        eager()
        g.replay()
        torch.cuda.synchronize()
        for a, b in zip(W1 + m1, W2 + m2):
            assert torch.equal(a, b)
    assert graphed.device_status() == (_lib.MUON_OK, 0)
    del g
