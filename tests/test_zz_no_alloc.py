"""The entry point that allocates nothing: muon_newton_schulz_static.

Some callers cannot hand this library a workspace: code running inside another
framework's caching allocator (a cudaMalloc of its own would fragment or bypass that
pool), plugins that only receive ready-made device buffers, and callers that must not
allocate between steps.  For them the Newton-Schulz iteration can run on a static
device array inside the library (MUON_STATIC_SCRATCH_BYTES, held by every GPU that
loads the library until exit).

The GPU test calls the entry point through the C ABI twice in a row, on different
inputs, and checks each result against the workspace entry point (muon_newton_schulz);
each call is repeated through the Python binding, which must give the same bits.
Both run the same kernels with the same per-matrix arithmetic in the same order, and
the library's results do not depend on how matrices are grouped into waves, so the two
must agree bit for bit (the workspace entry point is itself checked against the fp64
oracle by the parity tests).  The file is named to be collected last; it also passes when
run alone in a fresh process.
"""
import ctypes

import numpy as np
import pytest

from newton_schulz_11_b200 import _lib, api

TOL_NS = 2e-2  # relative Frobenius error of O, as in the parity tests


def _call_static(descs, n, table, steps, eps, status_ptr, stream):
    return _lib.lib().muon_newton_schulz_static(descs, n, steps, table, ctypes.c_float(eps), status_ptr, stream)


def test_static_scratch_rejects_matrices_beyond_the_limit():
    """A matrix whose scratch exceeds the static array is refused before anything runs
    (fake, aligned device pointers: no device is touched)."""
    h = _lib.lib()
    side = 4096  # hi/lo copies alone take 96 MiB
    arr = (_lib.MuonMatrix * 1)()
    arr[0].rows, arr[0].cols = side, side
    arr[0].grad = 1 << 20
    arr[0].ld_grad = side
    arr[0].out_update = 1 << 30
    table, steps = api._coeff_array(api.quintic_table())
    st = h.muon_newton_schulz_static(arr, 1, steps, table, ctypes.c_float(api.DEFAULT_EPS), None, None)
    assert st == _lib.MUON_ERR_STATIC_SCRATCH_LIMIT, _lib.status_str(st)
    assert "static" in _lib.status_str(st)


@pytest.mark.gpu
def test_static_scratch_matches_workspace_entry_point_on_two_calls():
    from tests.gpu_util import rel_fro, require_gpu, to_np, torch

    require_gpu()
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream(dev)
    table, steps = api._coeff_array(api.quintic_table())
    status = torch.full((2,), -1, dtype=torch.int32, device=dev)

    calls = [
        (11, [(1024, 2048), (768, 768), (3072, 768), (300, 500)]),
        (12, [(768, 3072), (1000, 130), (257, 257)]),
    ]
    for seed, shapes in calls:
        gen = torch.Generator(device=dev).manual_seed(seed)
        Gs = [torch.randn(r, c, device=dev, generator=gen) for r, c in shapes]
        ref = api.newton_schulz(Gs, workspace=api.Workspace(dev))
        outs = [torch.full_like(g, float("nan")) for g in Gs]
        descs = api._descriptors(None, Gs, None, outs, None, ns_only=True)
        status.fill_(-1)
        st = _call_static(descs, len(Gs), table, steps, api.DEFAULT_EPS, status.data_ptr(),
                          int(stream.cuda_stream))
        assert st == _lib.MUON_OK, _lib.status_str(st)
        torch.cuda.synchronize()
        assert status.tolist() == [0, 0]
        for (r, c), o, o_ref in zip(shapes, outs, ref):
            o_np, ref_np = to_np(o), to_np(o_ref)
            assert np.isfinite(o_np).all(), (r, c)
            assert torch.equal(o, o_ref), ((r, c), rel_fro(o_np, ref_np))
            assert rel_fro(o_np, ref_np) <= TOL_NS
        # the Python binding of the same entry point: the same bits
        outs2 = [torch.full_like(g, float("nan")) for g in Gs]
        status.fill_(-1)
        api.newton_schulz_static(Gs, outs=outs2, device_status=status)
        torch.cuda.synchronize()
        assert status.tolist() == [0, 0]
        for o, o2 in zip(outs, outs2):
            assert torch.equal(o, o2)


@pytest.mark.gpu
def test_static_scratch_reports_a_nonfinite_input():
    """A NaN in one matrix's G: the status output reads MUON_ERR_NONFINITE with that
    matrix's index, and the other matrix's O is still the workspace entry point's."""
    from tests.gpu_util import require_gpu, torch

    require_gpu()
    dev = torch.device("cuda", torch.cuda.current_device())
    gen = torch.Generator(device=dev).manual_seed(13)
    Gs = [torch.randn(256, 384, device=dev, generator=gen), torch.randn(192, 128, device=dev, generator=gen)]
    Gs[1][5, 7] = float("nan")
    status = torch.full((2,), -1, dtype=torch.int32, device=dev)
    outs = api.newton_schulz_static(Gs, device_status=status)
    ref = api.newton_schulz(Gs[:1], workspace=api.Workspace(dev))
    torch.cuda.synchronize()
    assert status.tolist() == [_lib.MUON_ERR_NONFINITE, 1]
    assert torch.equal(outs[0], ref[0])
