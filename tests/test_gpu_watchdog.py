"""Bounded device waits: a wait that runs out reports MUON_ERR_TIMEOUT and the context
stays usable.  The failure is made by a wait budget far shorter than any TMA load
takes, never by a fault or a trap; every role then leaves through its bounded
teardown (in-flight loads and MMAs are still waited for, up to two seconds)."""
import numpy as np
import pytest

import oracle
from tests.gpu_util import rel_fro, require_gpu, to_np, torch

pytestmark = pytest.mark.gpu


def test_short_wait_budget_reports_timeout_and_recovers():
    require_gpu()
    from newton_schulz_11_b200 import _lib, api

    g = torch.randn(1024, 2048, device="cuda")
    ws = api.Workspace(g.device)
    out = torch.empty_like(g)
    api.newton_schulz([g], outs=[out], workspace=ws)
    code, _ = api.device_status(ws)
    assert code == _lib.MUON_OK
    try:
        _lib.lib().muon_set_wait_timeout_us(1)  # far below one k-block's TMA latency
        api.newton_schulz([g], outs=[out], workspace=ws)
        code, where = api.device_status(ws)
        assert code == _lib.MUON_ERR_TIMEOUT, (code, where)
        assert 1 <= where <= 8
    finally:
        _lib.lib().muon_set_wait_timeout_us(0)
    # the context still works and a fresh status word reads OK
    _lib.check(_lib.lib().muon_workspace_init(ws.buf.data_ptr(), ws.nbytes,
                                              int(torch.cuda.current_stream().cuda_stream)), "init")
    O = api.newton_schulz([g], workspace=ws)[0]
    code, _ = api.device_status(ws)
    assert code == _lib.MUON_OK
    ref = oracle.newton_schulz(to_np(g), [oracle.QUINTIC] * 5)
    assert rel_fro(to_np(O), ref) <= 2e-2
