"""AdamW entry point, host side (no GPU needed): argument validation with fake device
pointers.  Nothing reaches a device here; a valid call stops at the device check."""
import ctypes

import pytest

from newton_schulz_11_b200 import _lib
from tests.conftest import cuda_present


@pytest.fixture(scope="module")
def L():
    return _lib.lib()


def tensors(sizes, dtype=_lib.MUON_F32):
    arr = (_lib.MuonAdamwTensor * len(sizes))()
    base = 1 << 40
    for i, n in enumerate(sizes):
        for f in ("param", "grad", "exp_avg", "exp_avg_sq"):
            setattr(arr[i], f, base)
            base += ((4 * n + 255) // 256) * 256 + 256
        arr[i].numel = n
        arr[i].param_dtype = dtype
    return arr


def call(L, arr, n=None, lr=1e-3, b1=0.9, b2=0.999, eps=1e-8, wd=0.0, step=1):
    return L.muon_adamw_step(arr, len(arr) if n is None else n, lr, b1, b2, eps, wd, step, None)


def test_valid_call_reaches_the_device_check(L):
    if cuda_present():
        pytest.skip("fake device pointers: only where no kernel can run")
    st = call(L, tensors([10, 1000, 3]))
    assert st in (_lib.MUON_ERR_NO_DEVICE, _lib.MUON_ERR_CUDA)


def test_rejects_bad_arguments(L):
    E = _lib
    good = tensors([10, 20])
    assert call(L, good, n=0) == E.MUON_ERR_INVALID_ARG
    for kw in (dict(lr=-1.0), dict(b1=1.0), dict(b2=-0.1), dict(eps=0.0), dict(wd=-1.0), dict(step=0),
               dict(lr=float("nan")), dict(b2=float("inf"))):
        assert call(L, good, **kw) == E.MUON_ERR_INVALID_ARG, kw
    bad = tensors([10]); bad[0].grad = None
    assert call(L, bad) == E.MUON_ERR_INVALID_ARG
    bad = tensors([10]); bad[0].numel = 0
    assert call(L, bad) == E.MUON_ERR_UNSUPPORTED_SHAPE
    bad = tensors([10]); bad[0].param_dtype = 5
    assert call(L, bad) == E.MUON_ERR_UNSUPPORTED_DTYPE
    bad = tensors([10]); bad[0].exp_avg += 2
    assert call(L, bad) == E.MUON_ERR_ALIGNMENT
    bad = tensors([10], dtype=_lib.MUON_BF16); bad[0].param += 1
    assert call(L, bad) == E.MUON_ERR_ALIGNMENT
    bad = tensors([10]); bad[0].exp_avg_sq = bad[0].exp_avg  # two written buffers alias
    assert call(L, bad) == E.MUON_ERR_INVALID_ARG
    bad = tensors([10, 10]); bad[1].param = bad[0].grad + 8  # a write over another tensor's grad
    assert call(L, bad) == E.MUON_ERR_INVALID_ARG
    ok = tensors([10, 10]); ok[1].grad = ok[0].grad  # two tensors reading one grad is allowed
    if not cuda_present():
        assert call(L, ok) in (E.MUON_ERR_NO_DEVICE, E.MUON_ERR_CUDA)


def test_struct_layout_matches_header():
    assert ctypes.sizeof(_lib.MuonAdamwTensor) == 48
