"""Host-side checks of the C ABI that need no GPU: the library loads, exports every
function include/muon_b200.h declares, sizes workspaces, plans waves and rejects bad
arguments before it touches CUDA."""
import ctypes
import os
import re

import pytest

from newton_schulz_11_b200 import _lib, build, inputs
from tests.conftest import cuda_present
from newton_schulz_11_b200._lib import MuonMatrix, MuonScratchView

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "muon_b200.h")


@pytest.fixture(scope="module")
def L():
    build.build()
    return _lib.lib()


def header_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(muon_[a-z_]+)\s*\(", text)))


def test_header_declares_the_binding_exports():
    assert header_functions() == sorted(_lib.EXPORTS)


def test_library_exports_every_declared_symbol(L):
    for name in header_functions():
        assert hasattr(L, name), name
        assert ctypes.cast(getattr(L, name), ctypes.c_void_p).value


def test_abi_version_and_status_strings(L):
    assert L.muon_abi_version() == _lib.MUON_ABI_VERSION == 4
    for code in range(11):
        assert L.muon_status_str(code).decode() not in ("", "unknown status")
    assert L.muon_status_str(99).decode() == "unknown status"


def test_status_codes_match_the_header():
    import re

    with open(os.path.join(ROOT, "include", "muon_b200.h")) as f:
        text = f.read()
    codes = {k: int(v) for k, v in re.findall(r"\b(MUON_(?:OK|ERR_[A-Z_]+))\s*=\s*(\d+)", text)}
    assert codes["MUON_ERR_NONFINITE"] == 10
    for name, value in codes.items():
        assert getattr(_lib, name) == value, name


def mats_of(shapes, base=1 << 40, dtype=_lib.MUON_BF16, spacing=1 << 34):
    """Descriptors with fake, disjoint, well-aligned device addresses (never dereferenced)."""
    n = len(shapes)
    arr = (MuonMatrix * n)()
    for i, (r, c) in enumerate(shapes):
        b = base + i * spacing
        arr[i].rows, arr[i].cols = r, c
        arr[i].param = b
        arr[i].grad = b + (spacing >> 2)
        arr[i].momentum = b + 2 * (spacing >> 2)
        arr[i].ld_param = arr[i].ld_grad = arr[i].ld_mom = c
        arr[i].param_dtype = dtype
    return arr


def ws_size(L, arr):
    out = ctypes.c_size_t(0)
    st = L.muon_workspace_size(arr, len(arr), ctypes.byref(out))
    return st, out.value


def coeffs(steps=5):
    return (ctypes.c_float * (3 * steps))(*([3.4445, -4.7750, 2.0315] * steps))


def step(L, arr, n=None, lr=0.02, beta=0.95, wd=0.0, nesterov=1, steps=5, c=None, eps=1e-7,
         ws=1 << 45, ws_bytes=1 << 36):
    return L.muon_step(arr, len(arr) if n is None else n, lr, beta, wd, nesterov, steps,
                       coeffs(steps) if c is None else c, eps, ws, ws_bytes, None)


def test_workspace_size_matches_layout(L):
    st, b = ws_size(L, mats_of([(768, 3072)]))
    assert st == 0
    x = 768 * 3072 * 2  # each bf16 hi buffer
    lo = 768 * 3072      # the 8-bit lo buffer
    a = 768 * 768 * 2
    assert b >= 2 * x + lo + 2 * a
    assert b < 2 * x + lo + 2 * a + 64 * 1024


def test_workspace_size_for_every_workload(L):
    for w in inputs.WORKLOADS.values():
        st, b = ws_size(L, mats_of(w.shapes))
        assert st == 0 and b > 0


def test_waves_split_by_matrix_limit_and_workspace(L):
    shapes = [(64, 64)] * 300
    arr = mats_of(shapes)
    st, full = ws_size(L, arr)
    assert st == 0
    v = MuonScratchView()
    assert L.muon_scratch_view(arr, 300, 299, full, ctypes.byref(v)) == 0
    assert v.wave == 2  # 128 matrices per wave at most
    st1, one = ws_size(L, mats_of([(64, 64)]))
    assert L.muon_scratch_view(arr, 300, 299, one, ctypes.byref(v)) == 0
    assert v.wave == 299
    assert L.muon_scratch_view(arr, 300, 0, one - 1024, ctypes.byref(v)) == _lib.MUON_ERR_WORKSPACE_TOO_SMALL


def test_scratch_view_tall_and_padding(L):
    arr = mats_of([(100, 36), (36, 100), (100, 36)])
    st, full = ws_size(L, arr)
    v = MuonScratchView()
    assert L.muon_scratch_view(arr, 3, 2, full, ctypes.byref(v)) == 0
    assert v.transposed == 1 and v.x_ld == 40 and v.a_ld == 40 and v.x_lo_ld == 48
    assert v.x_hi_offset[0] % 16 == 0 and v.a_offset % 16 == 0 and v.x_lo_offset % 16 == 0
    v0 = MuonScratchView()
    L.muon_scratch_view(arr, 3, 0, full, ctypes.byref(v0))
    assert v.x_hi_offset[0] - v0.x_hi_offset[0] == 100 * 40 * 2  # same class, next slot
    assert v.x_lo_offset - v0.x_lo_offset == 100 * 48


def test_validation_rejects_bad_descriptors_without_cuda(L):
    E = _lib
    good = mats_of([(64, 32), (32, 64)])
    # a valid call with fake pointers stops at the device check; never made with a device
    if not cuda_present():
        assert step(L, good) in (E.MUON_ERR_NO_DEVICE, E.MUON_ERR_CUDA)

    bad = mats_of([(64, 32)]); bad[0].grad = None
    assert step(L, bad) == E.MUON_ERR_INVALID_ARG
    bad = mats_of([(64, 32)]); bad[0].rows = 0
    assert step(L, bad) == E.MUON_ERR_UNSUPPORTED_SHAPE
    bad = mats_of([(64, 32)]); bad[0].ld_grad = 16
    assert step(L, bad) == E.MUON_ERR_UNSUPPORTED_SHAPE
    bad = mats_of([(64, 32)]); bad[0].param_dtype = 7
    assert step(L, bad) == E.MUON_ERR_UNSUPPORTED_DTYPE
    bad = mats_of([(64, 32)]); bad[0].grad = bad[0].grad + 2
    assert step(L, bad) == E.MUON_ERR_ALIGNMENT
    bad = mats_of([(64, 32)], dtype=_lib.MUON_BF16); bad[0].param = bad[0].param + 1
    assert step(L, bad) == E.MUON_ERR_ALIGNMENT
    # momentum aliasing the parameter
    bad = mats_of([(64, 32)]); bad[0].momentum = bad[0].param
    assert step(L, bad) == E.MUON_ERR_INVALID_ARG
    # two matrices sharing one momentum buffer
    bad = mats_of([(64, 32), (64, 32)]); bad[1].momentum = bad[0].momentum
    assert step(L, bad) == E.MUON_ERR_INVALID_ARG
    # overlapping a grad (read-only) by a written buffer of another matrix
    bad = mats_of([(64, 32), (64, 32)]); bad[1].param = bad[0].grad + 64
    assert step(L, bad) == E.MUON_ERR_INVALID_ARG
    # hyperparameters
    assert step(L, good, beta=1.5) == E.MUON_ERR_INVALID_ARG
    assert step(L, good, lr=float("nan")) == E.MUON_ERR_INVALID_ARG
    assert step(L, good, nesterov=2) == E.MUON_ERR_INVALID_ARG
    assert step(L, good, steps=0, c=coeffs(1)) == E.MUON_ERR_INVALID_ARG
    assert step(L, good, steps=17, c=coeffs(17)) == E.MUON_ERR_INVALID_ARG
    assert step(L, good, eps=0.0) == E.MUON_ERR_INVALID_ARG
    nanc = coeffs(5); nanc[4] = float("inf")
    assert step(L, good, c=nanc) == E.MUON_ERR_INVALID_ARG
    assert step(L, good, n=0) == E.MUON_ERR_INVALID_ARG
    assert step(L, good, ws=(1 << 45) + 16) == E.MUON_ERR_INVALID_ARG
    assert step(L, good, ws=0) == E.MUON_ERR_INVALID_ARG


def test_newton_schulz_needs_an_output(L):
    arr = mats_of([(64, 32)])
    st = L.muon_newton_schulz(arr, 1, 5, coeffs(), 1e-7, 1 << 45, 1 << 36, None)
    assert st == _lib.MUON_ERR_INVALID_ARG
    arr[0].out_update = (1 << 44) + 1024
    arr[0].param = None
    arr[0].momentum = None
    if not cuda_present():  # fake pointers: only where no kernel can run
        st = L.muon_newton_schulz(arr, 1, 5, coeffs(), 1e-7, 1 << 45, 1 << 36, None)
        assert st in (_lib.MUON_ERR_NO_DEVICE, _lib.MUON_ERR_CUDA)


def test_timeout_setter(L):
    assert L.muon_set_wait_timeout_us(500) == 0
    assert L.muon_set_wait_timeout_us(0) == 0


def test_python_binding_rejects_non_matrices():
    torch = pytest.importorskip("torch")
    from newton_schulz_11_b200 import api

    with pytest.raises(ValueError):
        api._check_2d(torch.zeros(3), "x", (torch.float32,))
    with pytest.raises(TypeError):
        api._check_2d(torch.zeros(3, 3, dtype=torch.float64), "x", (torch.float32,))


def _block_bytes(base, row0, col0, rows, cols, ld, elt):
    return {base + ((row0 + r) * ld + col0 + c) * elt + b for r in range(rows) for c in range(cols) for b in range(elt)}


def test_overlap_check_is_exact_for_blocks_of_one_matrix(L):
    """Blocks of one parent matrix (same pitch) may interleave without sharing bytes (per-
    head column blocks); the check agrees with brute force over random block pairs."""
    import random

    rnd = random.Random(5)
    R, C = 12, 20  # parent matrix, fp32, ld = C
    base_p = 1 << 40
    for trial in range(300):
        blocks = []
        for _ in range(2):
            rows, cols = rnd.randint(1, 6), rnd.randint(1, 8)
            blocks.append((rnd.randint(0, R - rows), rnd.randint(0, C - cols), rows, cols))
        arr = (MuonMatrix * 2)()
        for k, (r0, c0, rows, cols) in enumerate(blocks):
            d = arr[k]
            d.rows, d.cols = rows, cols
            d.param = base_p + (r0 * C + c0) * 4
            d.ld_param = C
            d.param_dtype = _lib.MUON_F32
            d.grad = (1 << 41) + k * (1 << 30)
            d.ld_grad = cols
            d.momentum = (1 << 42) + k * (1 << 30)
            d.ld_mom = cols
        shared = bool(_block_bytes(0, *blocks[0], C, 4) & _block_bytes(0, *blocks[1], C, 4))
        if shared:
            assert step(L, arr) == _lib.MUON_ERR_INVALID_ARG, (trial, blocks)
        elif not cuda_present():
            assert step(L, arr) in (_lib.MUON_ERR_NO_DEVICE, _lib.MUON_ERR_CUDA), (trial, blocks)
    # different pitches whose spans overlap are refused (not tested exactly)
    arr = mats_of([(4, 4), (4, 4)], dtype=_lib.MUON_F32)
    arr[1].param = arr[0].param + 4 * 4
    arr[0].ld_param, arr[1].ld_param = 8, 16
    assert step(L, arr) == _lib.MUON_ERR_INVALID_ARG
