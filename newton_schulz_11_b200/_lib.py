"""ctypes view of libmuon_b200.so (declarations mirror include/muon_b200.h)."""
from __future__ import annotations

import ctypes
import os
import threading

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libmuon_b200.so")

MUON_ABI_VERSION = 4  # the version of include/muon_b200.h these bindings follow
MUON_OK = 0
MUON_ERR_INVALID_ARG = 1
MUON_ERR_ALIGNMENT = 2
MUON_ERR_UNSUPPORTED_SHAPE = 3
MUON_ERR_UNSUPPORTED_DTYPE = 4
MUON_ERR_WORKSPACE_TOO_SMALL = 5
MUON_ERR_CUDA = 6
MUON_ERR_TIMEOUT = 7
MUON_ERR_NO_DEVICE = 8
MUON_ERR_STATIC_SCRATCH_LIMIT = 9
MUON_ERR_NONFINITE = 10
MUON_STATIC_SCRATCH_BYTES = 64 << 20

MUON_F32 = 0
MUON_BF16 = 1
MUON_MAX_NS_STEPS = 16

EXPORTS = (
    "muon_abi_version",
    "muon_status_str",
    "muon_workspace_size",
    "muon_workspace_init",
    "muon_step",
    "muon_newton_schulz",
    "muon_scratch_view",
    "muon_device_status",
    "muon_nonfinite_count",
    "muon_set_wait_timeout_us",
    "muon_profile_begin",
    "muon_profile_end",
    "muon_newton_schulz_static",
    "muon_adamw_step",
)

KIND_NAMES = ("momentum", "norm", "gram", "poly", "apply", "apply_last")


class MuonMatrix(ctypes.Structure):
    _fields_ = [
        ("param", ctypes.c_void_p),
        ("grad", ctypes.c_void_p),
        ("momentum", ctypes.c_void_p),
        ("out_update", ctypes.c_void_p),
        ("rows", ctypes.c_int64),
        ("cols", ctypes.c_int64),
        ("ld_param", ctypes.c_int64),
        ("ld_grad", ctypes.c_int64),
        ("ld_mom", ctypes.c_int64),
        ("param_dtype", ctypes.c_int32),
        ("shape_scale", ctypes.c_float),
    ]


class MuonAdamwTensor(ctypes.Structure):
    _fields_ = [
        ("param", ctypes.c_void_p),
        ("grad", ctypes.c_void_p),
        ("exp_avg", ctypes.c_void_p),
        ("exp_avg_sq", ctypes.c_void_p),
        ("numel", ctypes.c_int64),
        ("param_dtype", ctypes.c_int32),
        ("reserved", ctypes.c_int32),
    ]


class MuonScratchView(ctypes.Structure):
    _fields_ = [
        ("x_hi_offset", ctypes.c_uint64 * 2),
        ("x_lo_offset", ctypes.c_uint64),
        ("a_offset", ctypes.c_uint64),
        ("b_offset", ctypes.c_uint64),
        ("scale_offset", ctypes.c_uint64),
        ("norm_offset", ctypes.c_uint64),
        ("x_ld", ctypes.c_int64),
        ("x_lo_ld", ctypes.c_int64),
        ("a_ld", ctypes.c_int64),
        ("wave", ctypes.c_int32),
        ("transposed", ctypes.c_int32),
    ]


assert ctypes.sizeof(MuonMatrix) == 80


class MuonLibraryError(RuntimeError):
    """libmuon_b200.so is missing or cannot be loaded: there is no other code path."""


class MuonError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_str(status)} (status {status})")


_lib = None
_lock = threading.Lock()


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is not None:
        return _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(LIB_PATH):
            raise MuonLibraryError(
                f"{LIB_PATH} is not built; run `python -m newton_schulz_11_b200.build` (nvcc, sm_100a)")
        try:
            h = ctypes.CDLL(LIB_PATH)
        except OSError as e:  # pragma: no cover - depends on the machine
            raise MuonLibraryError(f"cannot load {LIB_PATH}: {e}") from e
        P = ctypes.POINTER
        h.muon_abi_version.restype = ctypes.c_int
        if h.muon_abi_version() != MUON_ABI_VERSION:
            raise MuonLibraryError(f"{LIB_PATH} implements ABI version {h.muon_abi_version()}, these bindings "
                                   f"version {MUON_ABI_VERSION}; rebuild with `python -m newton_schulz_11_b200.build`")
        h.muon_status_str.restype = ctypes.c_char_p
        h.muon_status_str.argtypes = [ctypes.c_int]
        h.muon_workspace_size.restype = ctypes.c_int
        h.muon_workspace_size.argtypes = [P(MuonMatrix), ctypes.c_int, P(ctypes.c_size_t)]
        h.muon_workspace_init.restype = ctypes.c_int
        h.muon_workspace_init.argtypes = [ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]
        h.muon_step.restype = ctypes.c_int
        h.muon_step.argtypes = [P(MuonMatrix), ctypes.c_int, ctypes.c_float, ctypes.c_float, ctypes.c_float,
                                ctypes.c_int, ctypes.c_int, P(ctypes.c_float), ctypes.c_float,
                                ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]
        h.muon_newton_schulz.restype = ctypes.c_int
        h.muon_newton_schulz.argtypes = [P(MuonMatrix), ctypes.c_int, ctypes.c_int, P(ctypes.c_float),
                                         ctypes.c_float, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]
        h.muon_scratch_view.restype = ctypes.c_int
        h.muon_scratch_view.argtypes = [P(MuonMatrix), ctypes.c_int, ctypes.c_int, ctypes.c_size_t,
                                        P(MuonScratchView)]
        h.muon_device_status.restype = ctypes.c_int
        h.muon_device_status.argtypes = [ctypes.c_void_p, ctypes.c_void_p, P(ctypes.c_int32), P(ctypes.c_int32)]
        h.muon_nonfinite_count.restype = ctypes.c_int
        h.muon_nonfinite_count.argtypes = [ctypes.c_void_p, ctypes.c_void_p, P(ctypes.c_int64)]
        h.muon_set_wait_timeout_us.restype = ctypes.c_int
        h.muon_set_wait_timeout_us.argtypes = [ctypes.c_int64]
        h.muon_profile_begin.restype = ctypes.c_int
        h.muon_profile_begin.argtypes = []
        h.muon_profile_end.restype = ctypes.c_int
        h.muon_profile_end.argtypes = [P(ctypes.c_double), P(ctypes.c_int64), ctypes.c_int]
        h.muon_adamw_step.restype = ctypes.c_int
        h.muon_adamw_step.argtypes = [P(MuonAdamwTensor), ctypes.c_int, ctypes.c_float, ctypes.c_float,
                                      ctypes.c_float, ctypes.c_float, ctypes.c_float, ctypes.c_int64,
                                      ctypes.c_void_p]
        h.muon_newton_schulz_static.restype = ctypes.c_int
        h.muon_newton_schulz_static.argtypes = [P(MuonMatrix), ctypes.c_int, ctypes.c_int, P(ctypes.c_float),
                                                ctypes.c_float, ctypes.c_void_p, ctypes.c_void_p]
        _lib = h
        return h


def status_str(status: int) -> str:
    try:
        return lib().muon_status_str(int(status)).decode()
    except MuonLibraryError:
        return "unknown"


def check(status: int, where: str) -> None:
    if status != MUON_OK:
        raise MuonError(status, where)
