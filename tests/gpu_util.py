"""Helpers shared by the GPU tests: device guard, workspace readers, oracle adapters."""
import math

import numpy as np
import pytest

torch = pytest.importorskip("torch")


def require_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    major, minor = torch.cuda.get_device_capability()
    if (major, minor) != (10, 0):
        pytest.skip(f"needs an sm_100 GPU, found sm_{major}{minor}")
    from newton_schulz_11_b200 import build

    build.build()


def ws_matrix(ws_buf, offset, rows, cols, ld, dtype=torch.bfloat16):
    """View a row-major matrix inside the uint8 workspace tensor as fp32."""
    esz = torch.tensor([], dtype=dtype).element_size()
    nbytes = rows * ld * esz
    raw = ws_buf[offset: offset + nbytes]
    return raw.view(dtype).reshape(rows, ld)[:, :cols].float()


def bits32(x):
    """fp32 bit patterns of a float tensor, as int64 (signed, so differences are exact)."""
    return x.float().contiguous().view(torch.int32).long()


def ws_lo8(ws_buf, offset, rows, cols, ld_bytes, hi):
    """The 8-bit lo part of X inside the workspace (include/muon_b200.h): the stored bytes
    minus 64, k, and the value hi + lo they encode, as fp64 -- the float whose bit pattern
    is bits(hi) + 2^9 k."""
    raw = ws_buf[offset: offset + rows * ld_bytes].view(torch.uint8).reshape(rows, ld_bytes)[:, :cols]
    k = raw.long() - 64
    x = (bits32(hi) + k * 512).to(torch.int32).view(torch.float32).double()
    return x - hi.double(), k


def ws_scalar(ws_buf, offset):
    return float(ws_buf[offset: offset + 4].view(torch.float32)[0])


def rel_fro(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def to_np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def bf16_ulp(x):
    """Spacing of bf16 numbers at |x| (for normal numbers)."""
    x = np.abs(np.asarray(x, np.float64))
    e = np.floor(np.log2(np.maximum(x, 1e-38)))
    return np.exp2(e - 7)
