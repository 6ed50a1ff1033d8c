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


def lo8_unit(hi):
    """2^(e' - 14) per element for a bf16-valued tensor hi, with e' its exponent raised to at
    least -113 (biased 14) -- the unit of the 8-bit lo part (include/muon_b200.h)."""
    E = (hi.float().contiguous().view(torch.int32) >> 23) & 0xFF
    # built from exponent bits: exactly 2^(e' - 14) (a pow() may be off in the last bit,
    # which moves exact ties of the rounding)
    return ((E.clamp(min=14) - 14) << 23).to(torch.int32).view(torch.float32).double().where(
        E > 14, torch.full_like(E, 2.0 ** -127, dtype=torch.float64))


def ws_lo8(ws_buf, offset, rows, cols, ld_bytes, hi):
    """The 8-bit lo part of X inside the workspace, as fp64 values (k * 2^(e' - 14)), and the
    residual integers k (stored byte - 64)."""
    raw = ws_buf[offset: offset + rows * ld_bytes].view(torch.uint8).reshape(rows, ld_bytes)[:, :cols]
    k = raw.double() - 64.0
    return k * lo8_unit(hi), k


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
