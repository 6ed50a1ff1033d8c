"""A numpy model of the CUDA path's rounding points in the Newton-Schulz iteration.

Test infrastructure, like the oracle: it explains the tolerances the GPU parity tests use
for the two cases where bf16 tensor-core operands cannot meet the 2e-2 bar.  It imports
neither the kernels nor the oracle; every rounding point is restated here from the kernel's
documented numerics ("NanoGPT Speedrun" README, zeroth_power_via_newtonschulz5 listing, run
in bfloat16 as the README's list of practices prescribes; the hi + lo carry of X is this
library's reading of that practice):

  * u is fp32.  X is carried as hi = bf16(x) (round to nearest even) plus an 8-bit
    fixed-point residual on the fp32 bit patterns: with d = bits(x) - bits(hi), the residual
    is k = floor((d + 2^8) / 2^9), and the carried value is the float with bits
    bits(hi) + 2^9 k.
  * s = 1 / (||u||_F + eps) in fp32.
  * Gram:        A = bf16(fp32(hi hi^T) * fp32(s^2))   (s^2 in iteration 0 only)
  * polynomial:  B = bf16(fma(c, fp32(A A), fp32(b A)))
  * apply:       x = s * fma(a, x_carried, fp32(B hi))  (s in iteration 0 only), split again
  * output:      O = x of the last iteration, fp32

Products of bf16 values are exact in fp32 and the tensor cores accumulate in fp32; the model
forms each product in fp64 and rounds it to fp32 once, which leaves out only the fp32
accumulation-order error (about sqrt(k) 2^-24 relative, far below the bf16 terms).
A tall matrix (rows > cols) runs the same recurrence on its transpose, as the listing does.
"""
from __future__ import annotations

import numpy as np


def bf16(x):
    """Round to the nearest bf16 value, ties to even (finite inputs)."""
    b = np.asarray(x, np.float32).view(np.uint32).astype(np.uint64)
    b = (b + 0x7FFF + ((b >> 16) & 1)) & 0xFFFF0000
    return b.astype(np.uint32).view(np.float32).astype(np.float64)


def f32(x):
    return np.asarray(x, np.float64).astype(np.float32).astype(np.float64)


def _bits(x):
    return np.asarray(x, np.float32).view(np.int32).astype(np.int64)


def carry(x):
    """(hi, the carried value) of the fp32 values x: the residual kept as k = floor((d + 2^8)
    / 2^9) on d = bits(x) - bits(hi), the carried value the float with bits bits(hi) + 2^9 k."""
    x = f32(x)
    hi = bf16(x)
    k = np.floor_divide(_bits(x) - _bits(hi) + 256, 512)
    carried = (_bits(hi) + 512 * k).astype(np.int32).view(np.float32).astype(np.float64)
    return hi, carried


def newton_schulz(G, coeffs, eps=1e-7):
    """O of the CUDA path's Newton-Schulz iteration, rounding point by rounding point."""
    u = f32(G)
    tall = u.shape[0] > u.shape[1]
    if tall:
        u = u.T
    s = float(f32(1.0 / (np.linalg.norm(u) + eps)))
    hi, x = carry(u)
    for k, (a, b, c) in enumerate(coeffs):
        a, b, c = float(f32(a)), float(f32(b)), float(f32(c))
        first = k == 0
        acc = f32(hi @ hi.T)
        A = bf16(f32(acc * f32(s * s))) if first else bf16(acc)
        B = bf16(f32(c * f32(A @ A) + f32(b * A)))
        y = f32(a * x + f32(B @ hi))
        if first:
            y = f32(s * y)
        if k + 1 < len(coeffs):
            hi, x = carry(y)
        else:
            x = y
    return x.T if tall else x
