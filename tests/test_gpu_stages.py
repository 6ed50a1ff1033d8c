"""Each CUDA stage checked on its own, through the C ABI, by reading the workspace.

After muon_newton_schulz with one or two iterations the workspace still holds the
split input (hi/lo), the norm and scale, and the latest A, B and X.  Each product is
recomputed from those very bf16 values with torch fp32 matmuls, so a failure points
at one kernel (elementwise, Gram, polynomial or apply) and one orientation.
"""
import numpy as np
import pytest

from tests.gpu_util import bits32, require_gpu, rel_fro, to_np, torch, ws_lo8, ws_matrix, ws_scalar

pytestmark = pytest.mark.gpu

SHAPES = [
    (128, 128), (64, 192), (192, 64),        # square, wide, tall
    (256, 640), (640, 256),                  # several tiles each way
    (200, 136), (136, 200),                  # ragged tails (multiples of 8)
    (40, 72), (72, 40),                      # single partial tile
    (100, 37), (37, 100),                    # sides that are not multiples of 8
    (600, 704), (704, 600),                  # three diagonal pair tiles, the last ragged (staged)
    (1048, 1152), (1152, 1048),              # Gram side above 1024: the streamed variant
]


def run_ns(G, coeffs):
    from newton_schulz_11_b200 import api

    ws = api.Workspace(G.device)
    out = api.newton_schulz([G], coeffs=coeffs, workspace=ws)[0]
    torch.cuda.synchronize()
    view = api.scratch_view([tuple(G.shape)], 0, ws.nbytes)
    return out, ws, view


def scratch(ws, view, rows, cols, which_hi):
    m = min(rows, cols)
    hi = ws_matrix(ws.buf, view.x_hi_offset[which_hi], rows, cols, view.x_ld)
    lo, _ = ws_lo8(ws.buf, view.x_lo_offset, rows, cols, view.x_lo_ld, hi)
    lo = lo.float()
    A = ws_matrix(ws.buf, view.a_offset, m, m, view.a_ld)
    B = ws_matrix(ws.buf, view.b_offset, m, m, view.a_ld)
    s = ws_scalar(ws.buf, view.scale_offset)
    nrm = ws_scalar(ws.buf, view.norm_offset)
    return hi, lo, A, B, s, nrm


def gram_of(X_hi, tall):
    return X_hi.t() @ X_hi if tall else X_hi @ X_hi.t()


def apply_of(X_hi, B, tall):
    return X_hi @ B if tall else B @ X_hi


def assert_bf16_close(got, want, what, rel=2 ** -7):
    err = (got - want).abs().max().item()
    scale = want.abs().max().item()
    assert err <= rel * scale + 1e-30, f"{what}: max err {err:.3e} vs scale {scale:.3e}"


@pytest.mark.parametrize("shape", SHAPES, ids=[f"{r}x{c}" for r, c in SHAPES])
def test_one_iteration_stage_by_stage(shape):
    require_gpu()
    rows, cols = shape
    tall = rows > cols
    gen = torch.Generator(device="cuda").manual_seed(rows * 1000 + cols)
    G = torch.randn(shape, device="cuda", generator=gen) * 0.01
    G[: max(1, rows // 3)] *= 7.0
    a, b, c = 2.5, -1.25, 0.5
    O, ws, view = run_ns(G, [(a, b, c)])
    assert view.transposed == int(tall)
    hi, lo, A, B, s, nrm = scratch(ws, view, rows, cols, 0)

    # elementwise: hi = bf16(G) and lo = the 8-bit residual, exactly as the format states
    Gd = G.double()
    assert torch.equal(hi, G.to(torch.bfloat16).float())
    lo_val, q = ws_lo8(ws.buf, view.x_lo_offset, rows, cols, view.x_lo_ld, hi)
    d = bits32(G) - bits32(hi)  # |d| <= 2^15: rounding to bf16 rounds the bit pattern
    assert d.abs().max().item() <= 2 ** 15
    q_ref = torch.div(d + 256, 512, rounding_mode="floor")  # d rounded to a multiple of 2^9, halves up
    assert q_ref.abs().max().item() <= 64
    bad = q != q_ref
    if bad.any():
        i, j = [int(v) for v in bad.nonzero()[0]]
        raise AssertionError(f"8-bit lo differs from (bits(x) - bits(hi) + 2^8) >> 9 at {int(bad.sum())} "
                             f"elements, first ({i}, {j}): got {int(q[i, j])} want {int(q_ref[i, j])}, "
                             f"x {float(Gd[i, j])!r} hi {float(hi[i, j])!r}")
    # the float with bits bits(hi) + 2^9 k is within 2^8 fp32 ulps (2^-15 relative) of the input
    assert ((hi.double() + lo_val) - Gd).abs().le(2 ** -15 * Gd.abs() + 1e-38).all()
    assert abs(nrm - Gd.norm().item()) <= 1e-6 * Gd.norm().item()
    assert abs(s - 1.0 / (Gd.norm().item() + 1e-7)) <= 1e-6 * s

    # Gram: A = s^2 hi hi^T (or hi^T hi for tall)
    A_ref = (s * s) * gram_of(hi, tall)
    assert_bf16_close(A, A_ref, f"Gram {shape}")
    assert torch.equal(A, A.t()), "Gram is not exactly symmetric"

    # polynomial: B = b A + c A A from the stored A
    B_ref = b * A + c * (A @ A)
    assert_bf16_close(B, B_ref, f"poly {shape}")
    assert torch.equal(B, B.t()), "polynomial is not exactly symmetric"

    # apply (last): O = s (a (hi + lo) + B hi)
    O_ref = s * (a * (hi + lo) + apply_of(hi, B, tall))
    err = rel_fro(to_np(O), to_np(O_ref))
    assert err < 1e-5, f"apply {shape}: rel err {err:.3e}"


@pytest.mark.parametrize("shape", [(128, 384), (384, 128), (136, 200)], ids=["wide", "tall", "ragged"])
def test_two_iterations_ping_pong(shape):
    """Iteration 1 reads the hi buffer the first apply wrote, and lo in place."""
    require_gpu()
    rows, cols = shape
    tall = rows > cols
    gen = torch.Generator(device="cuda").manual_seed(7 + rows)
    G = torch.randn(shape, device="cuda", generator=gen)
    coeffs = [(3.4445, -4.7750, 2.0315), (2.0, -1.5, 0.5)]
    O, ws, view = run_ns(G, coeffs)
    hi1, lo1, A, B, s, _ = scratch(ws, view, rows, cols, 1)
    a, b, c = coeffs[1]
    A_ref = gram_of(hi1, tall)
    assert_bf16_close(A, A_ref, "Gram, iteration 1")
    assert_bf16_close(B, b * A + c * (A @ A), "poly, iteration 1")
    O_ref = a * (hi1 + lo1) + apply_of(hi1, B, tall)
    assert rel_fro(to_np(O), to_np(O_ref)) < 1e-5
    # X1 itself: hi1 + lo1 equals the first iteration's result recomputed from G
    hi0 = ws_matrix(ws.buf, view.x_hi_offset[0], rows, cols, view.x_ld)
    a0, b0, c0 = coeffs[0]
    A0 = (s * s) * gram_of(hi0, tall)
    B0 = b0 * A0 + c0 * (A0 @ A0)
    X1 = s * (a0 * G + apply_of(hi0, B0, tall))
    assert rel_fro(to_np(hi1 + lo1), to_np(X1)) < 2e-2
