"""PyTorch-facing binding: turns tensors into muon_matrix_t descriptors and calls the C ABI.

Only argument marshalling happens here; every step of the Muon update runs in
libmuon_b200.so.  PyTorch provides the device memory and the current stream.
"""
from __future__ import annotations

import ctypes
from typing import List, Optional, Sequence, Tuple

import torch

from . import _lib
from ._lib import MUON_BF16, MUON_F32, MuonAdamwTensor, MuonError, MuonLibraryError, MuonMatrix, MuonScratchView, check, lib  # noqa: F401,E501

# "NanoGPT Speedrun" README, zeroth_power_via_newtonschulz5 listing: (a, b, c), 5 steps, eps.
QUINTIC = (3.4445, -4.7750, 2.0315)
DEFAULT_STEPS = 5
DEFAULT_EPS = 1e-7


def quintic_table(steps: int = DEFAULT_STEPS) -> List[Tuple[float, float, float]]:
    return [QUINTIC] * steps


def _coeff_array(coeffs) -> Tuple[ctypes.Array, int]:
    rows = [tuple(float(v) for v in r) for r in coeffs]
    if not rows or any(len(r) != 3 for r in rows):
        raise ValueError("coeffs must be a non-empty sequence of (a, b, c) rows")
    flat = (ctypes.c_float * (3 * len(rows)))(*[v for r in rows for v in r])
    return flat, len(rows)


def _check_2d(t: torch.Tensor, what: str, dtypes) -> None:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{what} must be a torch.Tensor")
    if t.dim() != 2:
        raise ValueError(f"{what} must be 2-D (Muon orthogonalises matrices only), got shape {tuple(t.shape)}")
    if t.dtype not in dtypes:
        raise TypeError(f"{what} has dtype {t.dtype}, expected one of {dtypes}")
    if not t.is_cuda:
        raise ValueError(f"{what} must live on a CUDA device")
    if t.stride(1) != 1 and t.shape[1] > 1:
        raise ValueError(f"{what} must have unit stride along its last dimension")


def _ld(t: torch.Tensor) -> int:
    return t.stride(0) if t.shape[0] > 1 else t.shape[1]


def _descriptors(params, grads, moms, outs, shape_scales, ns_only: bool) -> ctypes.Array:
    n = len(grads)
    arr = (MuonMatrix * n)()
    dev = grads[0].device
    for i in range(n):
        g = grads[i]
        _check_2d(g, f"grads[{i}]", (torch.float32,))
        if g.device != dev:
            raise ValueError("all tensors must be on the same device")
        d = arr[i]
        d.rows, d.cols = g.shape
        d.grad = g.data_ptr()
        d.ld_grad = _ld(g)
        d.shape_scale = 0.0 if shape_scales is None or shape_scales[i] is None else float(shape_scales[i])
        if outs is not None and outs[i] is not None:
            o = outs[i]
            _check_2d(o, f"outs[{i}]", (torch.float32,))
            if tuple(o.shape) != tuple(g.shape) or not o.is_contiguous():
                raise ValueError(f"outs[{i}] must be a contiguous fp32 tensor of shape {tuple(g.shape)}")
            d.out_update = o.data_ptr()
        if ns_only:
            d.param_dtype = _lib.MUON_F32
            continue
        p, m = params[i], moms[i]
        _check_2d(p, f"params[{i}]", (torch.float32, torch.bfloat16))
        _check_2d(m, f"moms[{i}]", (torch.float32,))
        if tuple(p.shape) != tuple(g.shape) or tuple(m.shape) != tuple(g.shape):
            raise ValueError(f"params[{i}], grads[{i}] and moms[{i}] must have the same shape")
        if p.device != dev or m.device != dev:
            raise ValueError("all tensors must be on the same device")
        d.param = p.data_ptr()
        d.param_dtype = _lib.MUON_BF16 if p.dtype == torch.bfloat16 else _lib.MUON_F32
        d.ld_param = _ld(p)
        d.momentum = m.data_ptr()
        d.ld_mom = _ld(m)
    return arr


class Workspace:
    """Device scratch owned by the caller (PyTorch memory), grown on demand, one per device."""

    def __init__(self, device):
        self.device = torch.device(device)
        self.buf: Optional[torch.Tensor] = None

    @property
    def nbytes(self) -> int:
        return 0 if self.buf is None else self.buf.numel()

    def ensure(self, nbytes: int, stream: int) -> Tuple[int, int]:
        if self.buf is None or self.buf.numel() < nbytes:
            self.buf = None
            self.buf = torch.empty(int(nbytes), dtype=torch.uint8, device=self.device)
            check(lib().muon_workspace_init(self.buf.data_ptr(), self.buf.numel(), stream), "muon_workspace_init")
        return self.buf.data_ptr(), self.buf.numel()


_workspaces = {}


def default_workspace(device) -> Workspace:
    device = torch.device(device)
    key = device.index if device.index is not None else torch.cuda.current_device()
    ws = _workspaces.get(key)
    if ws is None:
        ws = _workspaces[key] = Workspace(torch.device("cuda", key))
    return ws


def workspace_size(shapes: Sequence[Tuple[int, int]]) -> int:
    n = len(shapes)
    arr = (MuonMatrix * n)()
    for i, (r, c) in enumerate(shapes):
        arr[i].rows, arr[i].cols = int(r), int(c)
    out = ctypes.c_size_t(0)
    check(lib().muon_workspace_size(arr, n, ctypes.byref(out)), "muon_workspace_size")
    return int(out.value)


def _stream_handle(device, stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return int(stream.cuda_stream)


def muon_step(params: Sequence[torch.Tensor], grads: Sequence[torch.Tensor], moms: Sequence[torch.Tensor], *,
              lr: float, beta: float = 0.95, weight_decay: float = 0.0, nesterov: bool = True,
              coeffs=None, eps: float = DEFAULT_EPS, shape_scales=None, outs=None,
              workspace: Optional[Workspace] = None, workspace_bytes: Optional[int] = None, stream=None) -> None:
    """One grouped Muon step, in place on params and moms (see include/muon_b200.h).

    ``outs`` (optional, fp32, same shapes) receives the orthogonalised update O.
    ``workspace_bytes`` caps the scratch used (fewer bytes -> more waves).
    """
    if not (len(params) == len(grads) == len(moms)) or len(grads) == 0:
        raise ValueError("params, grads and moms must be equally long, non-empty lists")
    table, steps = _coeff_array(coeffs if coeffs is not None else quintic_table())
    device = grads[0].device
    arr = _descriptors(params, grads, moms, outs, shape_scales, ns_only=False)
    n = len(grads)
    h = lib()
    need = ctypes.c_size_t(0)
    check(h.muon_workspace_size(arr, n, ctypes.byref(need)), "muon_workspace_size")
    s = _stream_handle(device, stream)
    ws = workspace or default_workspace(device)
    want = int(need.value) if workspace_bytes is None else int(workspace_bytes)
    ptr, size = ws.ensure(want, s)
    check(h.muon_step(arr, n, float(lr), float(beta), float(weight_decay), 1 if nesterov else 0, steps, table,
                      float(eps), ptr, min(size, want), s), "muon_step")


def newton_schulz(Gs: Sequence[torch.Tensor], *, coeffs=None, eps: float = DEFAULT_EPS, outs=None,
                  workspace: Optional[Workspace] = None, workspace_bytes: Optional[int] = None,
                  stream=None) -> List[torch.Tensor]:
    """zeroth_power_via_newtonschulz5 on each fp32 matrix of Gs, grouped; returns fp32 O's."""
    Gs = list(Gs)
    if not Gs:
        raise ValueError("Gs must be a non-empty list")
    if outs is None:
        outs = [torch.empty_like(g) for g in Gs]
    table, steps = _coeff_array(coeffs if coeffs is not None else quintic_table())
    device = Gs[0].device
    arr = _descriptors(None, Gs, None, outs, None, ns_only=True)
    n = len(Gs)
    h = lib()
    need = ctypes.c_size_t(0)
    check(h.muon_workspace_size(arr, n, ctypes.byref(need)), "muon_workspace_size")
    s = _stream_handle(device, stream)
    ws = workspace or default_workspace(device)
    want = int(need.value) if workspace_bytes is None else int(workspace_bytes)
    ptr, size = ws.ensure(want, s)
    check(h.muon_newton_schulz(arr, n, steps, table, float(eps), ptr, min(size, want), s), "muon_newton_schulz")
    return outs


def newton_schulz_static(Gs: Sequence[torch.Tensor], *, coeffs=None, eps: float = DEFAULT_EPS, outs=None,
                         device_status: Optional[torch.Tensor] = None, stream=None) -> List[torch.Tensor]:
    """newton_schulz with the library's static device scratch in place of a workspace.

    For callers that cannot allocate device memory of their own.  `outs` (if given) and
    `device_status` (an int32 tensor of 2, device or pinned host) are the only buffers
    written; nothing is allocated on the device when `outs` is given.
    """
    Gs = list(Gs)
    if not Gs:
        raise ValueError("Gs must be a non-empty list")
    if outs is None:
        outs = [torch.empty_like(g) for g in Gs]
    table, steps = _coeff_array(coeffs if coeffs is not None else quintic_table())
    device = Gs[0].device
    arr = _descriptors(None, Gs, None, outs, None, ns_only=True)
    st_ptr = None
    if device_status is not None:
        if device_status.dtype != torch.int32 or device_status.numel() < 2 or not device_status.is_contiguous():
            raise ValueError("device_status must be a contiguous int32 tensor of at least 2 elements")
        st_ptr = device_status.data_ptr()
    s = _stream_handle(device, stream)
    check(lib().muon_newton_schulz_static(arr, len(Gs), steps, table, float(eps), st_ptr, s),
          "muon_newton_schulz_static")
    return outs


def _adamw_descriptors(params, grads, exp_avgs, exp_avg_sqs):
    params, grads, exp_avgs, exp_avg_sqs = list(params), list(grads), list(exp_avgs), list(exp_avg_sqs)
    n = len(params)
    if n == 0 or not (len(grads) == len(exp_avgs) == len(exp_avg_sqs) == n):
        raise ValueError("params, grads, exp_avgs and exp_avg_sqs must be non-empty lists of equal length")
    device = params[0].device
    arr = (MuonAdamwTensor * n)()
    for i, (p, g, m, v) in enumerate(zip(params, grads, exp_avgs, exp_avg_sqs)):
        for t, what in ((p, "param"), (g, "grad"), (m, "exp_avg"), (v, "exp_avg_sq")):
            if t.device != device or t.device.type != "cuda":
                raise ValueError(f"{what} {i} is not on {device}")
            if not t.is_contiguous():
                raise ValueError(f"{what} {i} must be contiguous")
            if t.numel() != p.numel():
                raise ValueError(f"{what} {i} has {t.numel()} elements, param has {p.numel()}")
        if p.dtype not in (torch.float32, torch.bfloat16):
            raise ValueError(f"param {i} must be float32 or bfloat16")
        for t, what in ((g, "grad"), (m, "exp_avg"), (v, "exp_avg_sq")):
            if t.dtype != torch.float32:
                raise ValueError(f"{what} {i} must be float32")
        arr[i].param = p.data_ptr()
        arr[i].grad = g.data_ptr()
        arr[i].exp_avg = m.data_ptr()
        arr[i].exp_avg_sq = v.data_ptr()
        arr[i].numel = p.numel()
        arr[i].param_dtype = MUON_BF16 if p.dtype == torch.bfloat16 else MUON_F32
    return arr, n, device


def adamw_step(params: Sequence[torch.Tensor], grads: Sequence[torch.Tensor], exp_avgs: Sequence[torch.Tensor],
               exp_avg_sqs: Sequence[torch.Tensor], *, lr: float, step: int, betas=(0.9, 0.999),
               eps: float = 1e-8, weight_decay: float = 0.0, stream=None) -> None:
    """AdamW on a grouped list of contiguous tensors (the parameters Muon does not take).

    params fp32 or bf16; grads, exp_avgs, exp_avg_sqs fp32 of the same numel; `step` is the
    1-based count of updates including this one.  One launch per 128 tensors.  For a fixed
    set of tensors stepped repeatedly, PreparedAdamW avoids rebuilding the descriptors.
    """
    arr, n, device = _adamw_descriptors(params, grads, exp_avgs, exp_avg_sqs)
    b1, b2 = betas
    check(lib().muon_adamw_step(arr, n, float(lr), float(b1), float(b2), float(eps), float(weight_decay),
                                int(step), _stream_handle(device, stream)), "muon_adamw_step")


class PreparedMuonStep:
    """muon_step for a fixed set of tensors: the descriptor array, coefficient table and
    workspace are built once, so each call is one C ABI call (no per-call Python checks).
    The tensors must keep their storage (same data pointers) between calls."""

    def __init__(self, params, grads, moms, *, lr: float, beta: float = 0.95, weight_decay: float = 0.0,
                 nesterov: bool = True, coeffs=None, eps: float = DEFAULT_EPS, shape_scales=None, outs=None,
                 workspace: Optional[Workspace] = None):
        if not (len(params) == len(grads) == len(moms)) or len(grads) == 0:
            raise ValueError("params, grads and moms must be equally long, non-empty lists")
        self._keep = (list(params), list(grads), list(moms), None if outs is None else list(outs))
        self._arr = _descriptors(params, grads, moms, outs, shape_scales, ns_only=False)
        self._n = len(grads)
        self._table, self._steps = _coeff_array(coeffs if coeffs is not None else quintic_table())
        self.device = grads[0].device
        need = ctypes.c_size_t(0)
        check(lib().muon_workspace_size(self._arr, self._n, ctypes.byref(need)), "muon_workspace_size")
        self._ws = workspace or default_workspace(self.device)
        self._ptr, size = self._ws.ensure(int(need.value), _stream_handle(self.device, None))
        # the buffer this step was prepared on stays alive even if the shared workspace is
        # later grown (and its old buffer dropped) for a larger step
        self._buf = self._ws.buf
        self._bytes = min(size, int(need.value))
        self._hyper = (float(lr), float(beta), float(weight_decay), 1 if nesterov else 0)
        self._eps = float(eps)
        self._fn = lib().muon_step

    def __call__(self, stream=None) -> None:
        lr, beta, wd, nest = self._hyper
        st = self._fn(self._arr, self._n, lr, beta, wd, nest, self._steps, self._table, self._eps, self._ptr,
                      self._bytes, _stream_handle(self.device, stream))
        if st != 0:
            check(st, "muon_step")

    @property
    def workspace(self) -> Workspace:
        return self._ws

    def device_status(self, stream=None) -> Tuple[int, int]:
        """(code, where) of the device-side status word in this step's own workspace buffer
        (synchronises the stream)."""
        code, where = ctypes.c_int32(0), ctypes.c_int32(0)
        check(lib().muon_device_status(self._ptr, _stream_handle(self.device, stream), ctypes.byref(code),
                                       ctypes.byref(where)), "muon_device_status")
        return int(code.value), int(where.value)

    def nonfinite_count(self, stream=None) -> int:
        """Non-finite values of u counted in this step's workspace since it was cleared."""
        n = ctypes.c_int64(0)
        check(lib().muon_nonfinite_count(self._ptr, _stream_handle(self.device, stream), ctypes.byref(n)),
              "muon_nonfinite_count")
        return int(n.value)


class PreparedAdamW:
    """adamw_step for a fixed set of contiguous tensors: the descriptor array is built and
    checked once; each call passes the 1-based step count to one C ABI call."""

    def __init__(self, params, grads, exp_avgs, exp_avg_sqs, *, lr: float, betas=(0.9, 0.999),
                 eps: float = 1e-8, weight_decay: float = 0.0):
        self._keep = (list(params), list(grads), list(exp_avgs), list(exp_avg_sqs))
        self._arr, self._n, self.device = _adamw_descriptors(*self._keep)
        self._hyper = (float(lr), float(betas[0]), float(betas[1]), float(eps), float(weight_decay))
        self._fn = lib().muon_adamw_step

    def __call__(self, step: int, stream=None) -> None:
        lr, b1, b2, eps, wd = self._hyper
        st = self._fn(self._arr, self._n, lr, b1, b2, eps, wd, int(step), _stream_handle(self.device, stream))
        if st != 0:
            check(st, "muon_adamw_step")


def head_blocks(W: torch.Tensor, head_dim: int, heads_per_block: int = 2, dim: int = 0) -> List[torch.Tensor]:
    """Views of W split into blocks of `heads_per_block` heads along `dim` (0: the rows of a
    Q/K/V projection, 1: the columns of the output projection).  Each block is a strided
    2-D view of W's storage (no copy), so a grouped muon_step over the blocks orthogonalises
    every block as its own matrix and updates W in place -- per-head (heads_per_block=1)
    or paired-head (2) Muon."""
    if W.dim() != 2:
        raise ValueError("W must be 2-D")
    size = head_dim * heads_per_block
    if W.shape[dim] % size:
        raise ValueError(f"dimension {dim} of W ({W.shape[dim]}) is not a multiple of {size}")
    return list(torch.split(W, size, dim=dim))


def scratch_view(shapes: Sequence[Tuple[int, int]], index: int, workspace_bytes: int) -> MuonScratchView:
    n = len(shapes)
    arr = (MuonMatrix * n)()
    for i, (r, c) in enumerate(shapes):
        arr[i].rows, arr[i].cols = int(r), int(c)
    v = MuonScratchView()
    check(lib().muon_scratch_view(arr, n, int(index), int(workspace_bytes), ctypes.byref(v)), "muon_scratch_view")
    return v


def device_status(workspace: Workspace, stream=None) -> Tuple[int, int]:
    code, where = ctypes.c_int32(0), ctypes.c_int32(0)
    s = _stream_handle(workspace.device, stream)
    check(lib().muon_device_status(workspace.buf.data_ptr(), s, ctypes.byref(code), ctypes.byref(where)),
          "muon_device_status")
    return int(code.value), int(where.value)


def nonfinite_count(workspace: Workspace, stream=None) -> int:
    """Non-finite values of u (or G) counted in `workspace` since it was last cleared."""
    n = ctypes.c_int64(0)
    check(lib().muon_nonfinite_count(workspace.buf.data_ptr(), _stream_handle(workspace.device, stream),
                                     ctypes.byref(n)), "muon_nonfinite_count")
    return int(n.value)


def clear_device_status(workspace: Workspace, stream=None) -> None:
    """Clears the status word and the non-finite count of `workspace` (queued on the stream)."""
    check(lib().muon_workspace_init(workspace.buf.data_ptr(), workspace.buf.numel(),
                                    _stream_handle(workspace.device, stream)), "muon_workspace_init")
