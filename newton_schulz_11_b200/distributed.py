"""Data-parallel Muon across GPUs: each matrix's momentum and Newton-Schulz work live on
one owner rank; the owners then broadcast the updated parameters.

"Do You Know About NanoGPT Speedrun?" (the list of things that did not work, on DiLoCo)
notes that with several GPUs Muon's matrix multiplications are spread over the GPUs layer
by layer, and the "NanoGPT Speedrun" record table names a distributed Muon record.  The
reading taken here: every rank holds all parameters; the step of a matrix runs on its
owner alone, so only the owner needs that matrix's data-parallel gradient, and every rank
needs the updated parameters.

  owners  = longest-processing-time assignment of the matrices to ranks by Newton-Schulz
            flops (3 m^2 n + m^3 per iteration), ties to the lower rank
  waves   = each rank's owned matrices, by decreasing cost, dealt round-robin into
            `waves` groups; wave j of every rank forms one phase of the pipeline
  reduce  = (reduce_grads=True) per phase and owner, every rank packs its local gradients
            of the owner's matrices into one flat fp32 buffer and the buffers are averaged
            onto the owner -- a reduce-scatter with uneven shards.  With reduce_grads=False
            the gradients are taken as already averaged (as after a DDP all-reduce).
  step    = per phase, one grouped muon_step over the owned matrices of that wave (their
            momentum buffers are only read or written on the owner)
  gather  = per phase, owner and parameter dtype, the owner packs its updated parameters
            into one flat buffer and broadcasts it -- an all-gather with uneven shards; the
            others unpack it into their copies once every broadcast is done

The collectives are issued asynchronously in one fixed order on every rank (all reduces,
then the broadcasts phase by phase), so phase j's broadcasts overlap phase j+1's step.
torch.distributed carries them (NCCL on GPUs, gloo on CPU for tests); all arithmetic of
the Muon step runs in the library's kernels.  Flat-buffer offsets are padded to 64
elements so every view keeps the 16-byte alignment the library asks for.
"""
from __future__ import annotations

from typing import Callable, Dict, List, Optional, Sequence, Tuple

import torch
import torch.distributed as dist

_PAD = 64  # elements: flat-buffer offsets stay 256-byte aligned for fp32, 128 for bf16


def ns_flops(rows: int, cols: int, steps: int = 5) -> float:
    """Algorithmic Newton-Schulz flops of one matrix: (3 m^2 n + m^3) per iteration."""
    m, n = min(rows, cols), max(rows, cols)
    return float(steps) * (3.0 * m * m * n + float(m) ** 3)


def partition_lpt(costs: Sequence[float], world: int) -> List[int]:
    """Owner rank of each item: items by decreasing cost (stable), each to the rank with the
    least load so far (lowest rank on ties).  Deterministic, so every rank computes it."""
    if world < 1:
        raise ValueError("world must be >= 1")
    load = [0.0] * world
    owner = [0] * len(costs)
    for i in sorted(range(len(costs)), key=lambda k: (-costs[k], k)):
        r = min(range(world), key=lambda q: (load[q], q))
        owner[i] = r
        load[r] += costs[i]
    return owner


def assign_waves(costs: Sequence[float], owners: Sequence[int], waves: int) -> List[int]:
    """Wave of each item: per owner, its items by decreasing cost (stable) dealt round-robin
    over the waves, so every wave of a rank carries about 1/waves of its load."""
    if waves < 1:
        raise ValueError("waves must be >= 1")
    wave = [0] * len(costs)
    for r in sorted(set(owners)):
        mine = sorted((i for i, o in enumerate(owners) if o == r), key=lambda k: (-costs[k], k))
        for k, i in enumerate(mine):
            wave[i] = k % waves
    return wave


class _Flat:
    """One flat buffer with a padded (rows, cols) view per matrix."""

    def __init__(self, shapes: Sequence[Tuple[int, int]], dtype: torch.dtype, device: torch.device):
        offs, n = [], 0
        for r, c in shapes:
            offs.append(n)
            n += -(-(r * c) // _PAD) * _PAD
        self.buf = torch.zeros(max(n, 1), dtype=dtype, device=device)
        self.views = [self.buf[o:o + r * c].view(r, c) for o, (r, c) in zip(offs, shapes)]

    def pack(self, src: Sequence[torch.Tensor]) -> None:
        torch._foreach_copy_(self.views, list(src))

    def unpack(self, dst: Sequence[torch.Tensor]) -> None:
        torch._foreach_copy_(list(dst), self.views)


class ShardedMuon:
    """One Muon step over all matrices of a data-parallel model, the work split over ranks.

    `local_step(indices, grads)` performs the step for the matrices with those indices (in
    place on params[i] and moms[i]), reading the gradient of indices[k] from grads[k] (the
    averaged gradient when reduce_grads is set, else the caller's tensor); by default one
    PreparedMuonStep per wave over the owned matrices with the given hyperparameters.
    Every rank must construct it with the same shapes, in the same order, and call it
    collectively.
    """

    def __init__(self, params: Sequence[torch.Tensor], grads: Sequence[torch.Tensor], moms: Sequence[torch.Tensor],
                 *, group: Optional[dist.ProcessGroup] = None, ns_steps: int = 5, reduce_grads: bool = False,
                 waves: int = 1, local_step: Optional[Callable[[List[int], List[torch.Tensor]], None]] = None,
                 **hyper):
        if not (len(params) == len(grads) == len(moms)) or not params:
            raise ValueError("params, grads and moms must be equally long, non-empty lists")
        self.params, self.grads = list(params), list(grads)
        self.group = group
        self.world = dist.get_world_size(group) if dist.is_initialized() else 1
        self.rank = dist.get_rank(group) if dist.is_initialized() else 0
        self.reduce_grads = bool(reduce_grads) and self.world > 1
        costs = [ns_flops(*p.shape, steps=ns_steps) for p in self.params]
        self.owners = partition_lpt(costs, self.world)
        self.waves = max(1, min(int(waves), max(sum(1 for o in self.owners if o == r) for r in range(self.world))))
        self.wave_of = assign_waves(costs, self.owners, self.waves)
        self.owned = [i for i, o in enumerate(self.owners) if o == self.rank]
        dev = self.params[0].device
        shape = lambda i: tuple(self.params[i].shape)  # noqa: E731

        # per phase and owner: the gradient bucket (reduce_grads only)
        self._gbuckets: Dict[Tuple[int, int], Tuple[List[int], _Flat]] = {}
        if self.reduce_grads:
            for j in range(self.waves):
                for r in range(self.world):
                    idx = [i for i in range(len(self.params)) if self.owners[i] == r and self.wave_of[i] == j]
                    if idx:
                        self._gbuckets[(j, r)] = (idx, _Flat([shape(i) for i in idx], torch.float32, dev))
        # gradients the local step reads, per wave of this rank
        self.wave_idx: List[List[int]] = []
        self.wave_grads: List[List[torch.Tensor]] = []
        for j in range(self.waves):
            idx = [i for i in self.owned if self.wave_of[i] == j]
            if self.reduce_grads and idx:
                gidx, flat = self._gbuckets[(j, self.rank)]
                assert gidx == idx
                g = list(flat.views)
            else:
                g = [self.grads[i] for i in idx]
            self.wave_idx.append(idx)
            self.wave_grads.append(g)

        if local_step is None:
            local_step = self._default_local_step(moms, hyper)
        self.local_step = local_step

        # per phase, owner and parameter dtype: the broadcast bucket
        self.plan: List[Tuple[int, int, torch.dtype, List[int], int]] = []
        self._pbuckets: List[_Flat] = []
        if self.world > 1:
            for j in range(self.waves):
                for r in range(self.world):
                    mine = [i for i in range(len(self.params)) if self.owners[i] == r and self.wave_of[i] == j]
                    for dtype in sorted({self.params[i].dtype for i in mine}, key=str):
                        idx = [i for i in mine if self.params[i].dtype == dtype]
                        self.plan.append((j, r, dtype, idx, sum(self.params[i].numel() for i in idx)))
                        self._pbuckets.append(_Flat([shape(i) for i in idx], dtype, dev))

    def _default_local_step(self, moms, hyper):
        from .api import PreparedMuonStep, default_workspace, workspace_size

        steps = {}
        if self.owned:
            dev = self.params[self.owned[0]].device
            need = max(workspace_size([tuple(self.params[i].shape) for i in idx]) for idx in self.wave_idx if idx)
            ws = hyper.pop("workspace", None) or default_workspace(dev)
            ws.ensure(need, torch.cuda.current_stream(dev).cuda_stream)  # one buffer for every wave
            for j, idx in enumerate(self.wave_idx):
                if idx:
                    steps[tuple(idx)] = PreparedMuonStep([self.params[i] for i in idx], self.wave_grads[j],
                                                         [moms[i] for i in idx], workspace=ws, **hyper)

        def run(idx, grads):
            steps[tuple(idx)]()

        return run

    def load(self) -> List[float]:
        """Newton-Schulz flops assigned to each rank."""
        out = [0.0] * self.world
        for i, r in enumerate(self.owners):
            out[r] += ns_flops(*self.params[i].shape)
        return out

    def _global(self, r: int) -> int:
        return r if self.group is None else dist.get_global_rank(self.group, r)

    def __call__(self) -> None:
        if self.world == 1:
            for idx, g in zip(self.wave_idx, self.wave_grads):
                if idx:
                    self.local_step(idx, g)
            return
        avg = self.reduce_grads and dist.get_backend(self.group) == "nccl"
        # 1. every gradient bucket, in (phase, owner) order, reduced onto its owner
        pending = {}
        for (j, r), (idx, flat) in self._gbuckets.items():
            flat.pack([self.grads[i] for i in idx])
            pending[(j, r)] = dist.reduce(flat.buf, dst=self._global(r), group=self.group, async_op=True,
                                          op=dist.ReduceOp.AVG if avg else dist.ReduceOp.SUM)
        # 2. phase by phase: the owned wave's step, then its parameter broadcasts
        sends = []
        for j in range(self.waves):
            if (j, self.rank) in pending:
                pending.pop((j, self.rank)).wait()
                if not avg:
                    self._gbuckets[(j, self.rank)][1].buf.div_(self.world)
            if self.wave_idx[j]:
                self.local_step(self.wave_idx[j], self.wave_grads[j])
            for (pj, owner, dtype, idx, numel), flat in zip(self.plan, self._pbuckets):
                if pj != j:
                    continue
                if owner == self.rank:
                    flat.pack([self.params[i] for i in idx])
                sends.append((owner, idx, flat,
                              dist.broadcast(flat.buf, src=self._global(owner), group=self.group, async_op=True)))
        for work in pending.values():  # reduces onto other owners: complete before the buffers are reused
            work.wait()
        for owner, idx, flat, work in sends:
            work.wait()
            if owner != self.rank:
                flat.unpack([self.params[i] for i in idx])
