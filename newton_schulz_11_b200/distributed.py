"""Data-parallel Muon across GPUs: each matrix's momentum and Newton-Schulz work live on
one owner rank; the owners then broadcast the updated parameters.

"Do You Know About NanoGPT Speedrun?" (the list of things that did not work, on DiLoCo)
notes that with several GPUs Muon's matrix multiplications are spread over the GPUs layer
by layer, and the "NanoGPT Speedrun" record table names a distributed Muon record.  The
reading taken here: every rank holds all parameters and the data-parallel average of the
gradients (as after the all-reduce of a DDP backward), so the step of a matrix needs no
input from other ranks; only its result does.

  owners  = longest-processing-time assignment of the matrices to ranks by Newton-Schulz
            flops (3 m^2 n + m^3 per iteration), ties to the lower rank
  step    = one grouped muon_step over the matrices this rank owns (their momentum
            buffers are only read or written on the owner)
  gather  = per owner and dtype, the owner packs its updated parameters into one flat
            buffer and broadcasts it; the others unpack it into their copies

torch.distributed carries the collectives (NCCL on GPUs, gloo on CPU for tests); all
arithmetic of the step runs in the library's kernels.
"""
from __future__ import annotations

from typing import Callable, List, Optional, Sequence

import torch
import torch.distributed as dist


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


class ShardedMuon:
    """One Muon step over all matrices of a data-parallel model, the work split over ranks.

    `local_step(indices)` performs the step for the matrices with those indices (in place on
    params[i] and moms[i]); by default a PreparedMuonStep over the owned matrices with the
    given hyperparameters.  Every rank must construct it with the same shapes, in the same
    order, and call it collectively.
    """

    def __init__(self, params: Sequence[torch.Tensor], grads: Sequence[torch.Tensor], moms: Sequence[torch.Tensor],
                 *, group: Optional[dist.ProcessGroup] = None, ns_steps: int = 5,
                 local_step: Optional[Callable[[List[int]], None]] = None, **hyper):
        if not (len(params) == len(grads) == len(moms)) or not params:
            raise ValueError("params, grads and moms must be equally long, non-empty lists")
        self.params = list(params)
        self.group = group
        self.world = dist.get_world_size(group) if dist.is_initialized() else 1
        self.rank = dist.get_rank(group) if dist.is_initialized() else 0
        self.owners = partition_lpt([ns_flops(*p.shape, steps=ns_steps) for p in self.params], self.world)
        self.owned = [i for i, o in enumerate(self.owners) if o == self.rank]
        if local_step is None:
            from .api import PreparedMuonStep

            prepared = (PreparedMuonStep([params[i] for i in self.owned], [grads[i] for i in self.owned],
                                         [moms[i] for i in self.owned], **hyper) if self.owned else None)
            local_step = (lambda idx: prepared()) if prepared is not None else (lambda idx: None)
        self.local_step = local_step
        # broadcast plan: per owner rank, per parameter dtype, the matrices in order
        self.plan = []
        for r in range(self.world):
            mine = [i for i, o in enumerate(self.owners) if o == r]
            for dtype in sorted({self.params[i].dtype for i in mine}, key=str):
                idx = [i for i in mine if self.params[i].dtype == dtype]
                self.plan.append((r, dtype, idx, sum(self.params[i].numel() for i in idx)))

    def load(self) -> List[float]:
        """Newton-Schulz flops assigned to each rank."""
        out = [0.0] * self.world
        for i, r in enumerate(self.owners):
            out[r] += ns_flops(*self.params[i].shape)
        return out

    def __call__(self) -> None:
        if self.owned:
            self.local_step(self.owned)
        if self.world == 1:
            return
        for owner, dtype, idx, numel in self.plan:
            dev = self.params[idx[0]].device
            if owner == self.rank:
                flat = torch.cat([self.params[i].reshape(-1) for i in idx])
            else:
                flat = torch.empty(numel, dtype=dtype, device=dev)
            dist.broadcast(flat, src=owner, group=self.group)
            if owner != self.rank:
                off = 0
                for i in idx:
                    n = self.params[i].numel()
                    self.params[i].copy_(flat[off:off + n].view(self.params[i].shape))
                    off += n
