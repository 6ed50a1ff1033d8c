"""Seeded synthetic inputs for the Muon step: workload shapes and value recipes.

This module holds no arithmetic of the method.  It only draws the gradients,
momentum buffers and weights that both the CUDA path and the fp64 oracle are
fed, so that the two sides see identical inputs.  Nothing here reads a
dataset: the pages train on FineWeb, but the optimizer step only ever sees
gradient matrices, so seeded Gaussian matrices with low-rank "spikes" stand
in for them (a spike makes the momentum ill-conditioned, which is the case
Newton-Schulz orthogonalisation exists for).

Recipe for one matrix of shape rows x cols (all draws fp64, cast to fp32):

    noise  = std * N(0, 1)[rows, cols]                      role 0 (grad) / 3 (momentum)
    spike  = mult * std * U @ V.T,  U ~ N(0,1)[rows, r],     roles 1, 2 (grad) / 5, 6 (momentum)
                                    V ~ N(0,1)[cols, r]
    value  = noise + spike
    W      = 0.02 * N(0, 1)[rows, cols]                       role 4

Every draw has its own PCG64 stream, seeded with
``SeedSequence([root_seed, workload_index, step, matrix_index, role])``.
A device-side variant (``torch.Generator`` on the GPU, seeded from the same
SeedSequence) exists for the multi-GB workloads, where host generation would
take minutes; tests that use it copy the drawn matrices back to the host
before handing them to the oracle.
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional, Sequence, Tuple

import numpy as np


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic Muon workload: a list of 2-D parameter shapes and hyperparameters."""

    name: str
    index: int                       # position in the workload table (seed component)
    shapes: Tuple[Tuple[int, int], ...]
    param_dtype: str                 # "f32" or "bf16"
    grad_std: float
    spike_rank: int
    spike_mult: float
    mom_init: str                    # "spiked" (own draw), "zero", or "warmup" (= grad of step 0)
    beta: float = 0.95
    nesterov: bool = True
    lr: float = 0.02
    weight_decay: float = 0.0
    ns_steps: int = 5
    schedule: str = "quintic"        # "quintic" or "polar5"
    steps: int = 1                   # consecutive optimizer steps the workload describes

    @property
    def n_params(self) -> int:
        return sum(r * c for r, c in self.shapes)


def _layers(n_layers: int, d: int, hidden: int) -> Tuple[Tuple[int, int], ...]:
    per_layer = [(d, d)] * 4 + [(d, hidden), (hidden, d)]
    return tuple(per_layer * n_layers)


WORKLOADS = {
    w.name: w
    for w in [
        Workload("single-256x128-f32", 0, ((256, 128),), "f32", 1.0, 4, 20.0, "spiked",
                 lr=0.02, weight_decay=0.0),
        Workload("mlp-768x3072-bf16-3steps", 1, ((768, 3072),), "bf16", 1e-3, 16, 10.0, "zero",
                 lr=0.05, weight_decay=0.01, steps=3),
        Workload("gpt2-124m-72-matrices", 2, _layers(12, 768, 3072), "bf16", 1e-3, 8, 10.0,
                 "warmup", lr=0.02, weight_decay=0.0),
        Workload("gpt2-medium-144-matrices", 3, _layers(24, 1024, 4096), "bf16", 1e-3, 8, 10.0,
                 "warmup", lr=0.02, weight_decay=0.0, schedule="polar5"),
        Workload("wide-4096-192-matrices", 4, _layers(32, 4096, 14336), "bf16", 1e-4, 32, 10.0,
                 "warmup", lr=0.02, weight_decay=0.1),
    ]
}

WORKLOAD_ORDER = [w.name for w in sorted(WORKLOADS.values(), key=lambda w: w.index)]
ROOT_SEED = 0

ROLE_GRAD_NOISE, ROLE_GRAD_U, ROLE_GRAD_V, ROLE_MOM_NOISE, ROLE_W, ROLE_MOM_U, ROLE_MOM_V = range(7)


def seed_sequence(workload: Workload, step: int, mat: int, role: int) -> np.random.SeedSequence:
    return np.random.SeedSequence([ROOT_SEED, workload.index, step, mat, role])


def _rng(workload: Workload, step: int, mat: int, role: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed_sequence(workload, step, mat, role)))


def _spiked_np(workload, step, mat, rows, cols, roles) -> np.ndarray:
    r_noise, r_u, r_v = roles
    std = workload.grad_std
    x = std * _rng(workload, step, mat, r_noise).standard_normal((rows, cols))
    if workload.spike_rank > 0:
        U = _rng(workload, step, mat, r_u).standard_normal((rows, workload.spike_rank))
        V = _rng(workload, step, mat, r_v).standard_normal((cols, workload.spike_rank))
        x = x + (workload.spike_mult * std) * (U @ V.T)
    return x.astype(np.float32)


def grad_np(workload: Workload, step: int, mat: int) -> np.ndarray:
    rows, cols = workload.shapes[mat]
    return _spiked_np(workload, step, mat, rows, cols, (ROLE_GRAD_NOISE, ROLE_GRAD_U, ROLE_GRAD_V))


def momentum_np(workload: Workload, mat: int) -> np.ndarray:
    rows, cols = workload.shapes[mat]
    if workload.mom_init == "zero":
        return np.zeros((rows, cols), np.float32)
    if workload.mom_init == "warmup":
        # One untimed warm-up step from a zero buffer leaves m = g_0.
        return grad_np(workload, 0, mat)
    return _spiked_np(workload, 0, mat, rows, cols, (ROLE_MOM_NOISE, ROLE_MOM_U, ROLE_MOM_V))


def weight_np(workload: Workload, mat: int) -> np.ndarray:
    rows, cols = workload.shapes[mat]
    return (0.02 * _rng(workload, 0, mat, ROLE_W).standard_normal((rows, cols))).astype(np.float32)


def first_step_index(workload: Workload) -> int:
    """Step index of the first timed/checked gradient (1 when step 0 warmed the momentum)."""
    return 1 if workload.mom_init == "warmup" else 0


def bf16_round_np(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to the nearest bf16 (ties to even), returned as fp32.

    Used to put bf16 weights on both sides of a comparison: the CUDA path
    stores them as bf16, the oracle reads the same values in fp64.
    """
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (b >> 16) & 1
    r = ((b + 0x7FFF + lsb) >> 16) << 16
    nan = np.isnan(x)
    out = r.astype(np.uint32).view(np.float32).copy()
    out[nan] = np.nan
    return out.reshape(np.shape(x))


# ----------------------------------------------------------------------------------------
# Device-side draws for the multi-GB workloads (torch is used only as a random source here).
# ----------------------------------------------------------------------------------------

def _torch_seed(workload: Workload, step: int, mat: int, role: int) -> int:
    return int(seed_sequence(workload, step, mat, role).generate_state(1, np.uint64)[0] >> 1)


def _spiked_torch(workload, step, mat, rows, cols, roles, device):
    import torch

    r_noise, r_u, r_v = roles
    std = workload.grad_std
    gen = torch.Generator(device=device)
    gen.manual_seed(_torch_seed(workload, step, mat, r_noise))
    x = torch.randn((rows, cols), generator=gen, device=device, dtype=torch.float32).mul_(std)
    if workload.spike_rank > 0:
        gen.manual_seed(_torch_seed(workload, step, mat, r_u))
        U = torch.randn((rows, workload.spike_rank), generator=gen, device=device)
        gen.manual_seed(_torch_seed(workload, step, mat, r_v))
        V = torch.randn((cols, workload.spike_rank), generator=gen, device=device)
        x.addmm_(U, V.t(), alpha=workload.spike_mult * std)
    return x


def grad_torch(workload: Workload, step: int, mat: int, device):
    rows, cols = workload.shapes[mat]
    return _spiked_torch(workload, step, mat, rows, cols,
                         (ROLE_GRAD_NOISE, ROLE_GRAD_U, ROLE_GRAD_V), device)


def momentum_torch(workload: Workload, mat: int, device):
    import torch

    rows, cols = workload.shapes[mat]
    if workload.mom_init == "zero":
        return torch.zeros((rows, cols), device=device, dtype=torch.float32)
    if workload.mom_init == "warmup":
        return grad_torch(workload, 0, mat, device)
    return _spiked_torch(workload, 0, mat, rows, cols,
                         (ROLE_MOM_NOISE, ROLE_MOM_U, ROLE_MOM_V), device)


def weight_torch(workload: Workload, mat: int, device):
    import torch

    rows, cols = workload.shapes[mat]
    gen = torch.Generator(device=device)
    gen.manual_seed(_torch_seed(workload, 0, mat, ROLE_W))
    w = torch.randn((rows, cols), generator=gen, device=device, dtype=torch.float32).mul_(0.02)
    return w.to(torch.bfloat16) if workload.param_dtype == "bf16" else w


# ------------------------------------------------------------------ AdamW tensors

def gpt2_124m_adamw_tensors() -> List[Tuple[str, int]]:
    """The parameters of the GPT-2 124M layout that the hybrid setup gives to AdamW (the
    1-D ones and the embeddings): token embedding 50257 x 768, position embedding
    1024 x 768, and per layer the two LayerNorm gains and biases and the four linear
    biases, plus the final LayerNorm.  Returned as (name, numel)."""
    d, vocab, ctx, layers = 768, 50257, 1024, 12
    out = [("wte", vocab * d), ("wpe", ctx * d)]
    for i in range(layers):
        out += [(f"h{i}.ln_1.weight", d), (f"h{i}.ln_1.bias", d), (f"h{i}.attn.c_attn.bias", 3 * d),
                (f"h{i}.attn.c_proj.bias", d), (f"h{i}.ln_2.weight", d), (f"h{i}.ln_2.bias", d),
                (f"h{i}.mlp.c_fc.bias", 4 * d), (f"h{i}.mlp.c_proj.bias", d)]
    out += [("ln_f.weight", d), ("ln_f.bias", d)]
    return out


ADAMW_WORKLOAD = "gpt2-124m-adamw-params"
ADAMW_INDEX = 10  # seed component, distinct from the Muon workloads


def adamw_grad_torch(step: int, i: int, numel: int, device, std: float = 1e-3):
    """fp32 gradient of AdamW tensor i at `step`: std * N(0, 1), seeded like the Muon inputs."""
    import torch

    gen = torch.Generator(device=device)
    gen.manual_seed(int(np.random.SeedSequence([ROOT_SEED, ADAMW_INDEX, step, i, ROLE_GRAD_NOISE])
                        .generate_state(1, np.uint64)[0] >> 1))
    return torch.randn(numel, generator=gen, device=device, dtype=torch.float32).mul_(std)


def adamw_param_torch(i: int, numel: int, device):
    """bf16 parameter of AdamW tensor i: 0.02 * N(0, 1)."""
    import torch

    gen = torch.Generator(device=device)
    gen.manual_seed(int(np.random.SeedSequence([ROOT_SEED, ADAMW_INDEX, 0, i, ROLE_W])
                        .generate_state(1, np.uint64)[0] >> 1))
    return torch.randn(numel, generator=gen, device=device, dtype=torch.float32).mul_(0.02).to(torch.bfloat16)


def scaled_workload(workload: Workload, shapes: Sequence[Tuple[int, int]], name: Optional[str] = None) -> Workload:
    """Same value recipe and hyperparameters on other shapes (small parity cases)."""
    return dataclasses.replace(workload, shapes=tuple(shapes), name=name or workload.name + "-scaled")
