"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle.

This module holds input generation and workload descriptions only: no step of
the optimizer's arithmetic lives here. Everything is generated on the host with
``torch.Generator('cpu')`` from a per-matrix seed, so a single matrix can be
regenerated on its own, and the same bytes feed the CUDA path and the oracle.

The pages train GPT-style models on FineWeb; the matrix banks below stand in
for those models' 2-D parameter shapes (the dataset itself is not used):
  * "Training NanoGPT in 39.9 Seconds" and the speedrun introduction page:
    the 124M-parameter GPT (12 layers, width 768, 4 attention matrices, a
    768x3072 fc and a 3072x768 projection per layer, a 50304-token readout).
  * "qlabs-eng/slowrun", section "仕組み": a 2.7B transformer trained with Muon
    and weight decay 1.6 (here 32 layers of width 2560).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Dict, List, Tuple

import torch

QUINTIC = (3.4445, -4.7750, 2.0315)
CUBIC = (1.5, -0.5, 0.0)

KIND_PARAM, KIND_GRAD = 1, 2


@dataclass(frozen=True)
class BankSpec:
    count: int
    rows: int
    cols: int
    label: str = ""


@dataclass
class Workload:
    """A matrix bank with its dtypes, value recipe and hyper-parameters."""
    cid: int
    name: str
    banks: List[BankSpec]
    param_dtype: str            # 'f32' | 'bf16'
    grad_dtype: str             # 'f32' | 'bf16'
    param_sigma: float
    grad_sigma: float
    spike_rank: int             # 0 = no low-rank spike
    spike_factor: float
    hp: Dict                    # plain numbers, read by both sides
    steps: int
    variant: str = "muon"       # 'muon' | 'anvil'
    extra: Dict = field(default_factory=dict)

    @property
    def n_params(self) -> int:
        return sum(b.count * b.rows * b.cols for b in self.banks)


def _gpt124m_banks() -> List[BankSpec]:
    return [BankSpec(48, 768, 768, "attn q/k/v/o"),
            BankSpec(12, 768, 3072, "mlp fc"),
            BankSpec(12, 3072, 768, "mlp proj")]


def workloads() -> Dict[int, Workload]:
    """The five workloads (ids 1..5)."""
    q5 = [QUINTIC] * 5
    return {
        1: Workload(1, "single_256x512_cubic", [BankSpec(1, 256, 512, "single")],
                    "f32", "f32", 0.02, 1.0, 0, 10.0,
                    dict(lr=0.02, mu=0.95, weight_decay=0.0, nesterov=1,
                         coeffs=[CUBIC] * 5, eps=1e-7), steps=3),
        2: Workload(2, "gpt124m_bank", _gpt124m_banks(),
                    "bf16", "bf16", 0.02, 1e-3, 4, 10.0,
                    dict(lr=0.05, mu=0.95, weight_decay=0.0, nesterov=1,
                         coeffs=q5, eps=1e-7), steps=10),
        3: Workload(3, "square_1024x1024x64", [BankSpec(64, 1024, 1024, "square")],
                    "bf16", "bf16", 0.02, 1.0, 0, 10.0,
                    dict(lr=0.02, mu=0.95, weight_decay=0.01, nesterov=0,
                         coeffs=q5, eps=1e-7), steps=25,
                    extra=dict(warmup=5, timed=20)),
        4: Workload(4, "transformer2p5b_bank",
                    [BankSpec(128, 2560, 2560, "attn"),
                     BankSpec(32, 2560, 10240, "mlp fc"),
                     BankSpec(32, 10240, 2560, "mlp proj")],
                    "bf16", "bf16", 0.02, 1e-4, 8, 10.0,
                    dict(lr=0.02, mu=0.95, weight_decay=1.6, nesterov=1,
                         coeffs=q5, eps=1e-7), steps=5),
        5: Workload(5, "anvil_gpt124m_readout",
                    _gpt124m_banks() + [BankSpec(1, 768, 50304, "readout")],
                    "bf16", "bf16", 0.02, 1e-3, 4, 10.0,
                    dict(lr=0.05, beta_fast=0.9, beta_slow=0.99, weight_decay=0.1,
                         coeffs=[QUINTIC] * 6, eps=1e-7, ema_beta=0.99,
                         readout_final_weight=0.35),
                    steps=50, variant="anvil"),
    }


def seed_for(cid: int, kind: int, step: int, bank: int, mat: int) -> int:
    """Distinct seed per (workload, kind, step, bank, matrix)."""
    return (((cid * 4 + kind) * 1000 + step) * 16 + bank) * 100000 + mat


_TORCH_DTYPE = {"f32": torch.float32, "bf16": torch.bfloat16}


def torch_dtype(name: str) -> torch.dtype:
    return _TORCH_DTYPE[name]


def gaussian(rows: int, cols: int, seed: int, sigma: float) -> torch.Tensor:
    g = torch.Generator().manual_seed(seed)
    return torch.randn(rows, cols, generator=g, dtype=torch.float32) * sigma


def spiked_gaussian(rows: int, cols: int, seed: int, sigma: float, rank: int,
                    factor: float) -> torch.Tensor:
    """N(0, sigma^2) plus a rank-`rank` spike whose entry RMS is factor*sigma:
    S = (sigma * factor / sqrt(rank)) * sum_j u_j v_j^T with u_j, v_j standard
    normal, so each entry of the sum has variance `rank`."""
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(rows, cols, generator=g, dtype=torch.float32) * sigma
    if rank > 0:
        u = torch.randn(rows, rank, generator=g, dtype=torch.float32)
        v = torch.randn(cols, rank, generator=g, dtype=torch.float32)
        x += (sigma * factor / math.sqrt(rank)) * (u @ v.T)
    return x


def make_params(w: Workload, bank: int, mats=None) -> torch.Tensor:
    """[count, R, C] (or the listed matrices) initial parameters, storage dtype."""
    b = w.banks[bank]
    idx = range(b.count) if mats is None else mats
    out = [gaussian(b.rows, b.cols, seed_for(w.cid, KIND_PARAM, 0, bank, i), w.param_sigma)
           for i in idx]
    return torch.stack(out).to(torch_dtype(w.param_dtype))


def make_grads(w: Workload, bank: int, step: int, mats=None) -> torch.Tensor:
    """[count, R, C] (or the listed matrices) gradients of `step`, storage dtype."""
    b = w.banks[bank]
    idx = range(b.count) if mats is None else mats
    out = [spiked_gaussian(b.rows, b.cols, seed_for(w.cid, KIND_GRAD, step, bank, i),
                           w.grad_sigma, w.spike_rank, w.spike_factor)
           for i in idx]
    return torch.stack(out).to(torch_dtype(w.grad_dtype))


def custom_workload(shapes: List[Tuple[int, int, int]], hp: Dict, *, cid: int = 90,
                    param_dtype="bf16", grad_dtype="bf16", grad_sigma=1.0,
                    spike_rank=0, variant="muon", steps=1) -> Workload:
    """A small ad-hoc bank for tests: shapes = [(count, rows, cols), ...]."""
    return Workload(cid, "custom", [BankSpec(*s) for s in shapes], param_dtype,
                    grad_dtype, 0.02, grad_sigma, spike_rank, 10.0, dict(hp),
                    steps=steps, variant=variant)
