"""Seeded synthetic inputs and the workload shapes they come in.

This module holds none of the quantisation arithmetic: it only draws random
numbers.  Both the CUDA path and the CPU oracle are fed from it.

Recipe (stand-in for Qwen3-8B weights and WikiText calibration activations,
neither of which is available):
  * W[r, j] ~ N(0, 0.02^2), rounded to fp16;
  * X[t, j] = z[t, j] * m[j] with z ~ N(0, 1), m[j] ~ lognormal(0, 1), and
    ceil(1% of d_in) channels, chosen by the same generator, multiplied by 50;
    rounded to fp16.
Every draw comes from a ``torch.Generator`` seeded per workload (and per
layer for the stack), on the CPU unless a CUDA generator is asked for.

Shapes follow the Qwen3-8B decoder block (hidden 4096, q/o 4096x4096,
k/v 1024x4096, gate/up 12288x4096, down 4096x12288) that the pages quantise
("From-Scratch AWQ INT4 Quantization on Qwen3-8B", results section).
"""
from __future__ import annotations

import math
from dataclasses import dataclass
from typing import Tuple

import torch

HIDDEN = 4096
INTER = 12288
KV = 1024
N_LAYERS = 36


@dataclass(frozen=True)
class SearchGroup:
    """Linears that share one input (one scale vector is searched for all)."""
    name: str
    members: Tuple[Tuple[str, int], ...]   # (linear name, d_out)
    d_in: int


BLOCK_GROUPS: Tuple[SearchGroup, ...] = (
    SearchGroup("qkv", (("q_proj", HIDDEN), ("k_proj", KV), ("v_proj", KV)), HIDDEN),
    SearchGroup("o", (("o_proj", HIDDEN),), HIDDEN),
    SearchGroup("gate_up", (("gate_proj", INTER), ("up_proj", INTER)), HIDDEN),
    SearchGroup("down", (("down_proj", HIDDEN),), INTER),
)


@dataclass(frozen=True)
class Workload:
    name: str
    groups: Tuple[SearchGroup, ...]
    tokens: int
    group_sizes: Tuple[int, ...] = (128,)
    n_grid: int = 20
    seed: int = 0
    layers: int = 1
    output_mode: bool = False

    @property
    def params(self) -> int:
        """Weights quantised by one pass over the whole workload."""
        return self.layers * sum(d * g.d_in for g in self.groups
                                 for _, d in g.members)


WORKLOADS = {
    "single_linear_256x512": Workload(
        "single_linear_256x512",
        (SearchGroup("linear", (("linear", 256),), 512),), tokens=64, seed=0),
    "q_proj_4096x4096": Workload(
        "q_proj_4096x4096",
        (SearchGroup("q_proj", (("q_proj", HIDDEN),), HIDDEN),),
        tokens=4096, seed=1),
    "qwen3_8b_block": Workload(
        "qwen3_8b_block", BLOCK_GROUPS, tokens=16384, group_sizes=(128, 64),
        seed=2),
    "down_proj_output_error": Workload(
        "down_proj_output_error",
        (SearchGroup("down", (("down_proj", HIDDEN),), INTER),),
        tokens=8192, seed=3, output_mode=True),
    "qwen3_8b_stack36": Workload(
        "qwen3_8b_stack36", BLOCK_GROUPS, tokens=2048, seed=4,
        layers=N_LAYERS),
}


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def weight(d_out: int, d_in: int, seed: int, device="cpu") -> torch.Tensor:
    """W ~ N(0, 0.02^2) as fp16 [d_out, d_in]."""
    g = _gen(seed, device)
    w = torch.randn(d_out, d_in, generator=g, device=device, dtype=torch.float32)
    return (w * 0.02).to(torch.float16)


def activations(tokens: int, d_in: int, seed: int, device="cpu") -> torch.Tensor:
    """Heavy-tailed calibration activations X as fp16 [tokens, d_in]."""
    g = _gen(seed, device)
    mag = torch.empty(d_in, device=device, dtype=torch.float32)
    mag.log_normal_(0.0, 1.0, generator=g)
    n_out = max(1, math.ceil(0.01 * d_in))
    outliers = torch.randperm(d_in, generator=g, device=device)[:n_out]
    mag[outliers] *= 50.0
    z = torch.randn(tokens, d_in, generator=g, device=device, dtype=torch.float32)
    return (z * mag).to(torch.float16)


def layer_seed(workload: Workload, layer: int) -> int:
    """Seed of one layer of a workload (layer 0 of a one-layer workload is
    the workload's own seed)."""
    if workload.layers == 1:
        return workload.seed
    return 1000 * (workload.seed + 1) + layer


def group_inputs(workload: Workload, layer: int = 0, device="cpu", seed=None):
    """Weights and activations of every search group of one layer.

    Returns a list of (SearchGroup, [W per member], X).  With base = 100 *
    (``seed`` if given, else the layer's seed), member m of group k uses seed
    ``base + 16*k + m + 1`` and the group's X uses ``base + 16*k``.
    """
    base = 100 * (layer_seed(workload, layer) if seed is None else int(seed))
    out = []
    for k, grp in enumerate(workload.groups):
        Ws = [weight(d, grp.d_in, base + 16 * k + m + 1, device)
              for m, (_, d) in enumerate(grp.members)]
        X = activations(workload.tokens, grp.d_in, base + 16 * k, device)
        out.append((grp, Ws, X))
    return out
