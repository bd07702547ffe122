"""Seeded synthetic inputs shaped like the pages' workloads.

This module holds no attention arithmetic: it only draws random tensors.
Both the CUDA path's tests/benchmark and the fp64 oracle take their inputs
from here, so they see bit-identical values (the oracle widens them to fp64).

Recipe: ``torch.Generator('cpu').manual_seed(seed)``, ``randn`` in fp32,
multiplied by the tensor's standard deviation, then rounded to the compute
dtype (round-to-nearest-even for bf16).  Seeds are
``1000 + 10 * config_index + tensor_id`` with tensor ids
q=0, k=1, v=2, do=3, y=4, w_k=5, w_v=6, dk=7, dv=8 (dk and dv, unit
Gaussians, stand in for the gradients the attention backward hands to the
K/V recomputation when that step is exercised on its own).

Workloads whose inputs are tens of GB (VMME) are drawn on the device instead
(``make_device``: same seeds, torch's device generator).

The shapes stand in for the LV-XAttn review page's workloads (Llama 3-V,
long-video cross-attention with S_Q << S_KV, Figure 1 / "The reading"; the
pages' Video-MME inputs are not available, synthetic Gaussians replace them)
and for Ring-Attention-style causal self-attention.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field, replace
from typing import Optional

import torch

TENSOR_IDS = {"q": 0, "k": 1, "v": 2, "do": 3, "y": 4, "w_k": 5, "w_v": 6, "dk": 7, "dv": 8}


@dataclass(frozen=True)
class Workload:
    name: str
    index: int
    B: int
    H: int
    H_kv: int
    d: int
    S_Q: int
    S_KV: int
    n_blocks: int
    causal: bool
    dtype: str                     # "f32" or "bf16"
    qkv_std: float
    backward: bool
    d_embed: int = 0               # > 0: K, V recomputed from y
    desc: str = field(default="", compare=False)

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    def scaled(self, **kw) -> "Workload":
        """Same recipe (seeds, distributions) at other sizes."""
        return replace(self, **kw)

    def fwd_flops(self) -> float:
        """4 B H S_Q S_KV d, counting only unmasked (query, key) pairs."""
        if self.causal:
            pairs = self.S_Q * (self.S_Q + 1) / 2
        else:
            pairs = self.S_Q * self.S_KV
        return 4.0 * self.B * self.H * pairs * self.d

    def bwd_flops(self) -> float:
        """Five GEMMs against the forward's two: 2.5x the forward count."""
        return 2.5 * self.fwd_flops() if self.backward else 0.0

    def kv_flops(self) -> float:
        return 2.0 * 2.0 * self.B * self.S_KV * self.d_embed * self.H_kv * self.d if self.d_embed else 0.0


_R2 = 1.0 / math.sqrt(2.0)

WORKLOADS = {
    "C0": Workload("C0", 0, B=1, H=1, H_kv=1, d=64, S_Q=128, S_KV=1024, n_blocks=4,
                   causal=False, dtype="f32", qkv_std=1.0, backward=False,
                   desc="single-head non-causal cross-attention, fp32, n=4, forward"),
    "C1": Workload("C1", 1, B=1, H=32, H_kv=8, d=128, S_Q=2048, S_KV=65536, n_blocks=8,
                   causal=False, dtype="bf16", qkv_std=_R2, backward=False,
                   desc="Llama-3-V-like GQA cross-attention forward, bf16"),
    "C2": Workload("C2", 2, B=1, H=32, H_kv=8, d=128, S_Q=2048, S_KV=65536, n_blocks=8,
                   causal=False, dtype="bf16", qkv_std=_R2, backward=True, d_embed=4096,
                   desc="C1 forward + backward, K/V recomputed from shared visual features"),
    "C3": Workload("C3", 3, B=1, H=32, H_kv=32, d=128, S_Q=131072, S_KV=131072, n_blocks=8,
                   causal=True, dtype="bf16", qkv_std=_R2, backward=True,
                   desc="causal self-attention forward + backward, n=8 block skipping"),
    "C4": Workload("C4", 4, B=2, H=16, H_kv=16, d=128, S_Q=512, S_KV=262144, n_blocks=16,
                   causal=False, dtype="bf16", qkv_std=_R2, backward=True,
                   desc="long-video cross-attention forward + backward, n=16"),
    # The pages' average Video-MME input for Llama 3-V (LV-XAttn review page, "The reading"):
    # 5,514 text tokens against 15,279,944 visual tokens; K+V = 62.6 GB in bf16.  Neither
    # length is a multiple of the 128-row tiles.
    "VMME": Workload("VMME", 5, B=1, H=32, H_kv=8, d=128, S_Q=5514, S_KV=15279944, n_blocks=8,
                     causal=False, dtype="bf16", qkv_std=_R2, backward=False,
                     desc="Video-MME-average-shaped long-video cross-attention forward, "
                          "Llama-3-V heads"),
}


def seed_for(w: Workload, tensor: str) -> int:
    return 1000 + 10 * w.index + TENSOR_IDS[tensor]


def _randn(shape, seed: int, std: float, dtype: torch.dtype) -> torch.Tensor:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    t = torch.randn(*shape, generator=g, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(dtype)


def spec(w: Workload, name: str):
    """(shape, standard deviation) of input tensor ``name`` of workload ``w``."""
    if name in ("q", "do"):
        return (w.B, w.S_Q, w.H, w.d), (w.qkv_std if name == "q" else 1.0)
    if name in ("k", "v"):
        return (w.B, w.S_KV, w.H_kv, w.d), w.qkv_std
    if name in ("dk", "dv"):
        return (w.B, w.S_KV, w.H_kv, w.d), 1.0
    if name == "y":
        return (w.B, w.S_KV, w.d_embed), 1.0
    if name in ("w_k", "w_v"):
        return (w.d_embed, w.H_kv * w.d), 1.0 / math.sqrt(w.d_embed)
    raise KeyError(name)


def make(w: Workload, tensors=("q", "k", "v"), dtype: Optional[torch.dtype] = None) -> dict:
    """Host tensors for workload ``w`` (contiguous, CPU)."""
    dt = dtype or w.torch_dtype
    out = {}
    for name in tensors:
        shape, std = spec(w, name)
        out[name] = _randn(shape, seed_for(w, name), std, dt)
    return out


def make_device(w: Workload, tensors=("q", "k", "v"), device="cuda",
                dtype: Optional[torch.dtype] = None, chunk: int = 1 << 28) -> dict:
    """Device tensors for workloads too large to draw on the host in reasonable
    time (the VMME shape: 31 GB per K or V).  Same seeds and distributions as
    ``make``, drawn with torch's device generator in row-major chunks of
    ``chunk`` elements; the values are a different stream from ``make``'s, so
    whatever checks them (the oracle) reads them back from the device."""
    dt = dtype or w.torch_dtype
    out = {}
    for name in tensors:
        shape, std = spec(w, name)
        g = torch.Generator(device=device)
        g.manual_seed(seed_for(w, name))
        t = torch.empty(shape, dtype=dt, device=device)
        flat = t.view(-1)
        for s0 in range(0, flat.numel(), chunk):
            n = min(chunk, flat.numel() - s0)
            x = torch.randn(n, generator=g, device=device, dtype=torch.float32)
            if std != 1.0:
                x.mul_(std)
            flat[s0:s0 + n].copy_(x)
        out[name] = t
    return out
