"""Seeded synthetic workloads shaped like the pages' experiments (no method arithmetic here).

The pages train a 530M Llama-3-style model at 98,304 tokens and scale to 1M tokens ("Long
Context Pre-Training with Lighthouse Attention", technical summary section 4). There is no
dataset here: Q, K, V are i.i.d. N(0, 1) rows times a per-row saliency scale shared by Q, K
and V of that (b, h, t), so that the l2 scores vary the way projected activations do. The
upstream gradient dO is N(0, 1). Both the CUDA path and the oracle take these same tensors.

Seeds: Q = s, K = s+1, V = s+2, dO = s+3, scales = s+4.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    d: int
    N: int
    p: int
    L: int
    S: int
    dtype: torch.dtype
    scale: str  # "none" | "lognormal" | "lognormal_spikes" | "random_walk"
    sigma: float = 0.0
    describe: str = ""


WORKLOADS = {
    "tiny-2k-fp32": Workload("tiny-2k-fp32", 1, 4, 64, 2048, 4, 3, 512, torch.float32, "none",
                             describe="N=2048 H=4 d=64 fp32, p=4 L=3 S=512, N(0,1)"),
    "32k": Workload("32k", 1, 16, 128, 32768, 4, 5, 4096, torch.bfloat16, "lognormal", 0.5,
                    describe="N=32768 H=16 d=128 bf16, p=4 L=5 S=4096, log-normal(0,0.5) rows"),
    "llama530m-98k": Workload("llama530m-98k", 1, 16, 64, 98304, 4, 6, 6144, torch.bfloat16,
                              "lognormal_spikes", 0.5,
                              describe="N=98304 H=16 d=64 bf16, p=4 L=6 S=6144, log-normal(0,0.5)"
                                       " rows plus 1% of tokens x4"),
    "128k": Workload("128k", 1, 32, 128, 131072, 4, 6, 8192, torch.bfloat16, "random_walk", 0.5,
                     describe="N=131072 H=32 d=128 bf16, p=4 L=6 S=8192, random-walk row scales"),
    "1m": Workload("1m", 1, 8, 128, 1048576, 4, 7, 16384, torch.bfloat16, "lognormal", 0.75,
                   describe="N=1048576 H=8 d=128 bf16, p=4 L=7 S=16384, log-normal(0,0.75) rows"),
}


def _gen(device, seed):
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def row_scales(w: Workload, device, seed=0, B=None, H=None, N=None):
    """Per-(b,h,t) saliency scale, shape [B, H, N, 1], float32."""
    B, H, N = B or w.B, H or w.H, N or w.N
    g = _gen(device, seed + 4)
    if w.scale == "none":
        return torch.ones(B, H, N, 1, device=device)
    if w.scale in ("lognormal", "lognormal_spikes"):
        s = torch.exp(w.sigma * torch.randn(B, H, N, 1, generator=g, device=device))
        if w.scale == "lognormal_spikes":
            n_spike = max(1, N // 100)
            pos = torch.randperm(N, generator=g, device=device)[:n_spike]
            s[:, :, pos] *= 4.0
        return s
    if w.scale == "random_walk":
        walk = torch.cumsum(torch.randn(B, H, N, 1, generator=g, device=device), dim=2)
        walk = walk - walk.mean(dim=2, keepdim=True)
        walk = walk * (w.sigma / walk.std(dim=2, keepdim=True))
        return torch.exp(walk)
    raise ValueError(w.scale)


def make_inputs(w: Workload, device="cuda", seed=0, B=None, H=None, N=None, unit=False):
    """(q, k, v, d_o) in the workload's dtype. B/H/N override the sizes (sampled heads)."""
    B, H, N = B or w.B, H or w.H, N or w.N
    scale = torch.ones(B, H, N, 1, device=device) if unit else row_scales(w, device, seed, B, H, N)
    out = []
    for i in range(3):
        x = torch.randn(B, H, N, w.d, generator=_gen(device, seed + i), device=device)
        out.append((x * scale).to(w.dtype))
        del x
    d_o = torch.randn(B, H, N, w.d, generator=_gen(device, seed + 3), device=device).to(w.dtype)
    return (*out, d_o)
