"""Seeded synthetic inputs for the Token Sparse Attention layer.

This module only draws random numbers: it holds none of the method's
arithmetic, and both the CUDA path and the CPU oracle consume what it returns.

The pages measure on real LLaMA-3.1-8B activations over RULER, InfiniteBench
and Needle-in-a-Haystack; none of that is available here, so these tensors
stand in for them with the same shapes (32 query heads, 8 KV heads, d = 128,
contexts of 4K / 32K / 128K).  Structure: Q, K, V, X ~ N(0, 1); per KV group a
random unit direction u_g; every query of that group's heads is shifted by
sqrt(d) * u_g and the keys of the four sink tokens plus a random 0.5 % of
"heavy hitter" tokens are shifted by `shift` * u_g, so those keys gain a logit
of about `shift` under the 1/sqrt(d) scale.  Values are drawn in fp32 on the
CPU from a torch Generator and rounded once (round-to-nearest-even) to the
run's dtype.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    L: int
    H: int
    Hkv: int
    d: int
    dtype: torch.dtype
    q: int
    tau: float
    shift: float
    heavy_frac: float
    shared_dir: bool  # one direction for all heads (MHA tiny case)


WORKLOADS = {
    # MHA correctness case: 4 heads with their own K/V, d = 64, fp32.
    "tiny_mha_1k": Workload("tiny_mha_1k", 1, 1024, 4, 4, 64, torch.float32, 16, 0.01,
                            3.0, 0.0, True),
    # LLaMA-3.1-8B-shaped GQA layer (32 / 8 heads, d = 128, bf16).
    "llama8b_4k": Workload("llama8b_4k", 1, 4096, 32, 8, 128, torch.bfloat16, 16, 0.005,
                           2.5, 0.005, False),
    "llama8b_32k": Workload("llama8b_32k", 1, 32768, 32, 8, 128, torch.bfloat16, 16, 0.01,
                            2.5, 0.005, False),
    "llama8b_128k": Workload("llama8b_128k", 1, 131072, 32, 8, 128, torch.bfloat16, 16, 0.01,
                             2.5, 0.005, False),
    "llama8b_64k_b2": Workload("llama8b_64k_b2", 2, 65536, 32, 8, 128, torch.bfloat16, 16,
                               0.005, 2.5, 0.005, False),
}


def make_inputs(B: int, L: int, H: int, Hkv: int, d: int, dtype: torch.dtype = torch.bfloat16,
                seed: int = 0, shift: float = 2.5, heavy_frac: float = 0.005,
                shared_dir: bool = False, n_sinks: int = 4):
    """Return dict(Q [B,L,H,d], K [B,L,Hkv,d], V [B,L,Hkv,d], X [B,L,H*d]) on the CPU."""
    g = torch.Generator().manual_seed(int(seed))
    Q = torch.randn(B, L, H, d, generator=g)
    K = torch.randn(B, L, Hkv, d, generator=g)
    V = torch.randn(B, L, Hkv, d, generator=g)
    X = torch.randn(B, L, H * d, generator=g)
    G = H // Hkv
    for b in range(B):
        n_dir = 1 if shared_dir else Hkv
        u = torch.randn(n_dir, d, generator=g)
        u = u / u.norm(dim=1, keepdim=True)
        if shared_dir:
            u = u.expand(Hkv, d)
        n_heavy = int(round(heavy_frac * L))
        pos = list(range(min(n_sinks, L)))
        if n_heavy > 0 and L > n_sinks:
            perm = torch.randperm(L - n_sinks, generator=g)[:n_heavy] + n_sinks
            pos += sorted(perm.tolist())
        pos_t = torch.tensor(pos, dtype=torch.long)
        for kv in range(Hkv):
            Q[b, :, kv * G:(kv + 1) * G, :] += (d ** 0.5) * u[kv]
            K[b, pos_t, kv, :] += shift * u[kv]
    return dict(Q=Q.to(dtype), K=K.to(dtype), V=V.to(dtype), X=X.to(dtype))


def make_workload(name: str, seed: int = 0, L: int | None = None, B: int | None = None):
    """Inputs of a named workload (optionally with another L or B)."""
    w = WORKLOADS[name]
    return make_inputs(B or w.B, L or w.L, w.H, w.Hkv, w.d, w.dtype, seed, w.shift,
                       w.heavy_frac, w.shared_dir)


def layer_mask(n_layers: int, seed: int = 0) -> list[int]:
    """A sparse-layer mask with half the layers sparse, drawn from the seed."""
    g = torch.Generator().manual_seed(int(seed) + 7919)
    perm = torch.randperm(n_layers, generator=g)[: n_layers // 2]
    m = [0] * n_layers
    for i in perm.tolist():
        m[i] = 1
    return m
