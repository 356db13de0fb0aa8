"""Seeded synthetic KV caches shaped like a long-context GQA prefill.

This module only draws random numbers; it holds none of the codec's arithmetic,
so both the CUDA path and the CPU oracle may consume its output.

Recipe (per layer and KV head, from one integer seed):
  * C unit directions u_c = g_c / ||g_c||, g_c ~ N(0, I_D);
  * each key picks c ~ Uniform{C}, a scale ~ LogNormal(0, 0.5) and noise
    N(0, 0.1^2 I):  K_t = scale * u_c + noise;
  * two outlier channels, fixed for the whole run, are multiplied by 8;
  * values V_t ~ N(0, I);
  * observation queries (W per query head) and decode queries are drawn
    like the keys of their KV head (same directions, fresh draws);
  * bf16 caches are drawn in fp32 and rounded to nearest-even.
The draws use torch generators on the requested device, so a CPU draw and a
CUDA draw of the same seed differ; a caller that compares both paths draws
once and copies.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

_DT = {"fp32": torch.float32, "bf16": torch.bfloat16}


@dataclass
class CacheSpec:
    n_layers: int
    n_kv_heads: int
    n_q_heads: int
    n_tokens: int
    head_dim: int = 128
    window: int = 32
    n_dirs: int = 128
    dtype: str = "bf16"
    seed: int = 0


def outlier_channels(spec: CacheSpec) -> torch.Tensor:
    g = torch.Generator().manual_seed(spec.seed * 7919 + 17)
    return torch.randperm(spec.head_dim, generator=g)[:2]


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _keys_like(g, dirs, n, D, outl, device):
    c = torch.randint(0, dirs.shape[0], (n,), generator=g, device=device)
    scale = torch.exp(0.5 * torch.randn(n, generator=g, device=device))
    x = scale[:, None] * dirs[c] + 0.1 * torch.randn(n, D, generator=g, device=device)
    x[:, outl] *= 8.0
    return x


def _head_seed(spec: CacheSpec, layer: int, head: int, salt: int) -> int:
    return ((spec.seed * 1_000_003 + layer) * 65_537 + head) * 8 + salt


def head_directions(spec: CacheSpec, layer: int, head: int, device) -> torch.Tensor:
    g = _gen(device, _head_seed(spec, layer, head, 0))
    d = torch.randn(spec.n_dirs, spec.head_dim, generator=g, device=device)
    return d / d.norm(dim=1, keepdim=True)


def make_layer(spec: CacheSpec, layer: int, device="cpu"):
    """K, V [H, N, D] and observation queries Q_obs [Hq, W, D] of one layer."""
    H, Hq, N, D, W = spec.n_kv_heads, spec.n_q_heads, spec.n_tokens, spec.head_dim, spec.window
    G = Hq // H
    dt = _DT[spec.dtype]
    outl = outlier_channels(spec).to(device)
    K = torch.empty(H, N, D, dtype=dt, device=device)
    V = torch.empty(H, N, D, dtype=dt, device=device)
    Q = torch.empty(Hq, W, D, dtype=dt, device=device)
    for h in range(H):
        dirs = head_directions(spec, layer, h, device)
        g = _gen(device, _head_seed(spec, layer, h, 1))
        K[h] = _keys_like(g, dirs, N, D, outl, device).to(dt)
        g = _gen(device, _head_seed(spec, layer, h, 2))
        V[h] = torch.randn(N, D, generator=g, device=device).to(dt)
        g = _gen(device, _head_seed(spec, layer, h, 3))
        Q[h * G:(h + 1) * G] = _keys_like(g, dirs, G * W, D, outl, device).reshape(G, W, D).to(dt)
    return K, V, Q


def make_decode_queries(spec: CacheSpec, layer: int, step: int, batch: int = 1, device="cpu"):
    """Decode queries q [batch, Hq, D] drawn like the keys."""
    H, Hq, D = spec.n_kv_heads, spec.n_q_heads, spec.head_dim
    G = Hq // H
    outl = outlier_channels(spec).to(device)
    q = torch.empty(batch, Hq, D, dtype=_DT[spec.dtype], device=device)
    for h in range(H):
        dirs = head_directions(spec, layer, h, device)
        g = _gen(device, _head_seed(spec, layer, h, 4) + 1_000_000 * (step + 1))
        q[:, h * G:(h + 1) * G] = _keys_like(g, dirs, batch * G, D, outl, device).reshape(batch, G, D).to(q.dtype)
    return q


def make_tail(spec: CacheSpec, layer: int, n_tail: int, batch: int = 1, device="cpu"):
    """Uncompressed decode-time tokens K_tail, V_tail [batch, H, n_tail, D]."""
    H, D = spec.n_kv_heads, spec.head_dim
    outl = outlier_channels(spec).to(device)
    dt = _DT[spec.dtype]
    Kt = torch.empty(batch, H, n_tail, D, dtype=dt, device=device)
    Vt = torch.empty(batch, H, n_tail, D, dtype=dt, device=device)
    for h in range(H):
        dirs = head_directions(spec, layer, h, device)
        g = _gen(device, _head_seed(spec, layer, h, 5))
        Kt[:, h] = _keys_like(g, dirs, batch * n_tail, D, outl, device).reshape(batch, n_tail, D).to(dt)
        g = _gen(device, _head_seed(spec, layer, h, 6))
        Vt[:, h] = torch.randn(batch, n_tail, D, generator=g, device=device).to(dt)
    return Kt, Vt


def gaussian_queries(n: int, D: int, seed: int, device="cpu") -> torch.Tensor:
    """Plain N(0, I) queries (the Theorem-1 error report)."""
    return torch.randn(n, D, generator=_gen(device, seed), device=device)


# Workloads named by what they are (layers, heads, tokens, precision, knob).
WORKLOADS = {
    "tiny-fp32-n1024": dict(spec=CacheSpec(1, 1, 4, 1024, dtype="fp32", n_dirs=32), theta=0.1),
    "llama8b-n32k-bf16": dict(spec=CacheSpec(32, 8, 32, 32768, n_dirs=128), theta=0.05),
    "llama70b-n128k-bf16": dict(spec=CacheSpec(80, 8, 64, 131072, n_dirs=256), theta=0.05),
    "llama8b-n32k-bf16-batch16": dict(spec=CacheSpec(32, 8, 32, 32768, n_dirs=128), theta=0.1, batch=16),
}
