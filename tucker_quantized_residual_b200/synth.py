"""Seeded synthetic KV caches shaped like the models in "A JoLT for the KV Cache"
(Krishnan & Schulz), Section 4.1 "Setup".

This module only makes INPUTS. It holds none of the compression method's
arithmetic, and both the oracle tests and the CUDA path draw their caches from
it. The real caches of the paper's experiments need model checkpoints and text
corpora; these synthetic caches stand in for them with the same shapes.

Recipe (one cell = one layer group's K or V, shape [L_g, H, T, D]):

* A in R^{T x R} and F in R^{D x R}: Haar-orthonormal (QR of a Gaussian),
  shared by every layer and head of the group, so token and feature subspaces
  line up inside a group, which is the structure the paper's Section 1 and
  Section 3 ("truncate only the token and feature modes") rely on.
* every (layer, head) gets its own Haar mixing W_lh in R^{R x R};
  S_lh = A diag(sigma) W_lh F^T with sigma_i = i^(-alpha), i = 1..R.
* keys only: ``k_outliers`` fixed feature channels (the same for every head,
  drawn once from the seed) are multiplied by ``outlier_scale``.
* Gaussian noise N_lh with ||N_lh||^2 = noise * ||S_lh||^2.
* each head is scaled to entry RMS 1.
* keys only, when ``rope_theta_k`` > 0: rotary position embedding over
  positions 0..T-1 with the rotate-half pairing (i, i + D/2) and inverse
  frequencies theta^(-2i/D), applied here in fp64 so that the cache holds
  post-RoPE keys the way a model would emit them.
* rounded once to the storage dtype (bf16 round-to-nearest-even, or fp32).

Every (seed, sequence, group, kind) has its own torch generator, so any subset
of groups can be regenerated alone with identical values.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional, Tuple

import torch

__all__ = ["CacheSpec", "SPECS", "make_cache", "make_group", "group_starts",
           "dense_bf16_bytes"]


@dataclasses.dataclass(frozen=True)
class CacheSpec:
    name: str
    batch: int
    n_layers: int
    n_heads: int
    seq_len: int
    head_dim: int
    group_size: int
    rank: int
    sigma_exp: float
    noise: float
    k_outliers: int = 4
    outlier_scale: float = 10.0
    rope_theta_k: float = 0.0
    dtype: str = "bf16"          # "bf16" or "f32"

    def replace(self, **kw) -> "CacheSpec":
        return dataclasses.replace(self, **kw)

    @property
    def n_groups(self) -> int:
        return len(group_starts(self)) - 1


SPECS: Dict[str, CacheSpec] = {
    # one group, fp32, no RoPE and no outliers
    "tiny": CacheSpec("tiny", 1, 2, 2, 256, 64, 2, 16, 1.0, 0.01,
                      k_outliers=0, rope_theta_k=0.0, dtype="f32"),
    # Mistral-7B-v0.3-shaped GQA cache
    "mistral": CacheSpec("mistral", 1, 32, 8, 1024, 128, 4, 128, 0.8, 0.02,
                         rope_theta_k=1e6),
    # LLaMA-2-13B-shaped MHA cache
    "llama2_13b": CacheSpec("llama2_13b", 1, 40, 40, 4096, 128, 4, 128, 0.8,
                            0.02, rope_theta_k=1e4),
    # LLaMA-3.1-8B-shaped long-context cache (64K tokens)
    "llama31_8b_64k": CacheSpec("llama31_8b_64k", 1, 32, 8, 65536, 128, 4, 128,
                                0.7, 0.03, rope_theta_k=5e5),
    # MoE/GQA batch of 16 sequences (T chosen per run)
    "moe_t1024": CacheSpec("moe_t1024", 16, 48, 4, 1024, 128, 6, 128, 0.8,
                           0.02, rope_theta_k=1e6),
    "moe_t8192": CacheSpec("moe_t8192", 16, 48, 4, 8192, 128, 6, 128, 0.8,
                           0.02, rope_theta_k=1e6),
    "moe_t32768": CacheSpec("moe_t32768", 16, 48, 4, 32768, 128, 6, 128, 0.8,
                            0.02, rope_theta_k=1e6),
}


def group_starts(spec: CacheSpec) -> List[int]:
    """Contiguous groups of ``group_size`` layers; a short trailing group is
    kept as its own group."""
    starts = list(range(0, spec.n_layers, spec.group_size))
    return starts + [spec.n_layers]


def dense_bf16_bytes(spec: CacheSpec) -> int:
    """Bytes of K plus V stored densely in bf16 (the unit of the GB/s metric)."""
    return 2 * 2 * spec.batch * spec.n_layers * spec.n_heads * spec.seq_len * spec.head_dim


def _gen(device: str, *key: int) -> torch.Generator:
    s = 0x9E3779B97F4A7C15
    for k in key:
        s = (s * 0x100000001B3 + (k & 0xFFFFFFFF) + 0x51) & 0x7FFFFFFFFFFFFFFF
    g = torch.Generator(device=device)
    g.manual_seed(s)
    return g


def _haar(n: int, r: int, g: torch.Generator, device: str) -> torch.Tensor:
    z = torch.randn(n, r, generator=g, device=device, dtype=torch.float64 if device == "cpu" else torch.float32)
    q, rr = torch.linalg.qr(z)
    d = torch.sign(torch.diagonal(rr))
    d[d == 0] = 1
    return q * d


def _outlier_channels(spec: CacheSpec, seed: int, device: str) -> torch.Tensor:
    g = _gen("cpu", seed, 0xC0FFEE)
    return torch.randperm(spec.head_dim, generator=g)[: spec.k_outliers].to(device)


def _rope_inplace(x: torch.Tensor, theta: float) -> None:
    """x: [..., T, D] float; rotate-half pairing, positions 0..T-1 (fp64 angles)."""
    T, D = x.shape[-2], x.shape[-1]
    half = D // 2
    inv = theta ** (-2.0 * torch.arange(half, dtype=torch.float64) / D)
    ang = torch.arange(T, dtype=torch.float64)[:, None] * inv[None, :]
    c = torch.cos(ang).to(x.device, x.dtype)
    s = torch.sin(ang).to(x.device, x.dtype)
    a = x[..., :half].clone()
    b = x[..., half:].clone()
    x[..., :half] = a * c - b * s
    x[..., half:] = b * c + a * s


def make_group(spec: CacheSpec, seed: int, b: int, g: int, kind: int,
               device: str = "cpu") -> torch.Tensor:
    """One cell [L_g, H, T, D] for sequence b, group g, kind 0=K / 1=V, as float
    (fp64 on CPU, fp32 on GPU) BEFORE the final storage rounding."""
    gs = group_starts(spec)
    Lg = gs[g + 1] - gs[g]
    H, T, D, R = spec.n_heads, spec.seq_len, spec.head_dim, spec.rank
    R = min(R, D, T)
    gen = _gen(device, seed, b, g, kind)
    ftype = torch.float64 if device == "cpu" else torch.float32
    A = _haar(T, R, gen, device).to(ftype)
    F = _haar(D, R, gen, device).to(ftype)
    sig = torch.arange(1, R + 1, dtype=ftype, device=device) ** (-spec.sigma_exp)
    out = torch.empty(Lg, H, T, D, dtype=ftype, device=device)
    ch = _outlier_channels(spec, seed, device) if (kind == 0 and spec.k_outliers > 0) else None
    for l in range(Lg):
        for h in range(H):
            W = _haar(R, R, gen, device).to(ftype)
            S = (A * sig[None, :]) @ (W @ F.T)
            if ch is not None:
                S[:, ch] *= spec.outlier_scale
            n = torch.randn(T, D, generator=gen, device=device, dtype=ftype)
            ns = torch.linalg.vector_norm(S)
            nn = torch.linalg.vector_norm(n)
            x = S + n * (math.sqrt(spec.noise) * ns / nn)
            x = x * (1.0 / torch.sqrt(torch.mean(x * x)))
            out[l, h] = x
    if kind == 0 and spec.rope_theta_k > 0:
        _rope_inplace(out, spec.rope_theta_k)
    return out


def make_cache(spec: CacheSpec, seed: int = 0, device: str = "cpu",
               groups: Optional[List[int]] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """K and V as [B, L, H, T, D] in the storage dtype (bf16 or fp32).

    ``groups`` restricts generation to a subset of layer groups (the other
    layers stay zero), which lets a test rebuild exactly the layers of one
    group of a large config without generating the rest."""
    dt = torch.bfloat16 if spec.dtype == "bf16" else torch.float32
    shape = (spec.batch, spec.n_layers, spec.n_heads, spec.seq_len, spec.head_dim)
    K = torch.zeros(shape, dtype=dt, device=device)
    V = torch.zeros(shape, dtype=dt, device=device)
    gs = group_starts(spec)
    for b in range(spec.batch):
        for g in range(len(gs) - 1):
            if groups is not None and g not in groups:
                continue
            for kind, dst in ((0, K), (1, V)):
                cell = make_group(spec, seed + b, b, g, kind, device)
                dst[b, gs[g]:gs[g + 1]] = cell.to(dt)
    return K, V
