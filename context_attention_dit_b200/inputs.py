"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle checks.

This module only draws numbers; it holds none of the attention arithmetic.
The workloads stand in for the DiT attention calls the context-parallelism
pages benchmark (FLUX.1-dev at 1024x1024, video DiTs): their weights and
prompts are not available, and the attention op only needs tensors of the
right shape and value distribution.

Recipe: ``torch.Generator("cpu").manual_seed(seed + i)`` for i = 0, 1, 2
(Q, K, V), iid N(0, 1) float32, optionally a per-(b, s, h) RMS normalisation
over the head dimension (``x / sqrt(mean(x^2) + 1e-6)``, weight 1, the QK-norm
that FLUX-style DiTs apply to Q and K before attention), then rounded to
bfloat16.  Seed 42 follows the pages' own example generator.
"""

from __future__ import annotations

import hashlib
from dataclasses import dataclass, field

import torch

DEFAULT_SEED = 42


def randn_bf16(shape, seed: int, rms_norm: bool = False) -> torch.Tensor:
    """One seeded bf16 CPU tensor of iid N(0,1) values (optionally RMS-normalised over the last dim)."""
    g = torch.Generator(device="cpu").manual_seed(int(seed))
    x = torch.randn(*shape, generator=g, dtype=torch.float32)
    if rms_norm:
        x = x * torch.rsqrt(x.pow(2).mean(dim=-1, keepdim=True) + 1e-6)
    return x.to(torch.bfloat16)


def make_qkv(B: int, H: int, Sq: int, Skv: int, D: int, seed: int = DEFAULT_SEED, rms_norm_qk: bool = False):
    """Q ``[B,Sq,H,D]``, K and V ``[B,Skv,H,D]`` as bf16 CPU tensors (BSHD layout)."""
    q = randn_bf16((B, Sq, H, D), seed + 0, rms_norm_qk)
    k = randn_bf16((B, Skv, H, D), seed + 1, rms_norm_qk)
    v = randn_bf16((B, Skv, H, D), seed + 2, False)
    return q, k, v


def sha256(t: torch.Tensor) -> str:
    """SHA-256 of a tensor's raw bytes (recorded next to results so inputs can be traced)."""
    t = t.detach().contiguous().cpu()
    return hashlib.sha256(t.view(torch.uint8).numpy().tobytes()).hexdigest()


def even_bounds(S: int, n: int):
    """Chunk bounds of an even split of ``S`` rows into ``n`` blocks (``S % n == 0``)."""
    assert S % n == 0
    return [i * (S // n) for i in range(n + 1)]


def bounds_from_sizes(sizes):
    """Chunk bounds ``[0, s0, s0+s1, ...]`` from a list of block sizes."""
    out = [0]
    for s in sizes:
        out.append(out[-1] + int(s))
    return out


@dataclass(frozen=True)
class Workload:
    """One synthetic attention workload (shape, input recipe and K/V splits)."""

    name: str
    B: int
    H: int
    S: int
    D: int
    rms_norm_qk: bool
    splits: tuple = field(default_factory=tuple)   # each split: tuple of block sizes
    ulysses_degree: int = 1

    @property
    def scale(self) -> float:
        return 1.0 / (self.D ** 0.5)

    @property
    def flop(self) -> int:
        """Algorithmic attention FLOP: two GEMMs, 4*B*H*Sq*Skv*D."""
        return 4 * self.B * self.H * self.S * self.S * self.D

    def qkv(self, seed: int = DEFAULT_SEED):
        return make_qkv(self.B, self.H, self.S, self.S, self.D, seed, self.rms_norm_qk)


# The five workloads: a tiny case, FLUX.1-dev 1024x1024 joint attention
# (4096 image + 512 text tokens, 24 heads of 128), the same shape split over a
# ring of 8 plus a Ulysses degree-8 exchange, an uneven "ring anything" split,
# and a long video-DiT sequence (21 latent frames x 1560 tokens, 40 heads).
WORKLOADS = {
    "tiny_s256_d64": Workload("tiny_s256_d64", 1, 2, 256, 64, False, ((128, 128),)),
    "flux_1024_ring1": Workload("flux_1024_ring1", 1, 24, 4608, 128, True, ((4608,),)),
    "flux_1024_ring8_ulysses8": Workload("flux_1024_ring8_ulysses8", 1, 24, 4608, 128, True,
                                         ((576,) * 8,), ulysses_degree=8),
    "uneven_s4173_ring3": Workload("uneven_s4173_ring3", 2, 24, 4173, 128, False,
                                   ((1391, 1391, 1391), (1392, 1391, 1390))),
    "video_s32760_ring4": Workload("video_s32760_ring4", 1, 40, 32760, 128, True, ((8190,) * 4,)),
}
