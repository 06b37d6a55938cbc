"""Seeded synthetic inputs for the rotate+quantise hot path and the W4A4 linear.

This module holds only random draws and the table of workload shapes. It contains
none of the method's arithmetic (no rotation, no quantisation, no block
construction): the random numbers the method consumes (±1 signs, Givens angles,
Gaussian matrices for the QR fallback mixer, stage permutations) are produced here
and handed, unchanged, to both the fp64 oracle and the CUDA library, which each
build what they need from them on their own.

Recipe (every generator is numpy ``Generator(PCG64(seed))``):

* activations ``A[M,K]``: base distribution drawn in float64 (``standard_normal``
  or ``standard_t(nu) * t_scale``), cast to float32; then ``ceil(frac*K)`` outlier
  channels are chosen with ``rng.choice(K, n, replace=False)`` and multiplied by
  the outlier factor in float32; bf16 workloads then round to bfloat16
  (round-to-nearest-even) -- the returned float32 array holds the exact bf16
  values.
* signs: drawn from the same generator right after the activations,
  ``1 - 2*rng.integers(0, 2, K)`` as int8.
* weights ``W[K,N]``: ``standard_normal * std`` from ``PCG64(seed + 1)``.
* HARP random draws from ``PCG64(seed + 2)``: per radix-2 stage ``K/2`` angles
  uniform in ``[-pi, pi)``; per non-power-of-two stage one (or ``K/b``) ``b x b``
  standard-normal matrices; one permutation of ``range(K)`` after every stage but
  the last.

The page workloads these shapes stand in for (page 1's Llama-3.2-1B activations,
page 2's synthetic and GGUF probes, pages 3/4's Llama 2 7B layers) are not in the
container; these seeded inputs replace them.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

__all__ = [
    "rng",
    "activations",
    "signs",
    "weights",
    "HarpDraws",
    "harp_draws",
    "HarpQ8Draws",
    "harp_q8_draws",
    "to_bf16_exact",
    "WORKLOADS",
    "Workload",
    "make_workload",
]


def rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def to_bf16_exact(a32: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (nearest-even) and return them as float32.

    Input preparation only; uses torch's CPU cast as the library routine.
    """
    import torch

    t = torch.from_numpy(np.ascontiguousarray(a32, dtype=np.float32))
    return t.to(torch.bfloat16).to(torch.float32).numpy()


def activations(
    g: np.random.Generator,
    M: int,
    K: int,
    *,
    dist: str = "normal",
    t_nu: float = 4.0,
    t_scale: float = 1.0,
    outlier_frac: float = 0.0,
    outlier_scale: float = 1.0,
    bf16: bool = True,
) -> np.ndarray:
    """Draw A[M,K] (float32 holding exact bf16 values when ``bf16``)."""
    if dist == "normal":
        a = g.standard_normal((M, K))
    elif dist == "student_t":
        a = g.standard_t(t_nu, (M, K)) * t_scale
    else:
        raise ValueError(dist)
    a = a.astype(np.float32)
    n_out = int(math.ceil(outlier_frac * K)) if outlier_frac > 0 else 0
    if n_out:
        ch = g.choice(K, n_out, replace=False)
        a[:, ch] *= np.float32(outlier_scale)
    if bf16:
        a = to_bf16_exact(a)
    return a


def signs(g: np.random.Generator, K: int) -> np.ndarray:
    return (1 - 2 * g.integers(0, 2, K)).astype(np.int8)


def weights(seed: int, K: int, N: int, std: float) -> np.ndarray:
    g = rng(seed)
    return (g.standard_normal((K, N)) * std).astype(np.float32)


@dataclass
class HarpDraws:
    """Raw random numbers of a HARP processor (no blocks built here)."""

    radices: list[int]
    angles: list[np.ndarray | None] = field(default_factory=list)   # radix-2 stages: [K/2]
    gaussians: list[np.ndarray | None] = field(default_factory=list)  # other radices: [n, b, b]
    perms: list[np.ndarray | None] = field(default_factory=list)    # after stage t: [K] int32


def harp_draws(seed: int, radices: list[int], *, per_block_gaussian: bool = False,
               with_perms: bool = True) -> HarpDraws:
    K = int(np.prod(radices))
    g = rng(seed)
    d = HarpDraws(list(radices))
    for t, b in enumerate(radices):
        if b == 2:
            d.angles.append(g.uniform(-np.pi, np.pi, K // 2))
            d.gaussians.append(None)
        else:
            n = K // b if per_block_gaussian else 1
            d.angles.append(None)
            d.gaussians.append(g.standard_normal((n, b, b)))
    for t in range(len(radices)):
        if with_perms and t < len(radices) - 1:
            d.perms.append(g.permutation(K).astype(np.int32))
        else:
            d.perms.append(None)
    return d


@dataclass
class HarpQ8Draws:
    """Raw random numbers of a HARP processor stored with int8 parameters: per stage int8 codes
    and an fp32 scale (theta = code * scale); Givens stages (b = 2) hold one code per block, the
    other stages b(b-1)/2 Cayley codes per block and, for a non-power-of-two radix, a Gaussian
    b x b matrix whose QR factor is the fallback base mixer. No block is built here."""

    radices: list[int]
    codes: list[np.ndarray] = field(default_factory=list)           # [n_blocks] or [n_blocks, b(b-1)/2] int8
    scales: list[float] = field(default_factory=list)
    mixer_gaussians: list[np.ndarray | None] = field(default_factory=list)
    perms: list[np.ndarray | None] = field(default_factory=list)


def harp_q8_draws(seed: int, radices: list[int], *, per_block: bool = True, with_perms: bool = True,
                  cayley_range: float = 0.3) -> HarpQ8Draws:
    """Seeded int8-stored HARP parameters: codes uniform in [-127, 127]; Givens scale pi / 127
    (angles over [-pi, pi]), Cayley scale cayley_range / 127."""
    K = int(np.prod(radices))
    g = rng(seed)
    d = HarpQ8Draws(list(radices))
    for b in radices:
        n = K // b if per_block else 1
        if b == 2:
            d.codes.append(g.integers(-127, 128, n).astype(np.int8))
            d.scales.append(float(np.float32(np.pi / 127)))
            d.mixer_gaussians.append(None)
        else:
            d.codes.append(g.integers(-127, 128, (n, b * (b - 1) // 2)).astype(np.int8))
            d.scales.append(float(np.float32(cayley_range / 127)))
            d.mixer_gaussians.append(None if (b & (b - 1)) == 0 else g.standard_normal((b, b)))
    for t in range(len(radices)):
        d.perms.append(g.permutation(K).astype(np.int32) if (with_perms and t < len(radices) - 1) else None)
    return d


@dataclass
class Workload:
    name: str
    M: int
    K: int
    A: np.ndarray            # float32 values (exact bf16 when bf16)
    bf16: bool
    signs: np.ndarray        # int8 [K]
    quant: list[tuple[int, int]]  # (bits, G) pairs this workload is run with
    W: np.ndarray | None = None   # float32 [K, N]
    extra: dict = field(default_factory=dict)


# Shapes and recipes of the five workloads (sizes as in the page workloads they stand in for).
WORKLOADS = {
    # page 2 synthetic probe (M=16, K=2048, N=512, x20 outliers), fp32 activations
    "pr1": dict(M=16, K=2048, dist="normal", frac=0.01, scale=20.0, bf16=False,
                quant=[(4, 128), (4, 32)], N=512, w_std=0.02),
    # Llama-3.2-1B hidden size 2048, heavy tails, strong outliers
    "llama32_1b": dict(M=8192, K=2048, dist="student_t", t_scale=0.5, frac=0.005, scale=100.0,
                       bf16=True, quant=[(4, 32)]),
    # MLP down_proj input, K=8192
    "down_proj": dict(M=4096, K=8192, dist="normal", frac=0.005, scale=50.0, bf16=True,
                      quant=[(4, 128), (2, 64)]),
    # HARP mixed radix K=11008 = 2^8 * 43
    "harp11008": dict(M=4096, K=11008, dist="normal", frac=0.01, scale=20.0, bf16=True,
                      quant=[(4, 128), (2, 64)], radices=[2] * 8 + [43]),
    # W4A4 linear, Llama-2-7B q_proj (N=4096) and up_proj (N=11008), K=4096
    "q_proj_prefill": dict(M=2048, K=4096, dist="normal", frac=0.01, scale=20.0, bf16=True,
                           quant=[(4, 128)], N=4096, w_std=0.02),
    "q_proj_decode": dict(M=16, K=4096, dist="normal", frac=0.01, scale=20.0, bf16=True,
                          quant=[(4, 128)], N=4096, w_std=0.02),
    "up_proj_prefill": dict(M=2048, K=4096, dist="normal", frac=0.01, scale=20.0, bf16=True,
                            quant=[(4, 128)], N=11008, w_std=0.02),
    "up_proj_decode": dict(M=16, K=4096, dist="normal", frac=0.01, scale=20.0, bf16=True,
                           quant=[(4, 128)], N=11008, w_std=0.02),
}


def make_workload(name: str, seed: int = 0, *, M: int | None = None) -> Workload:
    """Build one workload; ``M`` overrides the row count (same recipe, fewer rows)."""
    cfg = WORKLOADS[name]
    Mr = cfg["M"] if M is None else M
    g = rng(seed)
    A = activations(g, Mr, cfg["K"], dist=cfg["dist"], t_scale=cfg.get("t_scale", 1.0),
                    outlier_frac=cfg["frac"], outlier_scale=cfg["scale"], bf16=cfg["bf16"])
    s = signs(g, cfg["K"])
    W = None
    if "N" in cfg:
        W = weights(seed + 1, cfg["K"], cfg["N"], cfg["w_std"])
    wl = Workload(name, Mr, cfg["K"], A, cfg["bf16"], s, list(cfg["quant"]), W)
    if "radices" in cfg:
        wl.extra["radices"] = list(cfg["radices"])
    return wl
