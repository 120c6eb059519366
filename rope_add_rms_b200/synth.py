"""Seeded synthetic inputs for the fused row-normalisation workloads.

This is the one module that both the CUDA path's tests/benchmark and the CPU oracle's
callers use.  It draws random numbers and rounds them to the I/O type; it performs
none of the normalisation arithmetic.

Recipe: every tensor comes from its own ``torch.Generator('cpu')`` seeded with
``seed + k`` (k = 0 for x, 1 for r, 2 for w, 3 for b), drawn as float32 ``randn`` or
``rand``, shifted and scaled as the workload says, and rounded once (to nearest, ties to
even) to the I/O type.  The value distributions follow the decoder workloads the pages
describe: activations ~ N(0, 1), learned scales ~ U(0.5, 1.5), biases ~ N(0, 0.1^2),
LayerNorm input ~ N(0.5, 2^2) (non-zero mean).
"""
from __future__ import annotations

import numpy as np
import torch

X, R, W, B = 0, 1, 2, 3

DTYPES = {"bf16": torch.bfloat16, "f32": torch.float32}


def _gen(seed: int, k: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed) + int(k))
    return g


def normal(shape, mean, std, seed, k, dtype="bf16") -> torch.Tensor:
    """N(mean, std^2) draws, float32, rounded to ``dtype`` (a CPU tensor)."""
    t = torch.randn(tuple(shape), generator=_gen(seed, k), dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    if mean != 0.0:
        t.add_(mean)
    return t.to(DTYPES[dtype])


def uniform(shape, lo, hi, seed, k, dtype="bf16") -> torch.Tensor:
    """U(lo, hi) draws, float32, rounded to ``dtype`` (a CPU tensor)."""
    t = torch.rand(tuple(shape), generator=_gen(seed, k), dtype=torch.float32)
    t.mul_(hi - lo).add_(lo)
    return t.to(DTYPES[dtype])


def normal_device(shape, mean, std, seed, k, dtype="bf16", device="cuda") -> torch.Tensor:
    """N(mean, std^2) drawn by torch's generator on `device` (for inputs too large to
    draw on the host quickly), float32, rounded to ``dtype``."""
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) + int(k))
    t = torch.randn(tuple(shape), generator=g, dtype=torch.float32, device=device)
    if std != 1.0:
        t.mul_(std)
    if mean != 0.0:
        t.add_(mean)
    return t.to(DTYPES[dtype])


def uniform_device(shape, lo, hi, seed, k, dtype="bf16", device="cuda") -> torch.Tensor:
    """U(lo, hi) drawn by torch's generator on `device`, rounded to ``dtype``."""
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) + int(k))
    t = torch.rand(tuple(shape), generator=g, dtype=torch.float32, device=device)
    t.mul_(hi - lo).add_(lo)
    return t.to(DTYPES[dtype])


def to_numpy(t: torch.Tensor) -> np.ndarray:
    """The oracle's view of a CPU tensor: bfloat16 as raw uint16 bits, float32 as is."""
    t = t.contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype == torch.float32:
        return t.numpy()
    raise TypeError(f"unsupported dtype {t.dtype}")


# ---- workload recipes -------------------------------------------------------------

def rms_inputs(rows, D, dtype="f32", seed=0, weight=True):
    """rms_norm: x ~ N(0,1) [rows, D], w ~ U(0.5,1.5) [D]."""
    return {"x": normal((rows, D), 0.0, 1.0, seed, X, dtype),
            "w": uniform((D,), 0.5, 1.5, seed, W, dtype) if weight else None}


def add_rms_inputs(rows, D, dtype="bf16", seed=0, weight=True):
    """add_rms_norm: x, r ~ N(0,1) [rows, D], w ~ U(0.5,1.5) [D]."""
    return {"x": normal((rows, D), 0.0, 1.0, seed, X, dtype),
            "r": normal((rows, D), 0.0, 1.0, seed, R, dtype),
            "w": uniform((D,), 0.5, 1.5, seed, W, dtype) if weight else None}


def allreduce_inputs(rows, D, nparts, dtype="bf16", seed=0, weight=True):
    """all-reduce + add_rms_norm: nparts partial outputs ~ N(0, 1/nparts) each (their sum
    ~ N(0, 1), like the shards of a row-parallel layer), r ~ N(0,1), w ~ U(0.5,1.5)."""
    sd = 1.0 / nparts ** 0.5
    return {"parts": [normal((rows, D), 0.0, sd, seed, 16 + i, dtype) for i in range(nparts)],
            "r": normal((rows, D), 0.0, 1.0, seed, R, dtype),
            "w": uniform((D,), 0.5, 1.5, seed, W, dtype) if weight else None}


def layer_norm_inputs(rows, D, dtype="bf16", seed=0, weight=True, bias=True):
    """layer_norm: x ~ N(0.5, 2^2), w ~ U(0.5,1.5), b ~ N(0, 0.1^2)."""
    return {"x": normal((rows, D), 0.5, 2.0, seed, X, dtype),
            "w": uniform((D,), 0.5, 1.5, seed, W, dtype) if weight else None,
            "b": normal((D,), 0.0, 0.1, seed, B, dtype) if bias else None}


def norm_rope_inputs(Bsz, H, L, D, dtype="bf16", seed=0, weight=True):
    """norm_rope: x ~ N(0,1) [B, H, L, D] (flattened to rows), w ~ U(0.5,1.5) [D]."""
    return {"x": normal((Bsz * H * L, D), 0.0, 1.0, seed, X, dtype),
            "w": uniform((D,), 0.5, 1.5, seed, W, dtype) if weight else None}
