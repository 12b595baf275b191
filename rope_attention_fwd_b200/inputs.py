"""Seeded synthetic inputs shared by the CUDA path's tests/bench and the oracle.

This module holds no part of the attention arithmetic: it only draws random
numbers and rounds them to the storage type.  Recipe (fixed, so both sides see
identical values):

* generator: ``numpy.random.default_rng(seed)`` (PCG64);
* draw order: Q, K, V, E (each [B, H, n, d]) and then alpha ([d/2]);
* every value is drawn in float64 and rounded once, round-to-nearest-even,
  to the workload's dtype (bf16 or fp32); alpha is always rounded to fp32;
* the float64 copies handed to the oracle are those rounded values, widened
  exactly, so the comparison measures kernel error only.
"""
from dataclasses import dataclass

import numpy as np
import torch

from .configs import Workload

TORCH_DTYPE = {"f32": torch.float32, "bf16": torch.bfloat16}


@dataclass
class Inputs:
    wl: Workload
    q: torch.Tensor      # [B, H, n, d] in the workload dtype (CPU)
    k: torch.Tensor
    v: torch.Tensor
    e: torch.Tensor
    alpha: torch.Tensor  # [d/2] float32 (CPU)

    def f64(self, name: str) -> np.ndarray:
        """Exact float64 widening of one stored tensor, for the oracle."""
        return getattr(self, name).to(torch.float64).numpy()


def _draw(rng: np.random.Generator, shape, kind: str, lo: float, hi: float) -> np.ndarray:
    if kind == "normal":
        return rng.standard_normal(shape)
    if kind == "uniform":
        return rng.uniform(lo, hi, shape)
    raise ValueError(f"unknown distribution {kind!r}")


def _draw_alpha(rng: np.random.Generator, wl: Workload) -> np.ndarray:
    if wl.alpha == "zero":
        return np.zeros(wl.M)
    if wl.alpha == "normal":
        return wl.alpha_a * rng.standard_normal(wl.M)
    if wl.alpha == "uniform":
        return rng.uniform(wl.alpha_a, wl.alpha_b, wl.M)
    raise ValueError(f"unknown alpha distribution {wl.alpha!r}")


def make_inputs(wl: Workload, seed: int = None) -> Inputs:
    """Draw Q, K, V, E, alpha for ``wl`` (seed defaults to the workload's own)."""
    rng = np.random.default_rng(wl.seed if seed is None else seed)
    shape = (wl.B, wl.H, wl.n, wl.d)
    td = TORCH_DTYPE[wl.dtype]
    out = {}
    for name in ("q", "k", "v", "e"):
        x = _draw(rng, shape, wl.qkve, wl.lo, wl.hi)
        out[name] = torch.from_numpy(x).to(td)
        del x
    alpha = torch.from_numpy(_draw_alpha(rng, wl)).to(torch.float32)
    return Inputs(wl, out["q"], out["k"], out["v"], out["e"], alpha)
