"""Seeded synthetic inputs for the residual binarized linear layer.

This module draws random layers and activations only.  It holds none of the
method's arithmetic (no sign, residual, scale or packing step), so that the
CUDA path and the CPU oracle can both consume its output without sharing any
part of the computation they are checked on.

Recipe (all draws from numpy's PCG64 ``default_rng(seed)``, in float64, then
cast with round-to-nearest-even):
  * weights: N(0, std) or Laplace(0, b); optional outliers: floor(frac*N*K)
    distinct positions chosen uniformly without replacement, multiplied by
    ``mult``; cast to float32.
  * activations: N(0, 1); optional heavy columns: ceil(frac*K) distinct
    columns multiplied by ``mult``; cast float64 -> float32 -> bfloat16.
  * seeds: layer weights use 100*cfg + layer, activations 100*cfg + 50 + M
    (the first workload fixes weight seed 0).

The workload shapes follow the Llama-7B-style layers the method is reported
on (RaBiT, inference-speed paragraph: a 4096 x 4096 q_proj kernel); real
model weights are not used.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class Layer:
    name: str
    n_out: int
    k_in: int
    dist: str          # "normal" or "laplace"
    scale: float       # std for normal, b for laplace
    outlier_frac: float = 0.0
    outlier_mult: float = 1.0
    seed: int = 0


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    index: int
    layers: tuple
    k_planes: tuple    # plane counts exercised
    tokens: tuple      # M values
    x_col_frac: float = 0.0
    x_col_mult: float = 1.0


def _w(cfg, li, name, n, k, dist, scale, **kw):
    return Layer(name, n, k, dist, scale, seed=kw.pop("seed", 100 * cfg + li), **kw)


WORKLOADS = (
    Workload("single_k1_256x512", 0,
             (_w(0, 0, "layer", 256, 512, "normal", 0.02, seed=0),), (1,), (1,)),
    Workload("q_proj_4096x4096_k2", 1,
             (_w(1, 0, "q_proj", 4096, 4096, "normal", 0.02,
                 outlier_frac=1e-3, outlier_mult=20.0),), (2,), (1, 4, 16)),
    Workload("mlp_trio_7b_k2", 2,
             (_w(2, 0, "gate", 11008, 4096, "normal", 0.02),
              _w(2, 1, "up", 11008, 4096, "normal", 0.02),
              _w(2, 2, "down", 4096, 11008, "normal", 0.02)), (2,), (1, 8)),
    Workload("mlp_28672x8192", 3,
             (_w(3, 0, "mlp", 28672, 8192, "normal", 0.015),), (1, 2), (1, 16, 64)),
    Workload("prefill_14336x4096_k2", 4,
             (_w(4, 0, "up", 14336, 4096, "laplace", 0.01),
              _w(4, 1, "down", 4096, 14336, "laplace", 0.01)), (2,), (512, 2048),
             x_col_frac=0.01, x_col_mult=10.0),
)


def workload(name_or_index) -> Workload:
    for w in WORKLOADS:
        if w.name == name_or_index or w.index == name_or_index:
            return w
    raise KeyError(name_or_index)


def weights(layer: Layer, n_out: int | None = None, k_in: int | None = None) -> np.ndarray:
    """float32 [N][K] weight matrix of `layer` (shape overridable for small cases)."""
    n = layer.n_out if n_out is None else n_out
    k = layer.k_in if k_in is None else k_in
    rng = np.random.default_rng(layer.seed)
    if layer.dist == "normal":
        w = rng.standard_normal((n, k)) * layer.scale
    elif layer.dist == "laplace":
        w = rng.laplace(0.0, layer.scale, (n, k))
    else:
        raise ValueError(layer.dist)
    if layer.outlier_frac > 0:
        cnt = int(math.floor(layer.outlier_frac * n * k))
        pos = rng.choice(n * k, size=cnt, replace=False)
        w.reshape(-1)[pos] *= layer.outlier_mult
    return w.astype(np.float32)


def to_bf16_bits(a32: np.ndarray) -> np.ndarray:
    """float32 -> bfloat16 bit patterns (uint16), round-to-nearest-even."""
    t = torch.from_numpy(np.ascontiguousarray(a32, np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def activations(M: int, K: int, seed: int, col_frac: float = 0.0, col_mult: float = 1.0) -> np.ndarray:
    """bfloat16 bit patterns [M][K] of N(0,1) activations (optional heavy columns)."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((M, K))
    if col_frac > 0:
        cols = rng.choice(K, size=int(math.ceil(col_frac * K)), replace=False)
        x[:, cols] *= col_mult
    return to_bf16_bits(x.astype(np.float32))


def activations_for(wl: Workload, M: int, K: int) -> np.ndarray:
    return activations(M, K, 100 * wl.index + 50 + M, wl.x_col_frac, wl.x_col_mult)


def positive_scales(k: int, N: int, K: int, seed: int, lo: float = 0.05, hi: float = 0.5):
    """Random positive fp32 scales (g [k][N], h [k][K]) drawn uniformly in [lo, hi).

    Used by edge-case tests where the scale values are arbitrary inputs.
    """
    rng = np.random.default_rng(seed)
    g = rng.uniform(lo, hi, (k, N)).astype(np.float32)
    h = rng.uniform(lo, hi, (k, K)).astype(np.float32)
    return g, h
