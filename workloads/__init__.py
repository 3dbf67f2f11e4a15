"""Seeded synthetic inputs for the ButterflyMoE expert forward.

This module only draws random numbers.  It holds none of the method's
arithmetic (no rotation, no routing, no packing).  The CPU oracle (test
infrastructure) and the CUDA path both take their inputs from here, and they
share nothing else.

The five named workloads follow the layer sizes of the ButterflyMoE pages:
d x d experts over a shared ternary base (gist.science ButterflyMoE summary,
"2.1 basic parametrisation"), d=512 with 64 and 256 experts as in the
memory examples ("1. problem definition" and "4. results").  The pages name
no dataset, so synthetic tokens stand in for their unnamed language-modelling
benchmarks.

Recipe (one ``numpy.random.default_rng(seed)`` per workload, draws in this
fixed order, each drawn in float64):

1. ``w_base``  [d, d]: u ~ U[0,1); 0 where u < p0, +1 where
   p0 <= u < p0 + (1-p0)/2, else -1.  Stored int8.
2. ``theta``   [N, log2 d, d/2]: U[-pi, pi), rounded to float32.
3. ``phi``     [N, log2 d, d/2]: U[-pi, pi), rounded to float32.
4. ``w_gate``  [N, d]: N(0, variance 1/d), rounded to float32.
5. ``bias``    [N]: N(0, variance bias_var), float32, only when bias_var > 0.
6. outlier channel set: ``round(outlier_frac * d)`` distinct channels drawn
   without replacement (only when outlier_frac > 0).
7. ``x``       [T, d]: N(0, 1); the outlier columns are multiplied by
   ``outlier_scale``; rounded to float32, then to bfloat16 (round to nearest
   even, via torch) for bf16 workloads.

``alpha`` is float32(1/sqrt(d)).  A shorter token count draws a prefix of the
full token matrix, so a token sample is the first rows of the full workload.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    d: int
    n_experts: int
    k: int
    tokens: int
    dtype: str            # "f32" or "bf16": the dtype of x and y
    p0: float = 0.4       # P(W_base == 0); +1 and -1 share the rest equally
    bias_var: float = 0.0  # router bias variance (0: no bias)
    outlier_frac: float = 0.0
    outlier_scale: float = 1.0

    @property
    def stages(self) -> int:
        return int(round(math.log2(self.d)))

    @property
    def rows(self) -> int:
        return self.tokens * self.k

    def with_tokens(self, tokens: int) -> "Workload":
        return dataclasses.replace(self, tokens=tokens)

    def describe(self) -> str:
        return (f"{self.name}: d={self.d} N={self.n_experts} top-{self.k} "
                f"T={self.tokens} {self.dtype}")


# The five workloads: sizes and distributions as stated for each.
WORKLOADS = {
    "tiny_f32": Workload("tiny_f32", d=64, n_experts=8, k=2, tokens=256,
                         dtype="f32", p0=0.4),
    "d512_n64": Workload("d512_n64", d=512, n_experts=64, k=2, tokens=4096,
                         dtype="bf16", p0=0.4, outlier_frac=0.01,
                         outlier_scale=20.0),
    "d512_n256": Workload("d512_n256", d=512, n_experts=256, k=2, tokens=16384,
                          dtype="bf16", p0=0.4, bias_var=0.5),
    "d1024_n256": Workload("d1024_n256", d=1024, n_experts=256, k=2,
                           tokens=65536, dtype="bf16", p0=0.5,
                           outlier_frac=0.01, outlier_scale=20.0),
    "d2048_n1024": Workload("d2048_n1024", d=2048, n_experts=1024, k=4,
                            tokens=131072, dtype="bf16", p0=0.4, bias_var=1.0,
                            outlier_frac=0.005, outlier_scale=50.0),
}

# The headline workload that the throughput metric is quoted on.
HEADLINE = "d512_n256"


@dataclasses.dataclass
class Inputs:
    wl: Workload
    w_base: np.ndarray          # int8 [d, d], values in {-1, 0, +1}
    alpha: np.float32
    theta: np.ndarray           # float32 [N, L, d/2]
    phi: np.ndarray             # float32 [N, L, d/2]
    w_gate: np.ndarray          # float32 [N, d]
    bias: Optional[np.ndarray]  # float32 [N] or None
    outliers: np.ndarray        # int64 channel ids (possibly empty)
    x: "object"                 # torch tensor [T, d], float32 or bfloat16 (CPU)

    def x_f64(self) -> np.ndarray:
        """The stored token values, exactly, as float64."""
        return self.x.float().double().numpy()


def generate(wl: Workload, seed: int = 0, tokens: Optional[int] = None, token_offset: int = 0) -> Inputs:
    """Draw the inputs of ``wl`` (see the module docstring for the recipe).

    ``token_offset`` returns rows [token_offset, token_offset + tokens) of a
    longer token draw (one shard of a larger batch, same weights)."""
    import torch

    d, n = wl.d, wl.n_experts
    if d < 2 or d & (d - 1):
        raise ValueError("d must be a power of two >= 2")
    T = wl.tokens if tokens is None else int(tokens)
    L = wl.stages
    rng = np.random.default_rng(seed)

    u = rng.random((d, d))
    half = (1.0 - wl.p0) / 2.0
    w_base = np.where(u < wl.p0, 0, np.where(u < wl.p0 + half, 1, -1)).astype(np.int8)

    theta = rng.uniform(-np.pi, np.pi, size=(n, L, d // 2)).astype(np.float32)
    phi = rng.uniform(-np.pi, np.pi, size=(n, L, d // 2)).astype(np.float32)
    w_gate = rng.normal(0.0, 1.0 / math.sqrt(d), size=(n, d)).astype(np.float32)
    bias = None
    if wl.bias_var > 0:
        bias = rng.normal(0.0, math.sqrt(wl.bias_var), size=(n,)).astype(np.float32)
    n_out = int(round(wl.outlier_frac * d))
    outliers = (rng.choice(d, size=n_out, replace=False) if n_out > 0
                else np.zeros((0,), dtype=np.int64))
    x = rng.normal(0.0, 1.0, size=(token_offset + T, d))[token_offset:]
    if n_out > 0:
        x[:, outliers] *= wl.outlier_scale
    xt = torch.from_numpy(x.astype(np.float32))
    if wl.dtype == "bf16":
        xt = xt.to(torch.bfloat16)
    elif wl.dtype != "f32":
        raise ValueError(f"unknown dtype {wl.dtype}")
    alpha = np.float32(1.0 / math.sqrt(d))
    return Inputs(wl, w_base, alpha, theta, phi, w_gate, bias,
                  np.asarray(outliers, dtype=np.int64), xt)


def custom(name: str, d: int, n_experts: int, k: int, tokens: int,
           dtype: str = "bf16", **kw) -> Workload:
    """A small workload of the same family, for tests (tails, edge cases)."""
    return Workload(name, d=d, n_experts=n_experts, k=k, tokens=tokens,
                    dtype=dtype, **kw)
