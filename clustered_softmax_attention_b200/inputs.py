"""Seeded synthetic inputs for the MuSe forward pass.

This module draws numbers and nothing else: it holds none of the method's
arithmetic, so both the float64 oracle (tests, CPU baseline) and the CUDA path
(tests, bench) take their inputs from here.

Recipe, per (batch, head), drawn in this order from one
``numpy.random.Generator(PCG64(seed))`` in float64:

1. ``M`` component means, each ~ N(0, I/D);
2. queries: a component index uniform over the M components, then
   ``q = mean[idx] + sigma * N(0, I)``;
3. keys: an independent draw from the same means, same recipe;
4. values ~ N(0, I) of width Dv;
5. (outlier workloads only) exactly ``round(frac * N)`` key rows, picked without
   replacement, multiplied by ``outlier_scale``.

The float64 draws are then cast to float32, or rounded to bfloat16 (round to
nearest even, through float32).  The workloads follow the paper's acausal,
causal and retrieval settings: clustered queries/keys (the method clusters
queries and keys separately in representation space, pith.science review of
arXiv 2509.10406, "What carries the argument"), unit-variance values.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    D: int
    Dv: int
    dtype: str            # "f32" or "bf16"
    Cq: int
    Ck: int
    iters: int
    components: int
    sigma: float          # within-component standard deviation
    seed: int
    mode: str             # "acausal", "causal", "retrieval"
    block: int = 0        # spatial block size (causal / retrieval)
    k1: int = 0           # clusters retrieved per query cluster
    k2: int = 0           # blocks retrieved per retrieved cluster
    outlier_frac: float = 0.0
    outlier_scale: float = 1.0
    scale: float = 1.0    # logit scale s in exp(s q.k)

    @property
    def problems(self) -> int:
        return self.B * self.H


def _w(**kw) -> Workload:
    return Workload(**kw)


# The five workloads.  Names say what they are; sizes as (B, H, N, D).
WORKLOADS = {
    "acausal_n1k_f32": _w(name="acausal_n1k_f32", B=1, H=1, N=1024, D=64, Dv=64, dtype="f32",
                          Cq=32, Ck=32, iters=10, components=32, sigma=0.3 / math.sqrt(64),
                          seed=0, mode="acausal"),
    "acausal_n8k_bf16": _w(name="acausal_n8k_bf16", B=1, H=8, N=8192, D=64, Dv=64, dtype="bf16",
                           Cq=128, Ck=128, iters=10, components=256, sigma=0.5 / math.sqrt(64),
                           seed=1, mode="acausal"),
    "causal_n16k_bf16": _w(name="causal_n16k_bf16", B=4, H=8, N=16384, D=64, Dv=64, dtype="bf16",
                           Cq=64, Ck=64, iters=10, components=32, sigma=0.3 / math.sqrt(64),
                           seed=2, mode="causal", block=512),
    "retrieval_n32k_bf16": _w(name="retrieval_n32k_bf16", B=2, H=8, N=32768, D=64, Dv=64,
                              dtype="bf16", Cq=128, Ck=128, iters=10, components=512,
                              sigma=0.3 / math.sqrt(64), seed=3, mode="retrieval", block=512,
                              k1=4, k2=4, outlier_frac=0.05, outlier_scale=4.0),
    "acausal_n64k_d128_bf16": _w(name="acausal_n64k_d128_bf16", B=1, H=16, N=65536, D=128,
                                 Dv=128, dtype="bf16", Cq=256, Ck=256, iters=8, components=1024,
                                 sigma=0.4 / math.sqrt(128), seed=4, mode="acausal"),
}

# The order in which the workloads are listed (smallest first).
WORKLOAD_ORDER = ["acausal_n1k_f32", "acausal_n8k_bf16", "causal_n16k_bf16",
                  "retrieval_n32k_bf16", "acausal_n64k_d128_bf16"]


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round float64/float32 values to bfloat16 (RNE through float32), returned as float32."""
    f = np.ascontiguousarray(x, dtype=np.float32)
    bits = f.view(np.uint32).astype(np.uint64)
    lsb = (bits >> 16) & 1
    bits = (bits + 0x7FFF + lsb) & 0xFFFF0000
    return bits.astype(np.uint32).view(np.float32)


def draw_problem(rng: np.random.Generator, N: int, D: int, Dv: int, components: int,
                 sigma: float, outlier_frac: float = 0.0, outlier_scale: float = 1.0):
    """One (batch, head) problem in float64: (Q [N,D], K [N,D], V [N,Dv])."""
    means = rng.standard_normal((components, D)) / math.sqrt(D)
    qi = rng.integers(0, components, size=N)
    Q = means[qi] + sigma * rng.standard_normal((N, D))
    ki = rng.integers(0, components, size=N)
    K = means[ki] + sigma * rng.standard_normal((N, D))
    V = rng.standard_normal((N, Dv))
    if outlier_frac > 0.0:
        n_out = int(round(outlier_frac * N))
        rows = rng.choice(N, size=n_out, replace=False)
        K[rows] *= outlier_scale
    return Q, K, V


def make_inputs(w: Workload, heads: Optional[list] = None):
    """Seeded inputs for workload ``w`` as float32 numpy arrays of shape [B,H,N,D].

    bf16 workloads return the bf16-rounded values held in float32 (exactly
    representable); ``heads`` (a list of flat problem indices b*H+h) restricts the
    returned problems while keeping every problem's draws identical to a full draw.
    """
    rng = np.random.Generator(np.random.PCG64(w.seed))
    P = w.problems
    want = list(range(P)) if heads is None else list(heads)
    Qs, Ks, Vs = {}, {}, {}
    for p in range(P):
        Q, K, V = draw_problem(rng, w.N, w.D, w.Dv, w.components, w.sigma,
                               w.outlier_frac, w.outlier_scale)
        if p in want:
            Qs[p], Ks[p], Vs[p] = Q, K, V
        if p >= max(want):
            break
    cast = round_to_bf16 if w.dtype == "bf16" else (lambda a: a.astype(np.float32))
    Q = np.stack([cast(Qs[p]) for p in want])
    K = np.stack([cast(Ks[p]) for p in want])
    V = np.stack([cast(Vs[p]) for p in want])
    if heads is None:
        shape = (w.B, w.H)
    else:
        shape = (1, len(want))
    return (Q.reshape(*shape, w.N, w.D), K.reshape(*shape, w.N, w.D),
            V.reshape(*shape, w.N, w.Dv))


def small_problem(seed: int, N: int, D: int, Dv: int, components: int, sigma: float,
                  outlier_frac: float = 0.0, outlier_scale: float = 1.0):
    """A single float64 problem for tests (no rounding)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    return draw_problem(rng, N, D, Dv, components, sigma, outlier_frac, outlier_scale)
