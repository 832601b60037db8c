"""Seeded synthetic point-cloud workloads for entropic OT.

This module only draws inputs.  It holds none of the Sinkhorn arithmetic, so
both the CUDA path (through the C-ABI) and the CPU oracle can consume exactly
the same bytes.

The five workloads are the point clouds named for the FlashSinkhorn method
("FlashSinkhorn: IO-aware EOT on GPU", Risultati Sperimentali: synthetic
benchmarks).  The pages state no shapes for their synthetic clouds, so the
shapes below are the fixed benchmark set this library is measured on:

  tiny      n=m=1024,  d=3,   fp32  X,Y ~ N(0,I), Y shifted +1 on axis 0; uniform a,b; eps=0.1; 50 iters
  middim    n=m=16384, d=64,  fp32  X ~ N(0,I/d), Y ~ N(0.5*1, I/d); a,b = softmax(N(0,1)); eps=0.05; 100 iters
  cloud3d   n=70000, m=50000, d=3, fp32  X on the unit sphere + N(0,0.01^2); Y an 8-component
            isotropic Gaussian mixture (sigma 0.1, means U[-1,1]^3, equal weights); uniform; eps=0.01; 200 iters
  highdim   n=m=65536, d=128, bf16  X ~ N(0,I/d); Y = Z R, Z ~ N(0,I/d), R Haar orthogonal; uniform; eps=0.1; 100 iters
  batched   64 x (n=m=4096, d=32), fp32  mu_k ~ N(0,I); X_k,Y_k ~ N(mu_k, I/d); a,b = softmax(N(0,1)); eps=0.05; 50 iters

Everything is drawn in float64 with numpy's PCG64 (``default_rng(seed)``) and
cast once to the workload dtype.  ``X``/``Y`` hold the exact values of the
cast (float64 view) for the oracle; ``X_dev``/``Y_dev`` hold the bytes the GPU
receives (float32, or bfloat16 bit patterns as uint16).
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional

import numpy as np

__all__ = ["WORKLOADS", "Problem", "make_problem", "bf16_round", "workload_names"]


# name -> (batch, n, m, d, dtype, eps, iters, seed)
WORKLOADS = {
    "tiny": dict(batch=1, n=1024, m=1024, d=3, dtype="f32", eps=0.1, iters=50, seed=1001),
    "middim": dict(batch=1, n=16384, m=16384, d=64, dtype="f32", eps=0.05, iters=100, seed=1002),
    "cloud3d": dict(batch=1, n=70000, m=50000, d=3, dtype="f32", eps=0.01, iters=200, seed=1003),
    "highdim": dict(batch=1, n=65536, m=65536, d=128, dtype="bf16", eps=0.1, iters=100, seed=1004),
    "batched": dict(batch=64, n=4096, m=4096, d=32, dtype="f32", eps=0.05, iters=50, seed=1005),
}


def workload_names():
    return list(WORKLOADS.keys())


def bf16_round(x: np.ndarray):
    """Round float64 values to bfloat16 (round to nearest even via float32).

    Returns (bits uint16, exact float64 values of those bfloat16 numbers).
    The double rounding float64 -> float32 -> bfloat16 is the cast that
    ``torch.tensor(x, dtype=float32).to(bfloat16)`` performs; inputs here are
    finite and far from the overflow range.
    """
    f32 = np.ascontiguousarray(x, dtype=np.float32)
    u = f32.view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    r = ((u + np.uint64(0x7FFF) + lsb) >> np.uint64(16)).astype(np.uint16)
    vals = (r.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    return r, vals


@dataclass
class Problem:
    name: str
    batch: int
    n: int
    m: int
    d: int
    dtype: str          # "f32" or "bf16"
    eps: float
    iters: int
    seed: int
    X: np.ndarray       # [batch, n, d] float64, exact values of the device inputs
    Y: np.ndarray       # [batch, m, d] float64
    a: Optional[np.ndarray]  # [batch, n] float64 (exact float32 values) or None = uniform
    b: Optional[np.ndarray]  # [batch, m] float64 or None = uniform
    X_dev: np.ndarray = field(repr=False, default=None)  # float32 or uint16 (bf16 bits)
    Y_dev: np.ndarray = field(repr=False, default=None)
    a_dev: Optional[np.ndarray] = field(repr=False, default=None)  # float32 or None
    b_dev: Optional[np.ndarray] = field(repr=False, default=None)

    def weights(self):
        """(a, b) as float64 arrays, materialising uniform weights as 1/n."""
        a = self.a if self.a is not None else np.full((self.batch, self.n), 1.0 / self.n)
        b = self.b if self.b is not None else np.full((self.batch, self.m), 1.0 / self.m)
        return a, b


def _softmax_weights(rng, batch, n):
    z = rng.standard_normal((batch, n))
    w = np.exp(z - z.max(axis=1, keepdims=True))
    w = w / w.sum(axis=1, keepdims=True)
    w32 = w.astype(np.float32)
    return w32.astype(np.float64), w32


def _haar_orthogonal(rng, d):
    g = rng.standard_normal((d, d))
    q, r = np.linalg.qr(g)
    return q * np.sign(np.diag(r))[None, :]


def make_problem(name: str, n: Optional[int] = None, m: Optional[int] = None,
                 batch: Optional[int] = None, seed: Optional[int] = None,
                 d: Optional[int] = None) -> Problem:
    """Draw workload ``name``; sizes and seed may be overridden (same recipe)."""
    cfg = dict(WORKLOADS[name])
    if n is not None:
        cfg["n"] = n
    if m is not None:
        cfg["m"] = m
    if batch is not None:
        cfg["batch"] = batch
    if seed is not None:
        cfg["seed"] = seed
    if d is not None:
        cfg["d"] = d
    B, n, m, d = cfg["batch"], cfg["n"], cfg["m"], cfg["d"]
    rng = np.random.default_rng(cfg["seed"])
    a = b = None
    a32 = b32 = None

    if name == "tiny":
        X = rng.standard_normal((B, n, d))
        Y = rng.standard_normal((B, m, d))
        Y[..., 0] += 1.0
    elif name == "middim":
        s = 1.0 / np.sqrt(d)
        X = rng.standard_normal((B, n, d)) * s
        Y = 0.5 + rng.standard_normal((B, m, d)) * s
        a, a32 = _softmax_weights(rng, B, n)
        b, b32 = _softmax_weights(rng, B, m)
    elif name == "cloud3d":
        g = rng.standard_normal((B, n, d))
        X = g / np.linalg.norm(g, axis=2, keepdims=True) + 0.01 * rng.standard_normal((B, n, d))
        means = rng.uniform(-1.0, 1.0, size=(B, 8, d))
        comp = rng.integers(0, 8, size=(B, m))
        Y = np.take_along_axis(means, comp[..., None].repeat(d, axis=2), axis=1)
        Y = Y + 0.1 * rng.standard_normal((B, m, d))
    elif name == "highdim":
        s = 1.0 / np.sqrt(d)
        X = rng.standard_normal((B, n, d)) * s
        Z = rng.standard_normal((B, m, d)) * s
        Y = np.empty_like(Z)
        for k in range(B):
            Y[k] = Z[k] @ _haar_orthogonal(rng, d)
    elif name == "batched":
        s = 1.0 / np.sqrt(d)
        mu = rng.standard_normal((B, 1, d))
        X = mu + rng.standard_normal((B, n, d)) * s
        Y = mu + rng.standard_normal((B, m, d)) * s
        a, a32 = _softmax_weights(rng, B, n)
        b, b32 = _softmax_weights(rng, B, m)
    else:
        raise KeyError(name)

    if cfg["dtype"] == "bf16":
        X_dev, X = bf16_round(X)
        Y_dev, Y = bf16_round(Y)
    else:
        X_dev = X.astype(np.float32)
        Y_dev = Y.astype(np.float32)
        X = X_dev.astype(np.float64)
        Y = Y_dev.astype(np.float64)

    return Problem(name=name, batch=B, n=n, m=m, d=d, dtype=cfg["dtype"], eps=cfg["eps"],
                   iters=cfg["iters"], seed=cfg["seed"], X=X, Y=Y, a=a, b=b,
                   X_dev=np.ascontiguousarray(X_dev), Y_dev=np.ascontiguousarray(Y_dev),
                   a_dev=a32, b_dev=b32)
