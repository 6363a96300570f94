"""Seeded synthetic inputs for the fused Kronecker transform + INT4 path.

This module only draws random numbers and casts them to bf16. It holds none
of the method's arithmetic (no transform, no quantiser), so both the CUDA
path and the fp64 oracle can take their inputs from here without sharing any
computation.

Workload shapes follow the FlatQuant page ("Kronecker factorization": hidden
size 8192 factors as 64x128; LLaMA-2-7B hidden 4096) plus an FFN size of
14336 (= 112 x 128, the divisor pair minimising n1 + n2). The value
distributions (outlier channels, a pivot token, heavy tails, ReLU gating,
per-channel scaling c) stand in for real LLM activations, which are not used.

Conventions (one reading of the generator recipe, fixed here):
  * numpy ``default_rng(seed)`` (PCG64); draw order P1, P2, outlier channel
    set, c, then x (in chunks of ``CHUNK_ROWS`` rows).
  * shard r > 0 of a multi-GPU run draws its rows of x from
    ``default_rng([seed, r])``; factors, outlier channels and c are shared.
  * bf16 = round-to-nearest-even of the float32 value.
  * orthogonal factor: Q of QR(Gaussian) with columns multiplied by
    sign(diag R), cast to bf16 (so it is only nearly orthogonal).
  * non-orthogonal factor: I + 0.1 * N(0,1) / sqrt(n_i), formed in fp64.
  * "1% of channels": round(0.01 n) distinct channels, drawn without
    replacement, whose columns of x are multiplied by the outlier factor.
  * N(0, 2) means variance 2.  ReLU gating = independent Bernoulli(1/2) mask.
  * c ~ exp(U[ln 0.5, ln 2]); the path is given cinv = float32(1 / c).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np

CHUNK_ROWS = 1024


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns (uint16), round to nearest, ties to even."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    bias = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> float32, exact."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


@dataclasses.dataclass
class Workload:
    """One synthetic problem: T token rows of length n = n1 * n2."""

    name: str
    T: int
    n1: int
    n2: int
    x: np.ndarray            # [T, n] uint16, bf16 bit patterns, row-major
    P1: np.ndarray           # [n1, n1] uint16 bf16 bits, row-major
    P2: np.ndarray           # [n2, n2] uint16 bf16 bits, row-major
    cinv: Optional[np.ndarray]  # [n] float32 (= 1/c) or None (c = 1)
    alpha: float             # float32-representable clip ratio in (0, 1]
    seed: int
    P1_f64: np.ndarray       # the fp64 factor before the bf16 cast
    P2_f64: np.ndarray

    @property
    def n(self) -> int:
        return self.n1 * self.n2

    @property
    def c(self) -> Optional[np.ndarray]:
        """The per-channel scale c as float32 (1 / cinv), or None."""
        if self.cinv is None:
            return None
        return (1.0 / self.cinv.astype(np.float64)).astype(np.float32)


def _orthogonal(rng: np.random.Generator, k: int) -> np.ndarray:
    a = rng.standard_normal((k, k))
    q, r = np.linalg.qr(a)
    return q * np.sign(np.diag(r))[None, :]


def _near_identity(rng: np.random.Generator, k: int) -> np.ndarray:
    return np.eye(k) + 0.1 * rng.standard_normal((k, k)) / math.sqrt(k)


def _outlier_channels(rng: np.random.Generator, n: int, frac: float) -> np.ndarray:
    count = int(round(frac * n))
    return np.sort(rng.choice(n, size=count, replace=False))


def _sigmoid_f32(theta: float) -> float:
    return float(np.float32(1.0 / (1.0 + math.exp(-theta))))


# name -> recipe.  ``T`` may be overridden (the sweep uses several T).
CONFIGS = {
    # T=64, n=256 (16x16); N(0,1), channels {3,77,140,201} x50; orthogonal;
    # c = 1; alpha = 0.9; seed 0.
    "tiny": dict(T=64, n1=16, n2=16, seed=0, alpha=0.9, factors="orthogonal",
                 x_kind="normal", outliers=("fixed", (3, 77, 140, 201), 50.0),
                 pivot=None, scaled=False),
    # T=2048, n=4096 (64x64); N(0,1) + 1% channels x30; token 0 x100;
    # orthogonal; c = 1; alpha = sigmoid(2.0); seed 1.
    "llama7b_hidden": dict(T=2048, n1=64, n2=64, seed=1, alpha=_sigmoid_f32(2.0),
                           factors="orthogonal", x_kind="normal",
                           outliers=("frac", 0.01, 30.0), pivot=100.0, scaled=False),
    # T=8192, n=8192 (64x128); 0.5 * Student-t(3); c ~ logU[0.5, 2];
    # P = I + 0.1 N / sqrt(n_i); alpha = 0.85; seed 2.
    "hidden8192": dict(T=8192, n1=64, n2=128, seed=2, alpha=0.85, factors="near_identity",
                       x_kind="student_t", outliers=None, pivot=None, scaled=True),
    # T=4096, n=14336 (112x128); ReLU-gated N(0,2) + 0.5% channels x40;
    # orthogonal; alpha = 0.9; seed 3.
    "mlp14336": dict(T=4096, n1=112, n2=128, seed=3, alpha=0.9, factors="orthogonal",
                     x_kind="relu_gated", outliers=("frac", 0.005, 40.0), pivot=None,
                     scaled=False),
    # mlp14336 with a per-channel smoothing factor c ~ logU[0.5, 2] (cinv =
    # 1 / c folded into the transform, as in hidden8192); seed 7.
    "mlp14336_cinv": dict(T=4096, n1=112, n2=128, seed=7, alpha=0.9, factors="orthogonal",
                          x_kind="relu_gated", outliers=("frac", 0.005, 40.0), pivot=None,
                          scaled=True),
    # n=5120 (64x80), the hidden size of a 13B-class model: an n2 outside
    # {64, 128}; the hidden8192 recipe otherwise (Student-t, c ~ logU[0.5, 2],
    # near-identity factors, alpha = 0.85); seed 8.
    "hidden5120": dict(T=4096, n1=64, n2=80, seed=8, alpha=0.85, factors="near_identity",
                       x_kind="student_t", outliers=None, pivot=None, scaled=True),
    # n=4096 (64x64) at T in SWEEP_T; N(0,1) + 1% x30; orthogonal;
    # alpha = 0.9; seed 4.
    "sweep4096": dict(T=1024, n1=64, n2=64, seed=4, alpha=0.9, factors="orthogonal",
                      x_kind="normal", outliers=("frac", 0.01, 30.0), pivot=None,
                      scaled=False),
    # Factors above 128 (the two-stage path).  n=28672 (112x256), the FFN width
    # of a 70B-class model; the mlp14336 recipe otherwise; seed 5.
    "ffn28672": dict(T=2048, n1=112, n2=256, seed=5, alpha=0.9, factors="orthogonal",
                     x_kind="relu_gated", outliers=("frac", 0.005, 40.0), pivot=None,
                     scaled=False),
    # n=65536 (256x256), both factors above 128; the hidden8192 recipe
    # otherwise (Student-t, c ~ logU[0.5, 2], near-identity factors); seed 6.
    "square65536": dict(T=1024, n1=256, n2=256, seed=6, alpha=0.85, factors="near_identity",
                        x_kind="student_t", outliers=None, pivot=None, scaled=True),
}

SWEEP_T = (1, 16, 128, 1024, 16384, 65536)


def make_workload(name: str, T: Optional[int] = None, rows: Optional[int] = None,
                  shard: int = 0) -> Workload:
    """Build config ``name`` (see ``CONFIGS``) with its seed.

    ``T`` overrides the token count (the same seed gives the same factors and
    the same leading rows of x for every T).  ``rows`` generates only the
    first ``rows`` tokens of a T-token workload (identical to the leading
    rows of the full one): a cheap way to sample a large configuration.
    ``shard`` selects an independent block of rows with the same factors,
    outlier channels and c (one block per rank in a multi-GPU run).
    """
    cfg = CONFIGS[name]
    T = int(cfg["T"] if T is None else T)
    n1, n2 = cfg["n1"], cfg["n2"]
    n = n1 * n2
    rows_out = T if rows is None else min(int(rows), T)
    rng = np.random.default_rng(cfg["seed"])

    make_factor = _orthogonal if cfg["factors"] == "orthogonal" else _near_identity
    P1 = make_factor(rng, n1)
    P2 = make_factor(rng, n2)

    out = cfg["outliers"]
    if out is None:
        chan, factor = np.zeros(0, dtype=np.int64), 1.0
    elif out[0] == "fixed":
        chan, factor = np.asarray(out[1], dtype=np.int64), float(out[2])
    else:
        chan, factor = _outlier_channels(rng, n, float(out[1])), float(out[2])

    cinv = None
    if cfg["scaled"]:
        c = np.exp(rng.uniform(math.log(0.5), math.log(2.0), size=n))
        cinv = (1.0 / c).astype(np.float32)

    xrng = rng if shard == 0 else np.random.default_rng([cfg["seed"], int(shard)])
    x_bits = np.empty((rows_out, n), dtype=np.uint16)
    done = 0
    while done < rows_out:
        r = min(CHUNK_ROWS, T - done)
        kind = cfg["x_kind"]
        if kind == "normal":
            blk = xrng.standard_normal((r, n))
        elif kind == "student_t":
            blk = 0.5 * xrng.standard_t(3, size=(r, n))
        elif kind == "relu_gated":
            g = xrng.standard_normal((r, n)) * math.sqrt(2.0)
            mask = xrng.random((r, n)) < 0.5
            blk = np.where(mask, g, 0.0)
        else:  # pragma: no cover - recipe table is closed
            raise ValueError(kind)
        if chan.size:
            blk[:, chan] *= factor
        if cfg["pivot"] is not None and done == 0 and shard == 0:
            blk[0, :] *= cfg["pivot"]
        take = min(r, rows_out - done)
        x_bits[done:done + take] = f32_to_bf16_bits(blk[:take].astype(np.float32))
        done += r

    return Workload(name=name, T=T, n1=n1, n2=n2, x=x_bits,
                    P1=f32_to_bf16_bits(P1.astype(np.float32)),
                    P2=f32_to_bf16_bits(P2.astype(np.float32)),
                    cinv=cinv, alpha=float(np.float32(cfg["alpha"])), seed=cfg["seed"],
                    P1_f64=P1, P2_f64=P2)


def workload_bytes(T: int, n: int) -> int:
    """Algorithmic HBM bytes of one pass: x in (2n), codes out (n/2), scale (4)."""
    return T * (2 * n + n // 2 + 4)


def workload_flops(T: int, n1: int, n2: int) -> int:
    """Algorithmic flops of the factored contraction: 2 n (n1 + n2) per token."""
    return T * 2 * n1 * n2 * (n1 + n2)


def make_weights(n: int, n_out: int, seed: int) -> np.ndarray:
    """Synthetic linear-layer weight W [n_out, n] as bf16 bits: N(0, 1/n) entries
    with 1% of the input channels (columns) scaled by 8, the way trained
    weights carry a few large input channels.  Seeded; no method arithmetic."""
    rng = np.random.default_rng([seed, 7919])
    W = rng.standard_normal((n_out, n)) / np.sqrt(n)
    cols = rng.choice(n, size=max(1, round(0.01 * n)), replace=False)
    W[:, cols] *= 8.0
    return f32_to_bf16_bits(W.astype(np.float32))
