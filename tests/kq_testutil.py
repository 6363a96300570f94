"""Helpers shared by the tests: explicit Kronecker matrices and the parity rules.

Nothing here calls the CUDA path or the oracle; these are the independent
yardsticks the oracle is pinned against, and the comparison rules used when
the CUDA path is compared with the oracle.
"""
from __future__ import annotations

import numpy as np


def kron_by_definition(A: np.ndarray, B: np.ndarray) -> np.ndarray:
    """Entrywise Kronecker product (Kronecker Product page, 'Definition'):
    entry ((i-1)p + k, (j-1)q + l) is a_ij * b_kl (1-based); 0-based below."""
    m, n = A.shape
    p, q = B.shape
    K = np.empty((m * p, n * q), dtype=np.float64)
    for i in range(m):
        for j in range(n):
            for k in range(p):
                for l in range(q):
                    K[i * p + k, j * q + l] = A[i, j] * B[k, l]
    return K


def hadamard(k: int) -> np.ndarray:
    """Sylvester Hadamard matrix of order k (k a power of two), entries +-1."""
    H = np.ones((1, 1))
    while H.shape[0] < k:
        H = np.block([[H, H], [H, -H]])
    assert H.shape[0] == k
    return H


def parity_codes(codes_gpu: np.ndarray, codes_ref: np.ndarray, dist_ref: np.ndarray,
                 window: float = 1e-3, max_frac: float = 1e-3):
    """INT4 code parity: bit-exact except +-1 where the oracle's y/s lies within
    ``window`` of a rounding boundary; such mismatches at most ``max_frac`` of codes.
    Returns (ok, n_mismatch, n_bad, message)."""
    cg = codes_gpu.astype(np.int16)
    cr = codes_ref.astype(np.int16)
    diff = cg - cr
    mism = diff != 0
    n_m = int(mism.sum())
    allowed = mism & (np.abs(diff) == 1) & (dist_ref < window)
    bad = mism & ~allowed
    n_bad = int(bad.sum())
    frac = n_m / max(1, cg.size)
    ok = n_bad == 0 and frac <= max_frac
    msg = "mismatches=%d (%.2e of %d) outside-window=%d" % (n_m, frac, cg.size, n_bad)
    if n_bad:
        idx = np.argwhere(bad)[:5]
        msg += " first bad at %s: gpu=%s ref=%s dist=%s" % (
            idx.tolist(), cg[tuple(idx.T)].tolist(), cr[tuple(idx.T)].tolist(),
            dist_ref[tuple(idx.T)].tolist())
    return ok, n_m, n_bad, msg


def token_rel_err(y_gpu: np.ndarray, y_ref: np.ndarray) -> np.ndarray:
    """Per token: max_k |y_gpu - y_ref| / max_k |y_ref| (0 where the token is all zero)."""
    num = np.abs(y_gpu.astype(np.float64) - y_ref).max(axis=1)
    den = np.abs(y_ref).max(axis=1)
    out = np.zeros_like(num)
    nz = den > 0
    out[nz] = num[nz] / den[nz]
    out[~nz] = num[~nz]
    return out


def scale_rel_err(s_gpu: np.ndarray, s_ref: np.ndarray) -> float:
    s_gpu = s_gpu.astype(np.float64)
    s_ref = s_ref.astype(np.float64)
    den = np.where(s_ref > 0, s_ref, 1.0)
    return float(np.max(np.abs(s_gpu - s_ref) / den)) if s_ref.size else 0.0
