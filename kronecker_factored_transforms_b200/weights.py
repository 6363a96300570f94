"""Weight side of the W4A4 linear layer (offline preparation).

FlatQuant ("Learning the affine transformation", "Kronecker factorization")
pairs the online activation transform x -> Q(x diag(c)^-1 (P1 (x) P2)) with an
offline weight transform W -> Q((P1 (x) P2)^-1 diag(c) W^T), so that the
product of the two equals x W^T before quantisation.  For one weight row w
(an output channel, length n = n1 n2) the transformed row is

    w' = (w o c) (P1^-T (x) P2^-T),

i.e. the same Kronecker-factored transform as the activation path, with
factors P1^-T and P2^-T and the channel vector c itself in place of 1/c.
Quantising w' per row with the same symmetric INT4 rule gives one scale per
output channel.  So the weight transform runs through ``kq_transform_quant``
unchanged; only its factors are prepared here.

The factor inverses are taken in fp64 through the SVD (the page inverts the
learned P the same way, for numerical stability), once per layer, on the
host: two matrices of at most 128 x 128.  The result is rounded to bf16 for
the kernel.
"""
from __future__ import annotations

import numpy as np

from . import workloads


def svd_inverse(P: np.ndarray) -> np.ndarray:
    """fp64 inverse of a square matrix through its SVD: V diag(1/sigma) U^T."""
    U, sig, Vt = np.linalg.svd(np.asarray(P, dtype=np.float64))
    if sig[-1] <= sig[0] * 1e-12:
        raise ValueError("factor is numerically singular (condition number %.3g)" % (sig[0] / max(sig[-1], 1e-300)))
    return (Vt.T / sig) @ U.T


def weight_factors_bf16(P1_bits: np.ndarray, P2_bits: np.ndarray):
    """bf16 bit patterns of P1^-T and P2^-T, the factors of the weight-side transform.

    The inverses are those of the bf16 factors the activation path uses."""
    P1 = workloads.bf16_bits_to_f32(P1_bits).astype(np.float64)
    P2 = workloads.bf16_bits_to_f32(P2_bits).astype(np.float64)
    F1 = svd_inverse(P1).T
    F2 = svd_inverse(P2).T
    return (workloads.f32_to_bf16_bits(F1.astype(np.float32)),
            workloads.f32_to_bf16_bits(F2.astype(np.float32)))


def weight_transform_quant(W, F1, F2, c, alpha: float, q_out, scale_out, n1: int, n2: int, stream=None) -> None:
    """Transform and quantise weight rows on the GPU: per row w,
    Q((w o c)(F1 (x) F2)) with F1 = P1^-T, F2 = P2^-T from ``weight_factors_bf16``.

    W [N_out, n] bf16, F1 [n1, n1] bf16, F2 [n2, n2] bf16, c [n] fp32 (or None),
    q_out [N_out, n/2] uint8, scale_out [N_out] fp32, all device tensors."""
    from . import _lib
    _lib.kq_transform_quant(W, F1, F2, c, alpha, q_out, scale_out, W.shape[0], n1, n2, stream=stream)
