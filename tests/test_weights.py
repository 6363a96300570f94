"""Weight side of the W4A4 layer, checked on the CPU with the oracle.

FlatQuant ("Learning the affine transformation", "Kronecker factorization"):
x W^T = (x diag(c)^-1 P)(P^-1 diag(c) W^T) with P = P1 (x) P2.  Per weight row
w the transformed row is (w o c)(P1^-T (x) P2^-T), the activation transform
with factors P1^-T, P2^-T and c in place of 1/c.  These tests pin that
convention (a wrong transpose or a wrong direction of c fails by a wide margin)
and the size of the W4A4 product error against the high-rate model.
"""
import numpy as np
import pytest

from kronecker_factored_transforms_b200 import weights as kw
from kronecker_factored_transforms_b200.workloads import bf16_bits_to_f32, f32_to_bf16_bits, make_weights


def test_svd_inverse_is_an_inverse():
    rng = np.random.default_rng(5)
    for k in (16, 64, 128):
        P = np.eye(k) + 0.1 * rng.standard_normal((k, k)) / np.sqrt(k)
        Pi = kw.svd_inverse(P)
        assert np.abs(Pi @ P - np.eye(k)).max() < 1e-12
        assert np.abs(P @ Pi - np.eye(k)).max() < 1e-12


def test_svd_inverse_rejects_singular():
    P = np.ones((16, 16))
    with pytest.raises(ValueError):
        kw.svd_inverse(P)


def _layer(oracle_mod, n1, n2, T, n_out, seed, orthogonal):
    rng = np.random.default_rng(seed)
    if orthogonal:
        def fac(k):
            q, r = np.linalg.qr(rng.standard_normal((k, k)))
            return q * np.sign(np.diag(r))
    else:
        def fac(k):
            return np.eye(k) + 0.1 * rng.standard_normal((k, k)) / np.sqrt(k)
    P1 = f32_to_bf16_bits(fac(n1).astype(np.float32))
    P2 = f32_to_bf16_bits(fac(n2).astype(np.float32))
    n = n1 * n2
    c = np.exp(rng.uniform(np.log(0.5), np.log(2.0), n)).astype(np.float32)
    x = f32_to_bf16_bits(rng.standard_normal((T, n)).astype(np.float32))
    W = make_weights(n, n_out, seed)
    return x, W, P1, P2, c


@pytest.mark.parametrize("n1,n2", [(16, 16), (16, 32)])
def test_weight_factor_convention(oracle_mod, n1, n2):
    """Transforms of x (factors P, 1/c) and of W (factors P^-T, c) multiply to x W^T,
    up to the bf16 rounding of the inverse factors; the wrong conventions do not."""
    x, W, P1, P2, c = _layer(oracle_mod, n1, n2, 32, 48, 11, orthogonal=False)
    cinv = (1.0 / c.astype(np.float64)).astype(np.float32)
    F1, F2 = kw.weight_factors_bf16(P1, P2)
    xf = bf16_bits_to_f32(x).astype(np.float64)
    Wf = bf16_bits_to_f32(W).astype(np.float64)
    # x (1/c), rounded to fp32 the way the path receives it, times c, is x to ~1e-7
    ref = xf @ Wf.T
    yx = oracle_mod.transform(x, P1, P2, cinv, n1, n2)
    yw = oracle_mod.transform(W, F1, F2, c, n1, n2)
    rel = np.linalg.norm(yx @ yw.T - ref) / np.linalg.norm(ref)
    assert rel < 1e-2, rel
    # a missing transpose on the weight factors, or 1/c on the weight side, is far off
    Pi1 = f32_to_bf16_bits(kw.svd_inverse(bf16_bits_to_f32(P1).astype(np.float64)).astype(np.float32))
    Pi2 = f32_to_bf16_bits(kw.svd_inverse(bf16_bits_to_f32(P2).astype(np.float64)).astype(np.float32))
    wrong_t = oracle_mod.transform(W, Pi1, Pi2, c, n1, n2)
    wrong_c = oracle_mod.transform(W, F1, F2, cinv, n1, n2)
    for bad in (wrong_t, wrong_c):
        assert np.linalg.norm(yx @ bad.T - ref) / np.linalg.norm(ref) > 0.2


def test_w4a4_product_error_matches_high_rate_model(oracle_mod):
    """Quantise both sides (per-row INT4, alpha = 1).  With the quantisation noise
    white and of variance s^2 / 12 per element (uniform noise of width s, the
    high-rate model), E|dX Yw^T|^2 = sum_t s_t^2 / 12 * sum_o |yw_o|^2, likewise for
    the weight side; their sum over |x W^T|^2 predicts the measured relative
    squared error of the product within 10%."""
    n1, n2 = 32, 32
    x, W, P1, P2, c = _layer(oracle_mod, n1, n2, 256, 256, 3, orthogonal=True)
    cinv = (1.0 / c.astype(np.float64)).astype(np.float32)
    F1, F2 = kw.weight_factors_bf16(P1, P2)
    rx = oracle_mod.transform_quant(x, P1, P2, cinv, 1.0, n1, n2)
    rw = oracle_mod.transform_quant(W, F1, F2, c, 1.0, n1, n2)
    xh = rx["codes"].astype(np.float64) * rx["scale64"][:, None]
    wh = rw["codes"].astype(np.float64) * rw["scale64"][:, None]
    yx = oracle_mod.transform(x, P1, P2, cinv, n1, n2)
    yw = oracle_mod.transform(W, F1, F2, c, n1, n2)
    exact = yx @ yw.T
    err = np.linalg.norm(xh @ wh.T - exact) ** 2
    pred = (np.sum(rx["scale64"] ** 2 / 12.0) * np.sum(yw ** 2) +
            np.sum(rw["scale64"] ** 2 / 12.0) * np.sum(yx ** 2))
    assert 0.9 * pred < err < 1.1 * pred, (err / np.linalg.norm(exact) ** 2, pred / np.linalg.norm(exact) ** 2)


def test_weights_generator_is_seeded():
    a = make_weights(256, 8, 1)
    b = make_weights(256, 8, 1)
    assert np.array_equal(a, b) and not np.array_equal(a, make_weights(256, 8, 2))
    assert a.dtype == np.uint16 and a.shape == (8, 256)
