"""Pins of the fp64 oracle against things other than itself.

Each test checks the oracle against a fact the pages or the mathematics fix:
hand-derived worked examples (tests/golden), the explicit Kronecker matrix
built from its definition, exact orthogonality, special factors with closed
forms, quantiser invariants and high-rate statistics.  A plausible mistake in
the oracle (a dropped transpose, swapped factors, a wrong vec convention, the
scale applied after the transform, round-half-up instead of half-even, an
off-by-one clamp, a swapped nibble order) fails at least one of them.
"""
import glob
import json
import math
import os

import numpy as np
import pytest

from kq_testutil import hadamard, kron_by_definition
from kronecker_factored_transforms_b200.workloads import (bf16_bits_to_f32, f32_to_bf16_bits,
                                                          make_workload)

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def bf16(a):
    return f32_to_bf16_bits(np.asarray(a, dtype=np.float32))


def widen(bits):
    return bf16_bits_to_f32(bits).astype(np.float64)


def rand_bf16(rng, shape, scale=1.0):
    return bf16(rng.standard_normal(shape) * scale)


# --------------------------------------------------------------------------
# Golden worked examples (values derived by hand in the fixture files).

def _golden_files():
    return sorted(glob.glob(os.path.join(GOLDEN, "*.json")))


@pytest.mark.parametrize("path", _golden_files(), ids=lambda p: os.path.basename(p))
def test_golden_fixture(oracle_mod, path):
    g = json.load(open(path))
    n1, n2 = g["n1"], g["n2"]
    x = bf16(np.array(g["x"], dtype=np.float32))[None, :]
    P1, P2 = bf16(np.array(g["P1"])), bf16(np.array(g["P2"]))
    # The fixture values must be exact in bf16 (otherwise the derivation is moot).
    assert np.array_equal(widen(x)[0], np.array(g["x"], dtype=np.float64))
    assert np.array_equal(widen(P1), np.array(g["P1"], dtype=np.float64))
    cinv = None if g["cinv"] is None else np.array(g["cinv"], dtype=np.float32)
    cases = g.get("cases") or [dict(alpha=g["alpha"], codes=g["codes"], packed=g["packed"],
                                    scale_num=g["scale_num"], scale_den=g["scale_den"])]
    if "y" in g:
        y = oracle_mod.transform(x, P1, P2, cinv, n1, n2)
        np.testing.assert_allclose(y[0], np.array(g["y"], dtype=np.float64), rtol=0, atol=1e-12)
    for case in cases:
        r = oracle_mod.transform_quant(x, P1, P2, cinv, case["alpha"], n1, n2)
        assert r["codes"][0].tolist() == case["codes"]
        assert r["packed"][0].tolist() == case["packed"]
        s = case["scale_num"] / case["scale_den"]
        assert r["scale64"][0] == pytest.approx(s, rel=1e-15)
        assert r["scale32"][0] == np.float32(s)
        assert oracle_mod.unpack_codes(r["packed"])[0].tolist() == case["codes"]
        if "dist" in case:
            # distances to the nearest rounding boundary, in units of y/s: exact binary
            # fractions in these fixtures, so they must match exactly
            assert r["dist"][0].tolist() == case["dist"]
            q = oracle_mod.quantize(oracle_mod.transform(x, P1, P2, cinv, n1, n2), case["alpha"])
            assert q["dist"][0].tolist() == case["dist"]


def test_zero_token_gives_zero_scale_and_codes(oracle_mod):
    x = np.zeros((3, 16 * 16), dtype=np.uint16)
    x[1] = bf16(np.linspace(-1, 1, 256))
    rng = np.random.default_rng(5)
    P1, P2 = rand_bf16(rng, (16, 16)), rand_bf16(rng, (16, 16))
    r = oracle_mod.transform_quant(x, P1, P2, None, 0.9, 16, 16)
    for t in (0, 2):
        assert r["scale32"][t] == 0.0
        assert not r["codes"][t].any() and not r["packed"][t].any()
    assert r["scale32"][1] > 0


# --------------------------------------------------------------------------
# Explicit Kronecker matrix (brute force) and the vec identity.

def test_kron_definition_matches_block_form():
    # 2x2 (x) 2x3 gives a 4x6 block matrix [[a11 B, a12 B], [a21 B, a22 B]].
    A = np.array([[1.0, 2.0], [3.0, 4.0]])
    B = np.array([[1.0, -1.0, 2.0], [0.5, 3.0, -2.0]])
    K = kron_by_definition(A, B)
    assert K.shape == (4, 6)
    blocks = np.block([[A[0, 0] * B, A[0, 1] * B], [A[1, 0] * B, A[1, 1] * B]])
    np.testing.assert_array_equal(K, blocks)
    np.testing.assert_array_equal(K, np.kron(A, B))


@pytest.mark.parametrize("n1,n2,scaled", [(2, 3, False), (3, 2, True), (4, 8, False), (8, 4, True),
                                          (16, 16, False), (16, 16, True), (2, 16, True)])
def test_transform_equals_x_times_explicit_kron(oracle_mod, n1, n2, scaled):
    """y = x' (P1 (x) P2) with the explicit n x n matrix, non-symmetric factors, n1 != n2."""
    rng = np.random.default_rng(100 + n1 * 31 + n2)
    T = 5
    x = rand_bf16(rng, (T, n1 * n2), 2.0)
    P1, P2 = rand_bf16(rng, (n1, n1)), rand_bf16(rng, (n2, n2))
    cinv = rng.uniform(0.5, 2.0, size=n1 * n2).astype(np.float32) if scaled else None
    y = oracle_mod.transform(x, P1, P2, cinv, n1, n2)
    xs = widen(x) * (1.0 if cinv is None else cinv.astype(np.float64))
    K = kron_by_definition(widen(P1), widen(P2))
    ref = xs @ K
    np.testing.assert_allclose(y, ref, rtol=0, atol=1e-12 * np.abs(ref).max())
    # The swapped orders are genuinely different here (guards the test itself).
    assert np.abs(xs @ np.kron(widen(P2), widen(P1)) - ref).max() > 1e-3 * np.abs(ref).max()


def test_transform_spot_check_4096_against_explicit_kron(oracle_mod):
    """One 64x64 case: the 4096 x 4096 matrix P1 (x) P2 formed explicitly."""
    w = make_workload("llama7b_hidden", rows=3)
    K = np.kron(widen(w.P1), widen(w.P2))
    y = oracle_mod.transform(w.x, w.P1, w.P2, None, 64, 64)
    ref = widen(w.x) @ K
    np.testing.assert_allclose(y, ref, rtol=0, atol=1e-11 * np.abs(ref).max())


# --------------------------------------------------------------------------
# Orthogonal, permutation, diagonal and Hadamard factors.

@pytest.mark.parametrize("n1,n2", [(4, 16), (16, 64), (64, 64)])
def test_norm_preserved_by_exact_orthogonal_hadamard_factors(oracle_mod, n1, n2):
    """H_k / sqrt(k) with k = 4^m has entries +-2^-m: exact in bf16 and exactly
    orthogonal, so ||y||_2 = ||x'||_2 (rotations preserve norm)."""
    H1 = hadamard(n1) / math.sqrt(n1)
    H2 = hadamard(n2) / math.sqrt(n2)
    P1, P2 = bf16(H1), bf16(H2)
    assert np.array_equal(widen(P1), H1) and np.array_equal(widen(P2), H2)
    rng = np.random.default_rng(7)
    x = rand_bf16(rng, (6, n1 * n2), 3.0)
    cinv = rng.uniform(0.5, 2.0, size=n1 * n2).astype(np.float32)
    y = oracle_mod.transform(x, P1, P2, cinv, n1, n2)
    xs = widen(x) * cinv.astype(np.float64)
    np.testing.assert_allclose(np.linalg.norm(y, axis=1), np.linalg.norm(xs, axis=1), rtol=1e-12)
    # Orthogonal inverse is the transpose: x' = y (P1 (x) P2)^T.
    np.testing.assert_allclose(y @ np.kron(H1, H2).T, xs, rtol=0, atol=1e-12 * np.abs(xs).max())


def test_onehot_rows_of_hadamard_product(oracle_mod):
    """x = e_k gives row k of P1 (x) P2, i.e. P1[a, :] (x) P2[b, :] with k = a n2 + b."""
    n1, n2 = 4, 16
    H1, H2 = hadamard(n1) / 2.0, hadamard(n2) / 4.0
    x = np.zeros((n1 * n2, n1 * n2), dtype=np.float32)
    np.fill_diagonal(x, 1.0)
    y = oracle_mod.transform(bf16(x), bf16(H1), bf16(H2), None, n1, n2)
    for k in range(n1 * n2):
        a, b = divmod(k, n2)
        np.testing.assert_array_equal(y[k], np.outer(H1[a], H2[b]).ravel())


def test_permutation_factors_permute_x(oracle_mod):
    rng = np.random.default_rng(11)
    n1, n2 = 8, 16
    p1, p2 = rng.permutation(n1), rng.permutation(n2)
    P1 = np.zeros((n1, n1)); P1[p1, np.arange(n1)] = 1.0   # P1[p1[i], i] = 1
    P2 = np.zeros((n2, n2)); P2[p2, np.arange(n2)] = 1.0
    x = rand_bf16(rng, (4, n1 * n2))
    y = oracle_mod.transform(x, bf16(P1), bf16(P2), None, n1, n2)
    X = widen(x).reshape(4, n1, n2)
    # Y~[i][j] = sum_a P1[a][i] sum_b X~[a][b] P2[b][j] = X~[p1[i]][p2[j]].
    np.testing.assert_array_equal(y.reshape(4, n1, n2), X[:, p1][:, :, p2])


def test_diagonal_factors_scale_elementwise(oracle_mod):
    rng = np.random.default_rng(12)
    n1, n2 = 16, 8
    d1, d2 = widen(rand_bf16(rng, n1)), widen(rand_bf16(rng, n2))
    x = rand_bf16(rng, (3, n1 * n2))
    y = oracle_mod.transform(x, bf16(np.diag(d1)), bf16(np.diag(d2)), None, n1, n2)
    np.testing.assert_allclose(y, widen(x) * np.outer(d1, d2).ravel()[None, :], rtol=1e-15, atol=0)


# --------------------------------------------------------------------------
# Inverse and round trip.

@pytest.mark.parametrize("orth", [True, False])
def test_round_trip_through_inverse(oracle_mod, orth):
    """transform then (P1 (x) P2)^-1 = P1^-1 (x) P2^-1 recovers x' (no quantisation)."""
    rng = np.random.default_rng(13)
    n1, n2 = 8, 16
    if orth:
        Q1, _ = np.linalg.qr(rng.standard_normal((n1, n1)))
        Q2, _ = np.linalg.qr(rng.standard_normal((n2, n2)))
    else:
        Q1 = np.eye(n1) + 0.1 * rng.standard_normal((n1, n1)) / math.sqrt(n1)
        Q2 = np.eye(n2) + 0.1 * rng.standard_normal((n2, n2)) / math.sqrt(n2)
    P1, P2 = bf16(Q1), bf16(Q2)
    A1, A2 = widen(P1), widen(P2)
    assert np.linalg.cond(np.kron(A1, A2)) < 10
    x = rand_bf16(rng, (5, n1 * n2))
    cinv = rng.uniform(0.5, 2.0, size=n1 * n2).astype(np.float32)
    y = oracle_mod.transform(x, P1, P2, cinv, n1, n2)
    back = y @ np.kron(np.linalg.inv(A1), np.linalg.inv(A2))
    xs = widen(x) * cinv.astype(np.float64)
    np.testing.assert_allclose(back, xs, rtol=0, atol=1e-10 * np.abs(xs).max())


def test_dequant_inverse_matches_explicit_inverse_kron(oracle_mod):
    rng = np.random.default_rng(14)
    n1, n2 = 4, 8
    A1 = np.eye(n1) + 0.2 * rng.standard_normal((n1, n1))
    A2 = np.eye(n2) + 0.2 * rng.standard_normal((n2, n2))
    I1, I2 = np.linalg.inv(A1), np.linalg.inv(A2)
    T = 6
    packed = rng.integers(0, 256, size=(T, n1 * n2 // 2), dtype=np.uint8)
    scale = rng.uniform(0.1, 2.0, size=T).astype(np.float32)
    c = rng.uniform(0.5, 2.0, size=n1 * n2)
    xhat = oracle_mod.dequant_inverse(packed, scale, I1, I2, c, n1, n2)
    codes = oracle_mod.unpack_codes(packed).astype(np.float64)
    ref = (codes * scale.astype(np.float64)[:, None]) @ np.kron(I1, I2) * c[None, :]
    np.testing.assert_allclose(xhat, ref, rtol=0, atol=1e-12 * np.abs(ref).max())


def test_quantise_then_inverse_error_within_half_step(oracle_mod):
    """alpha = 1 never clips, so |y^ - y| <= s/2 and |x^ - x| <= (s/2) * colsum|P^-1| * c."""
    w = make_workload("hidden8192", rows=4)
    r = oracle_mod.transform_quant(w.x, w.P1, w.P2, w.cinv, 1.0, 64, 128)
    A1, A2 = widen(w.P1), widen(w.P2)
    I1, I2 = np.linalg.inv(A1), np.linalg.inv(A2)
    c = 1.0 / w.cinv.astype(np.float64)
    xhat = oracle_mod.dequant_inverse(r["packed"], r["scale32"], I1, I2, c, 64, 128)
    x = widen(w.x)
    colsum = (np.abs(I1).sum(0)[:, None] * np.abs(I2).sum(0)[None, :]).ravel()
    bound = 0.5 * r["scale32"].astype(np.float64)[:, None] * 1.0001 * colsum[None, :] * c[None, :]
    # the fp32 scale differs from the fp64 one by < 1e-7 relative; slack covers it
    assert np.all(np.abs(xhat - x) <= bound + 1e-6 * np.abs(x).max())


# --------------------------------------------------------------------------
# Quantiser invariants and statistics.

@pytest.mark.parametrize("alpha", [1.0, 0.9, 0.85, float(np.float32(1 / (1 + math.exp(-2.0)))), 0.3])
def test_quantiser_invariants(oracle_mod, alpha):
    rng = np.random.default_rng(15)
    y = rng.standard_t(3, size=(200, 256))
    y[3] = 0.0
    r = oracle_mod.quantize(y, alpha)
    codes, s = r["codes"].astype(np.int64), r["scale64"]
    assert codes.min() >= -8 and codes.max() <= 7
    m = np.abs(y).max(axis=1)
    np.testing.assert_allclose(s, np.float64(np.float32(alpha)) * m / 7.0, rtol=1e-15)
    nz = s > 0
    ratio = y[nz] / s[nz, None]
    inside = (ratio > -8.5) & (ratio < 7.5)
    err = np.abs(codes[nz] * s[nz, None] - y[nz])
    assert np.all(err[inside] <= 0.5 * np.broadcast_to(s[nz, None], err.shape)[inside] * (1 + 1e-12))
    # Outside the representable range the code saturates.
    assert np.all(codes[nz][ratio >= 7.5] == 7) and np.all(codes[nz][ratio <= -8.5] == -8)
    # The absmax element maps to +-7/alpha, rounded and clamped.
    k = np.abs(y).argmax(axis=1)
    top = codes[np.arange(len(k)), k][nz]
    expect = np.clip(np.rint(np.sign(y[np.arange(len(k)), k][nz]) * 7.0 / np.float32(alpha)), -8, 7)
    np.testing.assert_array_equal(top, expect)
    d = r["dist"]
    assert d.min() >= 0 and d.max() <= 0.5
    np.testing.assert_array_equal(oracle_mod.unpack_codes(r["packed"]), r["codes"])


def test_rounding_is_half_to_even_not_half_up(oracle_mod):
    y = np.array([[7.0, 0.5, 1.5, 2.5, -0.5, -1.5, -2.5, 6.5]])
    r = oracle_mod.quantize(y, 1.0)
    assert r["codes"][0].tolist() == [7, 0, 2, 2, 0, -2, -2, 6]


def test_high_rate_statistics_after_rotation(oracle_mod):
    """FlatQuant-style rotation of Gaussian rows: max^2 / mean-square is about
    2 ln n (high-rate INT analysis: the distortion factor concentrates near
    2 ln n after rotation) and the unclipped error variance is about s^2 / 12
    (additive uniform noise model)."""
    w = make_workload("sweep4096", T=256)
    y = oracle_mod.transform(w.x[:, :], w.P1, w.P2, None, 64, 64)
    # drop the outlier channels' influence by using the rotated output itself
    ratio = (np.abs(y).max(1) ** 2 / np.mean(y * y, 1)).mean()
    assert abs(ratio / (2 * math.log(4096)) - 1) < 0.2
    rng = np.random.default_rng(16)
    g = rng.standard_normal((256, 4096))
    r = oracle_mod.quantize(g, 1.0)
    mse = np.mean((r["codes"] * r["scale64"][:, None] - g) ** 2, axis=1)
    np.testing.assert_allclose((mse / (r["scale64"] ** 2 / 12.0)).mean(), 1.0, rtol=0.1)


# --------------------------------------------------------------------------
# Composition, determinism, threads.

def test_fused_oracle_equals_quantise_of_transform(oracle_mod):
    w = make_workload("mlp14336", rows=5)
    y = oracle_mod.transform(w.x, w.P1, w.P2, w.cinv, 112, 128)
    a = oracle_mod.quantize(y, w.alpha)
    b = oracle_mod.transform_quant(w.x, w.P1, w.P2, w.cinv, w.alpha, 112, 128)
    for k in ("codes", "packed", "scale32", "scale64", "dist"):
        np.testing.assert_array_equal(a[k], b[k])


def test_thread_count_does_not_change_results(oracle_mod):
    w = make_workload("tiny")
    a = oracle_mod.transform_quant(w.x, w.P1, w.P2, None, w.alpha, 16, 16, nthreads=1)
    b = oracle_mod.transform_quant(w.x, w.P1, w.P2, None, w.alpha, 16, 16, nthreads=7)
    for k in ("codes", "packed", "scale32", "dist"):
        np.testing.assert_array_equal(a[k], b[k])


def test_empty_input_is_a_no_op(oracle_mod):
    x = np.zeros((0, 256), dtype=np.uint16)
    P = bf16(np.eye(16))
    r = oracle_mod.transform_quant(x, P, P, None, 0.9, 16, 16)
    assert r["packed"].shape == (0, 128) and r["scale32"].shape == (0,)
