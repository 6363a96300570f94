"""Pins of the oracle's per-head (key / value cache) transform + INT4."""
import numpy as np
import pytest

from kronecker_factored_transforms_b200.workloads import f32_to_bf16_bits


def _inputs(T, heads, D, seed):
    rng = np.random.default_rng(seed)
    q, r = np.linalg.qr(rng.standard_normal((D, D)))
    Ph = f32_to_bf16_bits((q * np.sign(np.diag(r))).astype(np.float32))
    x = f32_to_bf16_bits(rng.standard_normal((T, heads * D)).astype(np.float32))
    return x, Ph


@pytest.mark.parametrize("heads", [16, 32])
def test_equals_kronecker_path_with_identity_left_factor(oracle_mod, heads):
    """With P1 = I (n1 = heads) the Kronecker transform is the per-head transform;
    the quantiser then differs only in scope (per token there, per head here)."""
    D = 64
    x, Ph = _inputs(6, heads, D, heads)
    I = f32_to_bf16_bits(np.eye(heads, dtype=np.float32))
    y_kron = oracle_mod.transform(x, I, Ph, None, heads, D)
    r = oracle_mod.headwise_transform_quant(x, Ph, 0.9, heads, D)
    q_rows = oracle_mod.quantize(y_kron.reshape(-1, D), 0.9)
    assert np.array_equal(r["codes"].reshape(-1, D), q_rows["codes"])
    assert np.array_equal(r["scale32"].reshape(-1), q_rows["scale32"])


def test_brute_force_small(oracle_mod):
    heads, D = 3, 16
    x, Ph = _inputs(2, heads, D, 5)
    r = oracle_mod.headwise_transform_quant(x, Ph, 0.85, heads, D)
    xf = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    Pf = (Ph.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    for t in range(2):
        for h in range(heads):
            y = [sum(xf[t, h * D + b] * Pf[b, j] for b in range(D)) for j in range(D)]
            s = float(np.float32(0.85)) * max(abs(v) for v in y) / 7.0  # alpha arrives as fp32
            assert abs(r["scale64"][t, h] - s) <= 1e-15 * s
            for j in range(D):
                q = max(-8, min(7, int(np.rint(y[j] / s))))
                assert r["codes"][t, h * D + j] == q


def test_gqa_head_count_and_layout(oracle_mod):
    """8 heads (grouped-query attention keys): rows stay in (token, head) order."""
    heads, D = 8, 128
    x, Ph = _inputs(5, heads, D, 8)
    r = oracle_mod.headwise_transform_quant(x, Ph, 1.0, heads, D)
    assert r["packed"].shape == (5, heads * D // 2) and r["scale32"].shape == (5, heads)
    one = oracle_mod.headwise_transform_quant(x[2:3, 3 * D:4 * D], Ph, 1.0, 1, D)
    assert np.array_equal(one["packed"][0], r["packed"][2, 3 * D // 2:4 * D // 2])
    assert one["scale32"][0, 0] == r["scale32"][2, 3]
