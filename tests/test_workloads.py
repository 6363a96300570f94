"""The seeded input generator: shapes, reproducibility and the recipe's facts."""
import math

import numpy as np
import pytest
import torch

from kronecker_factored_transforms_b200.workloads import (CONFIGS, SWEEP_T, bf16_bits_to_f32,
                                                          f32_to_bf16_bits, make_workload,
                                                          workload_bytes, workload_flops)


def test_bf16_cast_is_round_to_nearest_even():
    rng = np.random.default_rng(0)
    a = np.concatenate([rng.standard_normal(100000).astype(np.float32) * 1e3,
                        np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -1.0 - 2 ** -8], np.float32)])
    ours = f32_to_bf16_bits(a)
    ref = torch.from_numpy(a).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(ours, ref)
    np.testing.assert_array_equal(bf16_bits_to_f32(ours), torch.from_numpy(a).to(torch.bfloat16).float().numpy())


@pytest.mark.parametrize("name", ["tiny", "llama7b_hidden", "hidden8192", "mlp14336", "mlp14336_cinv",
                                  "hidden5120", "sweep4096", "ffn28672", "square65536"])
def test_shapes_and_reproducibility(name):
    a = make_workload(name, rows=8)
    b = make_workload(name, rows=8)
    cfg = CONFIGS[name]
    assert a.x.shape == (8, cfg["n1"] * cfg["n2"]) and a.x.dtype == np.uint16
    assert a.P1.shape == (cfg["n1"],) * 2 and a.P2.shape == (cfg["n2"],) * 2
    np.testing.assert_array_equal(a.x, b.x)
    np.testing.assert_array_equal(a.P1, b.P1)
    assert (a.cinv is None) == (not cfg["scaled"])
    if cfg["factors"] == "orthogonal":
        for P in (a.P1_f64, a.P2_f64):
            np.testing.assert_allclose(P @ P.T, np.eye(P.shape[0]), atol=1e-12)
    assert 0.0 < a.alpha <= 1.0 and a.alpha == float(np.float32(a.alpha))


def test_row_subset_equals_leading_rows_of_full_workload():
    full = make_workload("hidden8192", T=2500)
    part = make_workload("hidden8192", T=2500, rows=1100)
    np.testing.assert_array_equal(part.x, full.x[:1100])
    np.testing.assert_array_equal(part.cinv, full.cinv)


def test_sweep_shares_factors_and_leading_rows():
    small = make_workload("sweep4096", T=16)
    big = make_workload("sweep4096", T=128)
    np.testing.assert_array_equal(small.P1, big.P1)
    np.testing.assert_array_equal(small.x, big.x[:16])
    assert SWEEP_T == (1, 16, 128, 1024, 16384, 65536)


def test_recipe_facts():
    w = make_workload("llama7b_hidden", rows=64)
    x = bf16_bits_to_f32(w.x).astype(np.float64)
    # token 0 is the pivot token (x100): its absmax dwarfs the others
    assert np.abs(x[0]).max() > 20 * np.median(np.abs(x[1:]).max(axis=1))
    assert w.alpha == pytest.approx(1 / (1 + math.exp(-2.0)), rel=1e-7)
    m = make_workload("mlp14336", rows=16)
    zeros = (m.x == 0).mean()
    assert 0.45 < zeros < 0.55          # ReLU gating: half the entries exactly zero
    h = make_workload("hidden8192", rows=2)
    c = 1.0 / h.cinv.astype(np.float64)
    assert c.min() >= 0.5 - 1e-6 and c.max() <= 2.0 + 1e-6


def test_roofline_unit_counts():
    assert workload_bytes(1, 8192) == 2 * 8192 + 4096 + 4
    assert workload_flops(1, 64, 128) == 2 * 8192 * (64 + 128)
