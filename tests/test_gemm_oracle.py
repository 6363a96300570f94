"""Pins of the oracle's W4A4 product (the consumer of the packed codes)."""
import numpy as np


def _pack(codes: np.ndarray) -> np.ndarray:
    """Pack int codes in [-8, 7], element 2k in the low nibble (written here
    independently of the oracle's unpacking)."""
    c = (codes.astype(np.int64) & 0xF).astype(np.uint8)
    return (c[..., 0::2] | (c[..., 1::2] << 4)).astype(np.uint8)


def test_brute_force_small(oracle_mod):
    rng = np.random.default_rng(12)
    M, N, K = 5, 7, 32
    qx = rng.integers(-8, 8, (M, K))
    qw = rng.integers(-8, 8, (N, K))
    sx = rng.uniform(0.01, 2, M).astype(np.float32)
    sw = rng.uniform(0.01, 2, N).astype(np.float32)
    y = oracle_mod.w4a4_gemm(_pack(qx), sx, _pack(qw), sw)
    for m in range(M):
        for o in range(N):
            acc = 0
            for k in range(K):
                acc += int(qx[m, k]) * int(qw[o, k])
            assert y[m, o] == acc * float(sx[m]) * float(sw[o])


def test_extreme_codes():
    """-8 against 7 everywhere: the sum is -56 K; -8 against -8: 64 K."""
    import oracle
    K = 256
    a = _pack(np.full((2, K), -8))
    b = _pack(np.stack([np.full(K, 7), np.full(K, -8)]))
    y = oracle.w4a4_gemm(a, np.ones(2, np.float32), b, np.array([1.0, 0.5], np.float32))
    assert np.array_equal(y, np.array([[-56 * K, 0.5 * 64 * K]] * 2, dtype=np.float64))


def test_scales_apply_per_row_and_column(oracle_mod):
    rng = np.random.default_rng(3)
    qx = rng.integers(-8, 8, (4, 64))
    qw = rng.integers(-8, 8, (3, 64))
    base = oracle_mod.w4a4_gemm(_pack(qx), np.ones(4, np.float32), _pack(qw), np.ones(3, np.float32))
    sx = np.array([1, 2, 4, 0.5], np.float32)
    sw = np.array([3, 1, 0.25], np.float32)
    y = oracle_mod.w4a4_gemm(_pack(qx), sx, _pack(qw), sw)
    assert np.array_equal(y, base * sx[:, None].astype(np.float64) * sw[None, :].astype(np.float64))
    assert np.array_equal(base, (qx @ qw.T).astype(np.float64))
