"""The W4A4 product kernel (kq_w4a4_gemm) against the oracle.

The integer sums are exact on both sides; the kernel then rounds twice in
fp32 ((float(sum) * sx) * sw), so each output is within 2^-23 relative of the
oracle's fp64 value: the bound used below.  Nothing outside y is written.
"""
import numpy as np
import pytest
import torch

import oracle
from kronecker_factored_transforms_b200 import weights as kw
from kronecker_factored_transforms_b200.workloads import make_weights, make_workload

pytestmark = pytest.mark.gpu

REL = 2.0 ** -23 * 1.01
CANARY = 0x7FC00000  # a NaN bit pattern: any stray write is visible
PAD = 1024           # floats of canary on each side of y


@pytest.fixture(scope="module")
def kq():
    from kronecker_factored_transforms_b200 import _lib
    return _lib


def _codes(rng, rows, K):
    return rng.integers(0, 256, (rows, K // 2), dtype=np.uint8)


def _run(kq, qx, sx, qw, sw):
    M, N, K = qx.shape[0], qw.shape[0], qx.shape[1] * 2
    buf = torch.full((M * N + 2 * PAD,), CANARY, dtype=torch.int32, device="cuda")
    y = buf[PAD:PAD + M * N].view(torch.float32)
    kq.kq_w4a4_gemm(torch.from_numpy(qx).cuda(), torch.from_numpy(sx).cuda(), torch.from_numpy(qw).cuda(),
                    torch.from_numpy(sw).cuda(), y, M, N, K)
    torch.cuda.synchronize()
    b = buf.cpu().numpy()
    assert (b[:PAD] == CANARY).all() and (b[PAD + M * N:] == CANARY).all(), "write outside y"
    return y.cpu().numpy().reshape(M, N)


def _check(y, ref):
    err = np.abs(y.astype(np.float64) - ref)
    bad = err > REL * np.abs(ref)
    assert not bad.any(), "%d outputs off, worst at %s: %r vs %r" % (
        int(bad.sum()), np.argwhere(bad)[0].tolist(), y[tuple(np.argwhere(bad)[0])], ref[tuple(np.argwhere(bad)[0])])


@pytest.mark.parametrize("M,N,K", [(1, 1, 128), (37, 53, 256), (128, 128, 128), (129, 127, 384),
                                   (200, 300, 1024), (256, 384, 4096), (64, 1000, 8192), (513, 65, 14336)])
def test_gemm_matches_oracle(kq, M, N, K):
    rng = np.random.default_rng(M * 7 + N * 13 + K)
    qx, qw = _codes(rng, M, K), _codes(rng, N, K)
    sx = rng.uniform(1e-3, 2.0, M).astype(np.float32)
    sw = rng.uniform(1e-3, 2.0, N).astype(np.float32)
    _check(_run(kq, qx, sx, qw, sw), oracle.w4a4_gemm(qx, sx, qw, sw))


def test_gemm_extreme_codes(kq):
    """All -8 against all 7 / all -8: the largest sums the codes allow, K = 16384."""
    K = 16384
    qx = np.full((130, K // 2), 0x88, dtype=np.uint8)          # -8, -8
    qw = np.stack([np.full(K // 2, 0x77, dtype=np.uint8),      # 7, 7
                   np.full(K // 2, 0x88, dtype=np.uint8)])     # -8, -8
    y = _run(kq, qx, np.ones(130, np.float32), qw, np.ones(2, np.float32))
    assert (y[:, 0] == -56 * K).all() and (y[:, 1] == 64 * K).all()


def test_gemm_full_size_sampled_rows(kq):
    """M = N = K = 8192 (the hidden-size-8192 layer): 48 sampled rows against the oracle."""
    rng = np.random.default_rng(8192)
    M = N = K = 8192
    qx, qw = _codes(rng, M, K), _codes(rng, N, K)
    sx = rng.uniform(1e-3, 2.0, M).astype(np.float32)
    sw = rng.uniform(1e-3, 2.0, N).astype(np.float32)
    y = _run(kq, qx, sx, qw, sw)
    rows = np.sort(rng.choice(M, 48, replace=False))
    rows = np.unique(np.concatenate([rows, [0, 127, 128, M - 1]]))
    _check(y[rows], oracle.w4a4_gemm(qx[rows], sx[rows], qw, sw))


def _bf16_to_f64(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _f64_to_bf16_rne(a):
    """Round fp64 values to bf16 (nearest, ties to even) through float32 with
    a sticky bit, so that no double rounding changes a tie."""
    f = a.astype(np.float32)
    # float32 rounding may have created or broken a bf16 tie: fall back to exact
    # comparison of both bf16 neighbours of the float32 value
    b = f.view(np.uint32)
    lo = (b & 0xFFFF0000).view(np.float32).astype(np.float64)
    hi = ((b & 0xFFFF0000) + 0x10000).astype(np.uint32).view(np.float32).astype(np.float64)
    dlo, dhi = np.abs(a - lo), np.abs(hi - a)
    pick_hi = (dhi < dlo) | ((dhi == dlo) & (((b >> 16) & 1) == 1))
    return np.where(pick_hi, ((b >> 16) + 1) & 0xFFFF, (b >> 16) & 0xFFFF).astype(np.uint16)


@pytest.mark.parametrize("M,N,K", [(1, 1, 128), (37, 53, 256), (129, 127, 384), (200, 300, 1024), (513, 65, 14336)])
def test_gemm_bf16_output(kq, M, N, K):
    """kq_w4a4_gemm_bf16 rounds the fp32 value to the nearest bf16: equal to the
    oracle's fp64 product rounded to bf16, except (by one bf16 ulp) where the
    fp64 value lies within the fp32 error (2^-22 relative) of a bf16 midpoint."""
    rng = np.random.default_rng(M * 5 + N * 11 + K)
    qx, qw = _codes(rng, M, K), _codes(rng, N, K)
    sx = rng.uniform(1e-3, 2.0, M).astype(np.float32)
    sw = rng.uniform(1e-3, 2.0, N).astype(np.float32)
    PADH = 2048
    buf = torch.full((M * N + 2 * PADH,), 0x7FC1, dtype=torch.int16, device="cuda")
    y = buf[PADH:PADH + M * N]
    kq.kq_w4a4_gemm_bf16(torch.from_numpy(qx).cuda(), torch.from_numpy(sx).cuda(), torch.from_numpy(qw).cuda(),
                         torch.from_numpy(sw).cuda(), y, M, N, K)
    torch.cuda.synchronize()
    b = buf.cpu().numpy()
    assert (b[:PADH] == 0x7FC1).all() and (b[PADH + M * N:] == 0x7FC1).all(), "write outside y"
    got = y.cpu().numpy().view(np.uint16).reshape(M, N)
    ref64 = oracle.w4a4_gemm(qx, sx, qw, sw)
    want = _f64_to_bf16_rne(ref64)
    differ = got != want
    if differ.any():
        # only where the exact value is within the fp32 error of a bf16 midpoint
        v = ref64[differ]
        f = v.astype(np.float32).view(np.uint32)
        mid = ((f & 0xFFFF0000) | 0x8000).view(np.float32).astype(np.float64)
        assert (np.abs(v - mid) <= 2.0 ** -22 * np.abs(v)).all(), "bf16 outputs off beyond a midpoint"
        assert (np.abs(got[differ].astype(np.int32) - want[differ].astype(np.int32)) <= 1).all()
    assert differ.mean() < 1e-3


def test_layer_codes_through_the_gemm(kq):
    """Activation codes from kq_transform_quant and weight codes from the
    weight-side transform, multiplied by kq_w4a4_gemm, equal the oracle's product
    of the same codes."""
    w = make_workload("hidden8192", rows=256)
    n1, n2, n = w.n1, w.n2, w.n
    c = (1.0 / w.cinv.astype(np.float64)).astype(np.float32)
    F1, F2 = kw.weight_factors_bf16(w.P1, w.P2)
    W = make_weights(n, 384, 9)
    dev16 = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda()
    qx = torch.empty((256, n // 2), dtype=torch.uint8, device="cuda")
    sx = torch.empty((256,), dtype=torch.float32, device="cuda")
    qw = torch.empty((384, n // 2), dtype=torch.uint8, device="cuda")
    sw = torch.empty((384,), dtype=torch.float32, device="cuda")
    kq.kq_transform_quant(dev16(w.x), dev16(w.P1), dev16(w.P2), torch.from_numpy(w.cinv).cuda(), w.alpha,
                          qx, sx, 256, n1, n2)
    kw.weight_transform_quant(dev16(W), dev16(F1), dev16(F2), torch.from_numpy(c).cuda(), 1.0, qw, sw, n1, n2)
    y = torch.empty((256, 384), dtype=torch.float32, device="cuda")
    kq.kq_w4a4_gemm(qx, sx, qw, sw, y, 256, 384, n)
    torch.cuda.synchronize()
    ref = oracle.w4a4_gemm(qx.cpu().numpy(), sx.cpu().numpy(), qw.cpu().numpy(), sw.cpu().numpy())
    _check(y.cpu().numpy(), ref)
