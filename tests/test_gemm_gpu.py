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
