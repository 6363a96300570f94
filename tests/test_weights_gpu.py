"""Weight-side transform on the GPU (through kq_transform_quant) against the oracle.

The weight rows of a W4A4 layer are transformed with factors P1^-T, P2^-T and
the channel vector c, then quantised per row (one scale per output channel):
the same rules as the activation path apply (codes bit-exact except +-1 within
1e-3 of a rounding boundary, at most 0.1% of codes; scales within 1e-3).
"""
import numpy as np
import pytest
import torch

import oracle
from kq_testutil import parity_codes, scale_rel_err
from kronecker_factored_transforms_b200 import weights as kw
from kronecker_factored_transforms_b200.workloads import bf16_bits_to_f32, make_weights, make_workload

pytestmark = pytest.mark.gpu


def _dev16(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda()


def _gpu_weight_quant(W, F1, F2, c, alpha, n1, n2):
    n_out, n = W.shape
    q = torch.empty((n_out, n // 2), dtype=torch.uint8, device="cuda")
    s = torch.empty((n_out,), dtype=torch.float32, device="cuda")
    kw.weight_transform_quant(_dev16(W), _dev16(F1), _dev16(F2), torch.from_numpy(c).cuda(), alpha, q, s, n1, n2)
    torch.cuda.synchronize()
    return q.cpu().numpy(), s.cpu().numpy()


@pytest.mark.parametrize("alpha", [1.0, 0.9])
def test_weight_transform_parity(alpha):
    w = make_workload("hidden8192", rows=1)
    c = (1.0 / w.cinv.astype(np.float64)).astype(np.float32)
    F1, F2 = kw.weight_factors_bf16(w.P1, w.P2)
    W = make_weights(w.n, 512, 2)
    q, s = _gpu_weight_quant(W, F1, F2, c, alpha, w.n1, w.n2)
    ref = oracle.transform_quant(W, F1, F2, c, alpha, w.n1, w.n2)
    ok, _, _, msg = parity_codes(oracle.unpack_codes(q), ref["codes"], ref["dist"])
    assert ok, msg
    assert scale_rel_err(s, ref["scale32"]) <= 1e-3


def test_w4a4_product_from_gpu_codes():
    """x W^T from the GPU's activation and weight codes agrees with the same product
    from the oracle's codes (their codes differ only in allowed boundary cases), and its
    error against the exact product is what the high-rate model predicts, on a
    layer with orthogonal factors (the sweep configuration's, 64 x 64) where that
    model holds: within -10% / +15% (alpha = 0.9 clips a few activations)."""
    w = make_workload("sweep4096", rows=256)
    n1, n2, n = w.n1, w.n2, w.n
    F1, F2 = kw.weight_factors_bf16(w.P1, w.P2)
    W = make_weights(n, 256, 5)
    n_out = W.shape[0]
    qw = torch.empty((n_out, n // 2), dtype=torch.uint8, device="cuda")
    sw = torch.empty((n_out,), dtype=torch.float32, device="cuda")
    kw.weight_transform_quant(_dev16(W), _dev16(F1), _dev16(F2), None, 1.0, qw, sw, n1, n2)
    qx = torch.empty((256, n // 2), dtype=torch.uint8, device="cuda")
    sx = torch.empty((256,), dtype=torch.float32, device="cuda")
    from kronecker_factored_transforms_b200 import _lib
    _lib.kq_transform_quant(_dev16(w.x), _dev16(w.P1), _dev16(w.P2), None, w.alpha, qx, sx, 256, n1, n2)
    torch.cuda.synchronize()
    xh = oracle.unpack_codes(qx.cpu().numpy()).astype(np.float64) * sx.cpu().numpy()[:, None]
    wh = oracle.unpack_codes(qw.cpu().numpy()).astype(np.float64) * sw.cpu().numpy()[:, None]
    rx = oracle.transform_quant(w.x, w.P1, w.P2, None, w.alpha, n1, n2)
    rw = oracle.transform_quant(W, F1, F2, None, 1.0, n1, n2)
    xr = rx["codes"].astype(np.float64) * rx["scale32"][:, None]
    wr = rw["codes"].astype(np.float64) * rw["scale32"][:, None]
    y_gpu, y_ref = xh @ wh.T, xr @ wr.T
    # the codes agree up to the allowed +-1 boundary cases (checked code by code in
    # the parity tests); one such case moves a whole row of the product by
    # s_x |w'_k|, about 1 / (2 sqrt(n)) of that row, so the products agree to ~1e-2
    assert np.linalg.norm(y_gpu - y_ref) <= 1e-2 * np.linalg.norm(y_ref)
    yx = oracle.transform(w.x, w.P1, w.P2, None, n1, n2)
    yw = oracle.transform(W, F1, F2, None, n1, n2)
    exact = yx @ yw.T
    err = np.linalg.norm(y_gpu - exact) ** 2
    pred = (np.sum(rx["scale64"] ** 2 / 12.0) * np.sum(yw ** 2) + np.sum(rw["scale64"] ** 2 / 12.0) * np.sum(yx ** 2))
    assert 0.9 * pred < err < 1.15 * pred, err / pred
    # and the transformed pair reproduces x W^T of the untransformed layer
    plain = bf16_bits_to_f32(w.x).astype(np.float64) @ bf16_bits_to_f32(W).astype(np.float64).T
    assert np.linalg.norm(exact - plain) <= 1e-2 * np.linalg.norm(plain)
