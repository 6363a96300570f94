"""Per-head transform of the key / value cache (kq_headwise_transform_quant)
against the oracle: the rules of the fused path apply per (token, head) row
(codes bit-exact except +-1 within 1e-3 of a rounding boundary, at most 0.1% of
codes; scales within 1e-3 relative); nothing outside the outputs is written."""
import numpy as np
import pytest
import torch

import oracle
from kq_testutil import parity_codes, scale_rel_err
from kronecker_factored_transforms_b200.workloads import f32_to_bf16_bits

pytestmark = pytest.mark.gpu
CANARY, PAD = 0xA5, 4096


@pytest.fixture(scope="module")
def kq():
    from kronecker_factored_transforms_b200 import _lib
    return _lib


def _inputs(T, heads, D, seed, outliers=True):
    rng = np.random.default_rng(seed)
    q, r = np.linalg.qr(rng.standard_normal((D, D)))
    Ph = f32_to_bf16_bits((q * np.sign(np.diag(r))).astype(np.float32))
    x = rng.standard_normal((T, heads, D))
    if outliers:  # a few large channels per head, as keys carry
        x[:, :, rng.choice(D, 4, replace=False)] *= 20.0
    return f32_to_bf16_bits(x.reshape(T, heads * D).astype(np.float32)), Ph


def _run(kq, x, Ph, alpha, T, heads, D):
    nq, ns = T * heads * D // 2, T * heads * 4
    qb = torch.full((nq + 2 * PAD,), CANARY, dtype=torch.uint8, device="cuda")
    sb = torch.full((ns + 2 * PAD,), CANARY, dtype=torch.uint8, device="cuda")
    xd = torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).cuda()
    pd = torch.from_numpy(np.ascontiguousarray(Ph).view(np.int16)).cuda()
    kq.kq_headwise_transform_quant(xd, pd, alpha, qb.data_ptr() + PAD, sb.data_ptr() + PAD, T, heads, D)
    torch.cuda.synchronize()
    qh, sh = qb.cpu().numpy(), sb.cpu().numpy()
    for b, n in ((qh, nq), (sh, ns)):
        assert (b[:PAD] == CANARY).all() and (b[PAD + n:] == CANARY).all(), "write outside output"
    return qh[PAD:PAD + nq].reshape(T, heads * D // 2), sh[PAD:PAD + ns].view(np.float32).reshape(T, heads)


def _check(q, s, x, Ph, alpha, heads, D):
    ref = oracle.headwise_transform_quant(x, Ph, alpha, heads, D)
    ok, _, _, msg = parity_codes(oracle.unpack_codes(q), ref["codes"], ref["dist"])
    assert ok, msg
    assert scale_rel_err(s, ref["scale32"]) <= 1e-3


@pytest.mark.parametrize("T,heads,D", [(1, 1, 128), (5, 8, 128), (37, 32, 128), (3, 5, 64), (64, 32, 64),
                                       (1000, 8, 64), (257, 8, 128)])
def test_headwise_matches_oracle(kq, T, heads, D):
    x, Ph = _inputs(T, heads, D, T * 31 + heads * 7 + D)
    q, s = _run(kq, x, Ph, 0.9, T, heads, D)
    _check(q, s, x, Ph, 0.9, heads, D)


@pytest.mark.parametrize("alpha", [1.0, 0.75, 0.5])
def test_headwise_alpha(kq, alpha):
    x, Ph = _inputs(64, 8, 128, 77)
    q, s = _run(kq, x, Ph, alpha, 64, 8, 128)
    _check(q, s, x, Ph, alpha, 8, 128)


def test_headwise_zero_rows(kq):
    x, Ph = _inputs(16, 8, 128, 3)
    x = x.reshape(16, 8, 128)
    x[2] = 0          # a whole token
    x[5, 3] = 0       # one head of a token
    x = x.reshape(16, 8 * 128)
    q, s = _run(kq, x, Ph, 0.9, 16, 8, 128)
    assert (s[2] == 0).all() and s[5, 3] == 0
    assert (q[2] == 0).all() and (q[5, 3 * 64:4 * 64] == 0).all()
    _check(q, s, x, Ph, 0.9, 8, 128)


def test_headwise_full_size_kv_cache(kq):
    """8192 tokens x 8 key heads x 128 (a grouped-query layer's keys): all rows."""
    x, Ph = _inputs(8192, 8, 128, 8192)
    q, s = _run(kq, x, Ph, 0.9, 8192, 8, 128)
    _check(q, s, x, Ph, 0.9, 8, 128)
