"""The per-head transform with NVFP4 rows (kq_headwise_transform_quant_nvfp4)
against the fp64 oracle, through the C ABI.

Rules (the INT4 rules carried over to the two rounding steps of NVFP4):
  * row scales within 1e-5 relative (both are fp32 of max|y| / 2688);
  * block-scale codes equal, except for blocks whose raw scale lies within 1e-3
    of an E4M3 rounding boundary (in units of the local step): those blocks are
    left out of the element comparison;
  * element codes equal, except one step of magnitude where the oracle's value
    lies within 1e-3 of an E2M1 rounding boundary (in units of the local step);
    such mismatches at most 0.1 % of the compared codes;
  * a code of magnitude zero carries no sign;
  * nothing outside the three outputs is written.
"""
import numpy as np
import pytest
import torch

import oracle
from kronecker_factored_transforms_b200.workloads import f32_to_bf16_bits

pytestmark = pytest.mark.gpu

CANARY = 0xA5
PAD = 4096
WINDOW = 1e-3


@pytest.fixture(scope="module")
def kq():
    from kronecker_factored_transforms_b200 import _lib
    return _lib


class Guarded:
    def __init__(self, nbytes):
        self.n = nbytes
        self.buf = torch.full((nbytes + 2 * PAD,), CANARY, dtype=torch.uint8, device="cuda")

    def ptr(self):
        return self.buf.data_ptr() + PAD

    def payload(self):
        return self.buf[PAD:PAD + self.n].cpu().numpy()

    def check(self):
        b = self.buf.cpu().numpy()
        assert (b[:PAD] == CANARY).all() and (b[PAD + self.n:] == CANARY).all(), "write outside output"


def inputs(T, heads, D, seed, spread=3.0):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((T, heads * D))
    # per-row magnitudes over a wide range, a few outlier channels, and inside a
    # row some nearly-empty blocks (their E4M3 scales go subnormal)
    x *= np.exp(rng.uniform(-spread, spread, (T, 1)))
    x[:, rng.choice(heads * D, max(1, heads * D // 100), replace=False)] *= 30.0
    Q, R = np.linalg.qr(rng.standard_normal((D, D)))
    P = Q * np.sign(np.diag(R))
    return f32_to_bf16_bits(x.astype(np.float32)), f32_to_bf16_bits(P.astype(np.float32))


def run(kq, xb, Pb, T, heads, D):
    R = T * heads
    q, bs, s = Guarded(R * D // 2), Guarded(R * D // 16), Guarded(R * 4)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda()
    kq.kq_headwise_transform_quant_nvfp4(dev(xb), dev(Pb), q.ptr(), bs.ptr(), s.ptr(), T, heads, D)
    torch.cuda.synchronize()
    for g in (q, bs, s):
        g.check()
    assert kq.kq_device_error() == 0
    return (q.payload().reshape(R, D // 2), bs.payload().reshape(R, D // 16), s.payload().view(np.float32).copy())


def unpack(packed):
    return np.stack([packed & 0xF, packed >> 4], axis=-1).reshape(packed.shape[0], -1)


def check(packed, block, scale, ref, D):
    R = packed.shape[0]
    sref = ref["scale32"].astype(np.float64)
    np.testing.assert_allclose(scale.astype(np.float64), sref, rtol=1e-5, atol=0)
    bad_block = block != ref["block"]
    near_b = ref["bdist"] < WINDOW
    assert not (bad_block & ~near_b).any(), "block-scale codes differ away from a rounding boundary"
    codes = unpack(packed)
    mag, sgn = codes & 7, codes >> 3
    assert not ((mag == 0) & (sgn == 1)).any(), "signed zero code"
    rmag, rsgn = ref["codes"] & 7, ref["codes"] >> 3
    keep = ~np.repeat(near_b, 16, axis=1)
    diff = (codes != ref["codes"]) & keep
    allowed = diff & (np.abs(mag.astype(int) - rmag.astype(int)) == 1) & (ref["dist"] < WINDOW) & \
        ((sgn == rsgn) | (mag == 0) | (rmag == 0))
    bad = diff & ~allowed
    assert not bad.any(), "%d element codes differ outside the window; first %s" % (
        int(bad.sum()), np.argwhere(bad)[:3].tolist())
    assert diff.sum() <= 1e-3 * keep.sum()


@pytest.mark.parametrize("T,heads,D", [(1, 1, 128), (7, 8, 128), (33, 32, 128), (5, 3, 64), (130, 1, 128),
                                       (64, 8, 64)])
def test_nvfp4_matches_oracle(kq, T, heads, D):
    xb, Pb = inputs(T, heads, D, seed=T * 100 + heads + D)
    packed, block, scale = run(kq, xb, Pb, T, heads, D)
    check(packed, block, scale, oracle.headwise_transform_nvfp4(xb, Pb, heads, D), D)


def test_nvfp4_zero_rows_and_tiny_blocks(kq):
    T, heads, D = 9, 4, 128
    xb, Pb = inputs(T, heads, D, seed=21, spread=6.0)
    xb = xb.copy()
    xb[3] = 0                                   # all four heads of token 3 are zero
    packed, block, scale = run(kq, xb, Pb, T, heads, D)
    rows = slice(3 * heads, 4 * heads)
    assert (scale[rows] == 0).all() and (block[rows] == 0).all() and (packed[rows] == 0).all()
    check(packed, block, scale, oracle.headwise_transform_nvfp4(xb, Pb, heads, D), D)


def test_nvfp4_full_size_sampled(kq):
    """8192 tokens x 32 heads x 128 (the benchmark's size): sampled rows against the oracle."""
    T, heads, D = 8192, 32, 128
    xb, Pb = inputs(T, heads, D, seed=8192)
    packed, block, scale = run(kq, xb, Pb, T, heads, D)
    rng = np.random.default_rng(1)
    toks = np.unique(np.concatenate([rng.choice(T, 40, replace=False), [0, T - 1]]))
    rows = (toks[:, None] * heads + np.arange(heads)[None, :]).reshape(-1)
    ref = oracle.headwise_transform_nvfp4(xb[toks], Pb, heads, D)
    check(packed[rows], block[rows], scale[rows], ref, D)
