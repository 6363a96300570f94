"""The two-stage path for factors up to 256 (kq_transform_quant_two_stage,
FlatQuant page, "The fused kernel", Figure 8 (c)) against the fp64 oracle,
through the C ABI.

Rules (the same as for kq_transform_quant):
  * INT4 codes: bit-exact, except +-1 where the oracle's y/s lies within 1e-3
    of a rounding boundary; such mismatches at most 0.1% of the codes.
  * scales: within 1e-3 relative (both 0 for an all-zero token).
  * nothing outside the codes, the scales and the workspace is written.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from kq_testutil import parity_codes, scale_rel_err
from kronecker_factored_transforms_b200.workloads import f32_to_bf16_bits, make_workload

pytestmark = pytest.mark.gpu

CANARY = 0xA5
PAD = 4096


@pytest.fixture(scope="module")
def kq():
    from kronecker_factored_transforms_b200 import _lib
    return _lib


class Guarded:
    """A device byte buffer with canary bytes on both sides of the payload."""

    def __init__(self, nbytes: int):
        self.n = nbytes
        self.buf = torch.full((nbytes + 2 * PAD,), CANARY, dtype=torch.uint8, device="cuda")

    def ptr(self) -> int:
        return self.buf.data_ptr() + PAD

    def payload(self) -> np.ndarray:
        return self.buf[PAD:PAD + self.n].cpu().numpy()

    def check(self):
        head = self.buf[:PAD].cpu().numpy()
        tail = self.buf[PAD + self.n:].cpu().numpy()
        assert (head == CANARY).all() and (tail == CANARY).all(), "write outside the buffer"


def random_inputs(T, n1, n2, scaled, seed, factors="orthogonal"):
    """Seeded N(0,1) rows with 1% of the channels x30, bf16; orthogonal or
    near-identity bf16 factors; c ~ logU[0.5, 2] passed as 1/c."""
    rng = np.random.default_rng(seed)
    n = n1 * n2

    def factor(k):
        if factors == "orthogonal":
            Q, R = np.linalg.qr(rng.standard_normal((k, k)))
            return Q * np.sign(np.diag(R))
        return np.eye(k) + 0.1 * rng.standard_normal((k, k)) / math.sqrt(k)

    P1, P2 = factor(n1), factor(n2)
    x = rng.standard_normal((T, n))
    x[:, rng.choice(n, max(1, n // 100), replace=False)] *= 30.0
    cinv = None
    if scaled:
        cinv = (1.0 / np.exp(rng.uniform(math.log(0.5), math.log(2.0), n))).astype(np.float32)
    bits = lambda a: f32_to_bf16_bits(a.astype(np.float32))
    return bits(x), bits(P1), bits(P2), cinv


def dev_u16(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda()


def run_two_stage(kq, x, P1, P2, cinv, alpha, T, n1, n2, stream=None):
    n = n1 * n2
    need = kq.kq_two_stage_workspace_bytes(T, n1, n2)
    q, s, w = Guarded(T * n // 2), Guarded(T * 4), Guarded(need)
    xd, p1, p2 = dev_u16(x), dev_u16(P1), dev_u16(P2)
    cd = None if cinv is None else torch.from_numpy(cinv).cuda()
    kq.kq_transform_quant_two_stage(xd, p1, p2, cd, alpha, q.ptr(), s.ptr(), w.ptr(), need, T, n1, n2,
                                    stream=stream)
    torch.cuda.synchronize()
    for g in (q, s, w):
        g.check()
    assert kq.kq_device_error() == 0
    return q.payload().reshape(T, n // 2), s.payload().view(np.float32).copy()


def check_parity(packed, scales, ref):
    codes = oracle.unpack_codes(packed)
    ok, _, _, msg = parity_codes(codes, ref["codes"], ref["dist"])
    assert ok, msg
    assert scale_rel_err(scales, ref["scale32"]) <= 1e-3


SHAPES = [  # T, n1, n2, cinv, alpha
    (1, 256, 256, True, 0.85),
    (6, 256, 256, False, 0.9),
    (7, 144, 256, True, 0.9),
    (9, 256, 144, False, 0.9),
    (33, 112, 256, False, 0.9),
    (17, 16, 256, True, 0.85),
    (13, 256, 16, False, 0.9),
    (40, 64, 128, True, 0.85),
    (5, 208, 240, True, 0.7),
    (130, 128, 224, False, 0.9),
]


@pytest.mark.parametrize("T,n1,n2,scaled,alpha", SHAPES)
def test_two_stage_matches_oracle(kq, T, n1, n2, scaled, alpha):
    x, P1, P2, cinv = random_inputs(T, n1, n2, scaled, seed=T * 1000 + n1 + n2)
    packed, scales = run_two_stage(kq, x, P1, P2, cinv, alpha, T, n1, n2)
    check_parity(packed, scales, oracle.transform_quant(x, P1, P2, cinv, alpha, n1, n2))


def test_two_stage_near_identity_and_zero_token(kq):
    """Heavy-tailed rows through near-identity factors (the largest codes sit on
    single elements), with an all-zero token: scale 0 and all codes 0."""
    T, n1, n2 = 11, 256, 208
    x, P1, P2, cinv = random_inputs(T, n1, n2, True, seed=77, factors="near_identity")
    x[4] = 0
    packed, scales = run_two_stage(kq, x, P1, P2, cinv, 0.85, T, n1, n2)
    assert scales[4] == 0.0 and (packed[4] == 0).all()
    check_parity(packed, scales, oracle.transform_quant(x, P1, P2, cinv, 0.85, n1, n2))


def test_two_stage_deterministic_and_stream(kq):
    T, n1, n2 = 21, 160, 256
    x, P1, P2, cinv = random_inputs(T, n1, n2, True, seed=5)
    a = run_two_stage(kq, x, P1, P2, cinv, 0.9, T, n1, n2)
    st = torch.cuda.Stream()
    b = run_two_stage(kq, x, P1, P2, cinv, 0.9, T, n1, n2, stream=st)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])


@pytest.mark.parametrize("name,samples", [("square65536", 10), ("ffn28672", 24)])
def test_two_stage_full_size_sampled(kq, name, samples):
    """The full large-factor workloads (as the benchmark runs them) on the GPU;
    sampled tokens, the first and the last among them, against the oracle."""
    w = make_workload(name)
    packed, scales = run_two_stage(kq, w.x, w.P1, w.P2, w.cinv, w.alpha, w.T, w.n1, w.n2)
    rng = np.random.default_rng(w.T)
    rows = np.unique(np.concatenate([rng.choice(w.T, samples, replace=False), [0, w.T - 1]]))
    ref = oracle.transform_quant(w.x[rows], w.P1, w.P2, w.cinv, w.alpha, w.n1, w.n2)
    check_parity(packed[rows], scales[rows], ref)
    assert (scales > 0).all()
