"""Parity of the CUDA path (through the C ABI) with the fp64 oracle.

Rules (written here, from the contract of the path):
  * INT4 codes: bit-exact, except +-1 where the oracle's y/s lies within 1e-3
    of a rounding boundary; such mismatches at most 0.1% of the codes.
  * scales: within 1e-3 relative (both 0 for an all-zero token).
  * transform check entry: per token max|y_gpu - y_ref| / max|y_ref| <= 1e-2.
  * nothing outside the outputs is written (canary bytes around each buffer).
"""
import numpy as np
import pytest
import torch

import oracle
from kq_testutil import parity_codes, scale_rel_err, token_rel_err
from kronecker_factored_transforms_b200.workloads import (SWEEP_T, f32_to_bf16_bits, make_workload)

pytestmark = pytest.mark.gpu

CANARY = 0xA5
PAD = 4096  # bytes of canary on each side


@pytest.fixture(scope="module")
def kq():
    from kronecker_factored_transforms_b200 import _lib
    return _lib


def dev_u16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda()


def dev_f32(a) -> torch.Tensor:
    return None if a is None else torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


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
        b = self.buf.cpu().numpy()
        assert (b[:PAD] == CANARY).all() and (b[PAD + self.n:] == CANARY).all(), "write outside output"


def run_quant(kq, x, P1, P2, cinv, alpha, T, n1, n2, stream=None):
    n = n1 * n2
    xd, p1, p2, cd = dev_u16(x), dev_u16(P1), dev_u16(P2), dev_f32(cinv)
    q = Guarded(T * n // 2)
    s = Guarded(T * 4)
    kq.kq_transform_quant(xd, p1, p2, cd, alpha, q.ptr(), s.ptr(), T, n1, n2, stream=stream)
    torch.cuda.synchronize()
    q.check()
    s.check()
    return q.payload().reshape(T, n // 2), s.payload().view(np.float32).copy()


def run_transform(kq, x, P1, P2, cinv, T, n1, n2):
    y = torch.empty((T, n1 * n2), dtype=torch.float32, device="cuda")
    kq.kq_transform(dev_u16(x), dev_u16(P1), dev_u16(P2), dev_f32(cinv), y, T, n1, n2)
    torch.cuda.synchronize()
    return y.cpu().numpy().astype(np.float64)


def assert_quant_parity(x, P1, P2, cinv, alpha, n1, n2, q_gpu, s_gpu, chunk=1024):
    T = x.shape[0]
    tot_m = 0
    for t0 in range(0, T, chunk):
        ref = oracle.transform_quant(x[t0:t0 + chunk], P1, P2, cinv, alpha, n1, n2)
        codes_gpu = oracle.unpack_codes(q_gpu[t0:t0 + chunk])
        ok, n_m, n_bad, msg = parity_codes(codes_gpu, ref["codes"], ref["dist"])
        assert n_bad == 0, "tokens %d..: %s" % (t0, msg)
        tot_m += n_m
        assert scale_rel_err(s_gpu[t0:t0 + chunk], ref["scale32"]) <= 1e-3
        zero = ref["scale32"] == 0
        assert (s_gpu[t0:t0 + chunk][zero] == 0).all()
    assert tot_m <= 1e-3 * x.size, "too many window mismatches: %d of %d" % (tot_m, x.size)
    return tot_m


# ---------------------------------------------------------------------------
# The five configurations at full size.

@pytest.mark.parametrize("name", ["tiny", "llama7b_hidden", "hidden8192", "mlp14336", "mlp14336_cinv", "hidden5120"])
def test_config_full_size(kq, name):
    w = make_workload(name)
    q, s = run_quant(kq, w.x, w.P1, w.P2, w.cinv, w.alpha, w.T, w.n1, w.n2)
    assert_quant_parity(w.x, w.P1, w.P2, w.cinv, w.alpha, w.n1, w.n2, q, s)


@pytest.mark.parametrize("T", SWEEP_T)
def test_sweep(kq, T):
    w = make_workload("sweep4096", T=T)
    q, s = run_quant(kq, w.x, w.P1, w.P2, w.cinv, w.alpha, w.T, w.n1, w.n2)
    if T <= 16384:
        assert_quant_parity(w.x, w.P1, w.P2, w.cinv, w.alpha, 64, 64, q, s)
    else:
        # largest size: every leading token plus a random sample, token by token
        rng = np.random.default_rng(T)
        rows = np.unique(np.concatenate([np.arange(2048), rng.choice(T, 2048, replace=False), [T - 1]]))
        assert_quant_parity(w.x[rows], w.P1, w.P2, None, w.alpha, 64, 64, q[rows], s[rows])


@pytest.mark.parametrize("name", ["tiny", "llama7b_hidden", "hidden8192", "mlp14336", "mlp14336_cinv", "hidden5120"])
def test_transform_check_entry(kq, name):
    w = make_workload(name, rows=512 if name != "tiny" else None)
    T = w.x.shape[0]
    y = run_transform(kq, w.x, w.P1, w.P2, w.cinv, T, w.n1, w.n2)
    ref = oracle.transform(w.x, w.P1, w.P2, w.cinv, w.n1, w.n2)
    err = token_rel_err(y, ref)
    assert err.max() <= 1e-2
    # design target of the hi/lo split: far inside the contract
    assert err.max() <= 1e-4, err.max()


# ---------------------------------------------------------------------------
# Shapes, ragged sizes and degenerate inputs.

SHAPES = [(16, 16), (16, 128), (128, 16), (32, 48), (48, 32), (64, 64), (64, 128), (112, 128),
          (128, 128), (80, 96), (80, 64), (96, 128), (112, 64), (128, 64),
          # n2 padded to 64 or 128 columns on the tensor cores
          (64, 80), (16, 48), (128, 48), (112, 112), (96, 80), (128, 112), (48, 96),
          (64, 32), (112, 16), (32, 32), (128, 32), (80, 16)]


@pytest.mark.parametrize("n1,n2", SHAPES)
@pytest.mark.parametrize("scaled", [False, True])
def test_shapes_ragged(kq, n1, n2, scaled):
    rng = np.random.default_rng(n1 * 1000 + n2 + (7 if scaled else 0))
    T = 37  # not a multiple of any per-CTA token group
    n = n1 * n2
    x = f32_to_bf16_bits(rng.standard_normal((T, n)).astype(np.float32) *
                         np.where(rng.random(n) < 0.01, 20.0, 1.0).astype(np.float32))
    P1 = f32_to_bf16_bits(np.linalg.qr(rng.standard_normal((n1, n1)))[0].astype(np.float32))
    P2 = f32_to_bf16_bits((np.eye(n2) + 0.1 * rng.standard_normal((n2, n2)) / np.sqrt(n2)).astype(np.float32))
    cinv = rng.uniform(0.5, 2.0, n).astype(np.float32) if scaled else None
    alpha = 0.9
    q, s = run_quant(kq, x, P1, P2, cinv, alpha, T, n1, n2)
    assert_quant_parity(x, P1, P2, cinv, alpha, n1, n2, q, s)


@pytest.mark.parametrize("name,T", [("hidden8192", 148 * 4), ("hidden8192", 148 * 4 + 1),
                                    ("llama7b_hidden", 148 * 112), ("llama7b_hidden", 148 * 112 + 2)])
def test_dispatch_boundary(kq, name, T):
    """The last size of the pair-pipelined kernel (on 148 SMs: 4 groups per SM with
    cinv, 56 without) and the first of the batch-pipelined one, both against the oracle."""
    w = make_workload(name, T=T)
    per_sm = 4 if w.cinv is not None else 56
    expect = ("kq_fused_kernel" if (T + 128 // w.n2 - 1) // (128 // w.n2) <= per_sm * 148
              else "kq_tc05_fused_kernel")
    if torch.cuda.get_device_properties(0).multi_processor_count == 148:
        assert kq.kq_kernel_for(T, w.n1, w.n2, w.cinv is not None, w.alpha) == expect
    q, s = run_quant(kq, w.x, w.P1, w.P2, w.cinv, w.alpha, T, w.n1, w.n2)
    assert_quant_parity(w.x, w.P1, w.P2, w.cinv, w.alpha, w.n1, w.n2, q, s)


@pytest.mark.parametrize("T", [1, 2, 3, 7])
def test_small_T(kq, T):
    w = make_workload("hidden8192", rows=T)
    q, s = run_quant(kq, w.x, w.P1, w.P2, w.cinv, w.alpha, T, 64, 128)
    assert_quant_parity(w.x, w.P1, w.P2, w.cinv, w.alpha, 64, 128, q, s)


@pytest.mark.parametrize("alpha", [1.0, 0.5, 0.3, float(np.float32(1 / (1 + np.exp(-2.0))))])
def test_alpha_values(kq, alpha):
    w = make_workload("llama7b_hidden", rows=96)
    q, s = run_quant(kq, w.x, w.P1, w.P2, None, alpha, 96, 64, 64)
    assert_quant_parity(w.x, w.P1, w.P2, None, alpha, 64, 64, q, s)


# 2^-19 is the smallest alpha the tcgen05 kernels take (their rounding needs
# |y / s| <= 7 / alpha < 2^22); 1e-7 goes to the warp-MMA kernel.  With so small
# an alpha the quantisation step s = alpha max|y| / 7 lies far below the
# transform's own precision (about 2^-16 of max|y|, the hi/lo bf16 operands), so
# the code of an element whose y is within a few 2^-13 max|y| of zero is not
# determined by the arithmetic; every other code saturates at 7 or -8 and must
# match exactly, and the scales match within 1e-3.
@pytest.mark.parametrize("alpha", [2.0 ** -19, 1e-7])
def test_tiny_alpha(kq, alpha):
    w = make_workload("llama7b_hidden", rows=96)
    q, s = run_quant(kq, w.x, w.P1, w.P2, None, alpha, 96, 64, 64)
    ref = oracle.transform_quant(w.x, w.P1, w.P2, None, alpha, 64, 64)
    assert scale_rel_err(np.asarray(s), ref["scale32"]) <= 1e-3
    y = oracle.transform(w.x, w.P1, w.P2, None, 64, 64)
    r = y / ref["scale64"][:, None]
    band = 2.0 ** -13 * 7.0 / np.float32(alpha)  # the precision bound in units of s
    sure = np.abs(r) > 8.5 + band
    codes = oracle.unpack_codes(np.asarray(q))
    assert sure.mean() > 0.99
    np.testing.assert_array_equal(codes[sure], ref["codes"][sure])
    assert codes.min() >= -8 and codes.max() <= 7


def test_degenerate_tokens(kq):
    """All-zero tokens (s = 0, codes 0), tiny and huge magnitudes, one-hot rows."""
    w = make_workload("hidden8192", rows=12)
    x = w.x.copy()
    xf = (x.astype(np.uint32) << 16).view(np.float32)
    x[0] = 0
    x[5] = 0
    x[2] = f32_to_bf16_bits(xf[2] * np.float32(1e-20))
    x[3] = f32_to_bf16_bits(xf[3] * np.float32(1e20))
    x[4] = 0
    x[4, 1234] = f32_to_bf16_bits(np.array([3.0], np.float32))[0]
    x[11] = f32_to_bf16_bits(np.full(8192, -2.5, np.float32))
    q, s = run_quant(kq, x, w.P1, w.P2, w.cinv, w.alpha, 12, 64, 128)
    assert s[0] == 0 and s[5] == 0 and not q[0].any() and not q[5].any()
    assert_quant_parity(x, w.P1, w.P2, w.cinv, w.alpha, 64, 128, q, s)


def test_deterministic_and_stream_ordered(kq):
    w = make_workload("mlp14336", rows=300)
    outs = []
    st = torch.cuda.Stream()
    for k in range(3):
        with torch.cuda.stream(st):
            q, s = run_quant(kq, w.x, w.P1, w.P2, None, w.alpha, 300, 112, 128, stream=st)
        outs.append((q, s))
    for q, s in outs[1:]:
        np.testing.assert_array_equal(q, outs[0][0])
        np.testing.assert_array_equal(s, outs[0][1])


# ---------------------------------------------------------------------------
# The dequantise / inverse check entry.

def test_dequant_inverse_matches_oracle_and_round_trips(kq):
    w = make_workload("hidden8192", rows=64)
    T, n1, n2 = 64, 64, 128
    q, s = run_quant(kq, w.x, w.P1, w.P2, w.cinv, 1.0, T, n1, n2)
    A1 = (w.P1.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    A2 = (w.P2.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    I1, I2 = np.linalg.inv(A1), np.linalg.inv(A2)
    c = 1.0 / w.cinv.astype(np.float64)
    xh = torch.empty((T, n1 * n2), dtype=torch.float32, device="cuda")
    qd = torch.from_numpy(q).cuda()
    kq.kq_dequant_inverse(qd, dev_f32(s), dev_f32(I1), dev_f32(I2), dev_f32(c), xh, T, n1, n2)
    torch.cuda.synchronize()
    got = xh.cpu().numpy().astype(np.float64)
    I1f = I1.astype(np.float32).astype(np.float64)
    I2f = I2.astype(np.float32).astype(np.float64)
    ref = oracle.dequant_inverse(q, s, I1f, I2f, c.astype(np.float32).astype(np.float64), n1, n2)
    assert np.abs(got - ref).max() <= 1e-5 * np.abs(ref).max()
    # round trip: within the quantisation error bound of the oracle's own check
    x = (w.x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    colsum = (np.abs(I1).sum(0)[:, None] * np.abs(I2).sum(0)[None, :]).ravel()
    bound = 0.5 * s.astype(np.float64)[:, None] * colsum[None, :] * c[None, :] * 1.001
    assert np.all(np.abs(got - x) <= bound + 1e-4 * np.abs(x).max())


# ---------------------------------------------------------------------------
# Kernel selection and the bounded-wait failure path.

def test_fast_kernel_is_selected_for_the_configs(kq):
    # long launches: the batch-pipelined kernel; short ones of n1 = 64: the pair-pipelined one
    for n1, n2, scaled in [(64, 64, False), (64, 128, True), (112, 128, False)]:
        assert kq.kq_kernel_name(n1, n2, scaled) == "kq_tc05_fused_kernel"
    assert kq.kq_kernel_for(8192, 64, 128, True, 0.85) == "kq_tc05_fused_kernel"   # hidden8192
    assert kq.kq_kernel_for(65536, 64, 64, False, 0.9) == "kq_tc05_fused_kernel"   # sweep4096, largest T
    assert kq.kq_kernel_for(2048, 64, 64, False, 0.88) == "kq_fused_kernel"        # llama7b_hidden
    assert kq.kq_kernel_for(2048, 64, 128, True, 0.85) == "kq_tc05_fused_kernel"   # with cinv: 14 groups per SM
    assert kq.kq_kernel_for(1, 64, 128, True, 0.85) == "kq_fused_kernel"
    assert kq.kq_kernel_for(4096, 112, 128, False, 0.9) == "kq_tc05_fused_kernel"  # mlp14336
    for n1 in (16, 48, 64, 80, 96, 112, 128):  # cinv with n1 > 64; n2 padded to 64 or 128
        for n2 in (16, 32, 48, 64, 80, 96, 112, 128):
            for scaled in (False, True):
                assert kq.kq_kernel_name(n1, n2, scaled) == "kq_tc05_fused_kernel", (n1, n2, scaled)
    assert kq.kq_kernel_for(4096, 64, 80, True, 0.85) == "kq_tc05_fused_kernel"     # hidden5120
    assert kq.kq_kernel_for(64, 16, 16, False, 0.9) == "kq_tc05_fused_kernel"       # tiny
    assert kq.kq_kernel_for(64, 64, 64, False, 1e-7) == "kq_warp_mma_kernel"


def test_bounded_wait_times_out_without_fault(kq):
    """A wait on a barrier nobody signals gives up after the limit, reports its
    site code through the status word, and leaves the context usable."""
    assert kq.kq_device_error() == 0
    kq.kq_selftest_bounded_wait(20000)  # 20 ms
    assert kq.kq_device_error() == 256
    assert kq.kq_device_error() == 0    # read clears it
    w = make_workload("hidden8192", rows=8)
    q, s = run_quant(kq, w.x, w.P1, w.P2, w.cinv, w.alpha, 8, 64, 128)
    assert_quant_parity(w.x, w.P1, w.P2, w.cinv, w.alpha, 64, 128, q, s)
    assert kq.kq_device_error() == 0
