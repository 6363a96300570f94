"""Why the operands are split: the precision of x' = x * cinv against the code
window, on a sample of the hidden-size-8192 workload (no GPU).

The tensor cores take 16-bit (or 8-bit) operands, while x' = x * cinv carries
16 significant bits.  These checks round the operands as a kernel would, form
y in fp64 from the rounded operands and compare with the fp64 oracle: the
error of y/s against the path's window (a code may differ by one only where
the oracle's y/s lies within 1e-3 of a rounding boundary):

  * x' rounded to one bf16 value: errors of y/s well beyond 1e-3 and codes
    outside the window -- the reason the fused kernel carries x' (and Z) as a
    hi + lo pair of bf16 values;
  * the hi + lo bf16 pair: errors more than five times inside the window;
  * a candidate with half the lo bytes -- lo in E4M3 with a power-of-two scale
    per 32 values, times P2 rounded the same way -- has errors as large as the
    window itself, so it would need more than this to be safe.
"""
import numpy as np
import pytest

import oracle
from kronecker_factored_transforms_b200.workloads import make_workload

WINDOW = 1e-3


def bf16_rn(a):
    """Round to the nearest bf16 (ties to even), returned as float64."""
    u = np.asarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16
    return r.astype(np.uint32).view(np.float32).astype(np.float64)


def e4m3_block(a, block=32):
    """E4M3 (round to nearest even, saturating) with one power-of-two scale per
    `block` consecutive values of the last axis, chosen so the block maximum
    lands at or below 448."""
    b = np.asarray(a, dtype=np.float64).reshape(-1, block)
    amax = np.abs(b).max(axis=1, keepdims=True)
    e = np.where(amax > 0, np.floor(np.log2(np.where(amax > 0, amax, 1.0) / 448.0)) + 1, 0.0)
    scale = 2.0 ** e
    codes, _ = oracle.e4m3_round(np.abs(b) / scale)   # magnitudes; the sign is carried apart
    return (np.sign(b) * oracle.e4m3_decode(codes) * scale).reshape(np.shape(a))


@pytest.fixture(scope="module")
def sample():
    w = make_workload("hidden8192", rows=256)
    T, n1, n2 = w.x.shape[0], w.n1, w.n2
    widen = lambda bits: (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    x, P1, P2 = widen(w.x), widen(w.P1).reshape(n1, n1), widen(w.P2).reshape(n2, n2)
    xp = x * w.cinv.astype(np.float64)
    ref = oracle.transform_quant(w.x, w.P1, w.P2, w.cinv, w.alpha, n1, n2)
    yref = oracle.transform(w.x, w.P1, w.P2, w.cinv, n1, n2).reshape(T, -1)
    return dict(T=T, n1=n1, n2=n2, xp=xp, P1=P1, P2=P2, alpha=float(np.float32(w.alpha)), ref=ref, yref=yref)


def codes_from_Z(S, Z):
    """Stage 2 as the kernel takes it (Z as a hi + lo bf16 pair), then the
    quantiser in fp64; returns (codes, scales)."""
    Zh = bf16_rn(Z)
    Zl = bf16_rn(Z - Zh)
    Y = np.einsum("ai,taj->tij", S["P1"], Zh + Zl).reshape(S["T"], -1)
    s = S["alpha"] * np.abs(Y).max(axis=1) / 7
    q = np.clip(np.rint(Y / s[:, None]), -8, 7)
    return q, s


def outside_window(S, q):
    ref_codes, dist = S["ref"]["codes"], S["ref"]["dist"]
    diff = q != ref_codes
    bad = diff & ((np.abs(q - ref_codes) != 1) | (dist >= WINDOW))
    return int(bad.sum()), float(diff.mean())


def max_err(S, Z):
    """max |y/s - y_ref/s_ref| with Z taken as a hi + lo bf16 pair in stage 2."""
    Zh = bf16_rn(Z)
    Zl = bf16_rn(Z - Zh)
    Y = np.einsum("ai,taj->tij", S["P1"], Zh + Zl).reshape(S["T"], -1)
    return float(np.max(np.abs(Y - S["yref"]) / S["ref"]["scale64"][:, None]))


def test_single_bf16_x_prime_leaves_the_window(sample):
    S = sample
    Z = bf16_rn(S["xp"]).reshape(S["T"], S["n1"], S["n2"]) @ S["P2"]
    q, _ = codes_from_Z(S, Z)
    bad, _ = outside_window(S, q)
    assert bad > 0 and max_err(S, Z) > 10 * WINDOW


def test_hi_lo_bf16_pair_stays_in_the_window(sample):
    S = sample
    hi = bf16_rn(S["xp"])
    lo = bf16_rn(S["xp"] - hi)
    shape = (S["T"], S["n1"], S["n2"])
    Z = hi.reshape(shape) @ S["P2"] + lo.reshape(shape) @ S["P2"]
    q, s = codes_from_Z(S, Z)
    bad, frac = outside_window(S, q)
    assert bad == 0 and frac <= 1e-3
    assert max_err(S, Z) < WINDOW / 5
    np.testing.assert_allclose(s, S["ref"]["scale64"], rtol=1e-4)


def test_e4m3_lo_candidate_uses_up_the_window(sample):
    S = sample
    hi = bf16_rn(S["xp"])
    lo8 = e4m3_block(S["xp"] - hi)                  # blocks of 32 along j (the contraction)
    P2b = e4m3_block(S["P2"].T.copy()).T            # P2's columns, blocks of 32 along j
    shape = (S["T"], S["n1"], S["n2"])
    Z = hi.reshape(shape) @ S["P2"] + lo8.reshape(shape) @ P2b
    assert max_err(S, Z) > WINDOW / 2


def test_two_stage_intermediate_needs_the_pair():
    """The two-stage path keeps Z^T in its workspace as a hi + lo bf16 pair: on a
    sample of the 256 x 256 workload a single bf16 Z leaves the window, the pair
    does not."""
    w = make_workload("square65536", rows=16)
    T, n1, n2 = w.x.shape[0], w.n1, w.n2
    widen = lambda bits: (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    x, P1, P2 = widen(w.x), widen(w.P1).reshape(n1, n1), widen(w.P2).reshape(n2, n2)
    xp = (x * w.cinv.astype(np.float64)).reshape(T, n1, n2)
    ref = oracle.transform_quant(w.x, w.P1, w.P2, w.cinv, w.alpha, n1, n2)
    alpha = float(np.float32(w.alpha))
    hi = bf16_rn(xp)
    Z = hi @ P2 + bf16_rn(xp - hi) @ P2            # stage 1 with its own hi/lo operand

    def outside(Zq):
        Y = np.einsum("ai,taj->tij", P1, Zq).reshape(T, -1)
        s = alpha * np.abs(Y).max(axis=1) / 7
        q = np.clip(np.rint(Y / s[:, None]), -8, 7)
        diff = q != ref["codes"]
        return int((diff & ((np.abs(q - ref["codes"]) != 1) | (ref["dist"] >= WINDOW))).sum())

    Zh = bf16_rn(Z)
    assert outside(Zh) > 0
    assert outside(Zh + bf16_rn(Z - Zh)) == 0
