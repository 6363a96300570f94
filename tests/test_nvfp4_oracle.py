"""Pins of the NVFP4 oracle functions (E2M1 elements, E4M3 block scales of 16
values, one fp32 scale per row) against the formats' definitions and cases
worked by hand; no GPU."""
import numpy as np

import oracle


def test_e2m1_table():
    np.testing.assert_array_equal(oracle.e2m1_values(), [0, 0.5, 1, 1.5, 2, 3, 4, 6])
    codes = np.arange(16)
    v = oracle.e2m1_decode(codes)
    np.testing.assert_array_equal(v[:8], [0, 0.5, 1, 1.5, 2, 3, 4, 6])
    np.testing.assert_array_equal(v[8:], [-0.0, -0.5, -1, -1.5, -2, -3, -4, -6])


def test_e4m3_table():
    v = oracle.e4m3_values()
    assert len(v) == 127 and v[0] == 0 and (np.diff(v) > 0).all()
    assert v[1] == 2.0 ** -9                 # smallest subnormal
    assert v[7] == 7 * 2.0 ** -9             # largest subnormal
    assert v[8] == 2.0 ** -6                 # smallest normal
    assert v[0x38] == 1.0 and v[0x39] == 1.125
    assert v[0x7E] == 448.0                  # largest finite (0x7F is NaN)


def test_e2m1_rounding_cases():
    a = [0.0, 0.2, 0.25, 0.3, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 5.5, 6.0, 7.0, 1e9, -0.75, -0.2, -6.5]
    want = [0, 0, 0, 1, 2, 2, 4, 4, 6, 6, 7, 7, 7, 7, 8 | 2, 0, 8 | 7]
    codes, _ = oracle.e2m1_round(a)
    np.testing.assert_array_equal(codes, want)


def test_e4m3_rounding_cases():
    a = [1 + 1 / 16, 1 + 3 / 16, 448.0, 456.0, 1e6, 0.5 * 2.0 ** -9, 1.5 * 2.0 ** -9, 2.0 ** -6 * (1 + 1 / 32)]
    want = [0x38, 0x3A, 0x7E, 0x7E, 0x7E, 0, 2, 0x08]
    codes, _ = oracle.e4m3_round(a)
    np.testing.assert_array_equal(codes, want)


def test_rounding_picks_a_nearest_entry():
    rng = np.random.default_rng(5)
    for table, rnd in ((oracle.e2m1_values(), lambda a: oracle.e2m1_round(a)[0] & 7),
                       (oracle.e4m3_values(), lambda a: oracle.e4m3_round(a)[0])):
        a = rng.uniform(0, table[-1], 20000)
        got = table[rnd(a)]
        best = np.abs(a[:, None] - table[None, :]).min(axis=1)
        np.testing.assert_allclose(np.abs(a - got), best, rtol=0, atol=1e-15)


def test_hand_row():
    """y = 448 (6, 3, -1.5, 0.75, 0.2, 0 ...): row scale 1, block scale 448
    (code 0x7E), elements 6, 3, -1.5, 1 (0.75 is a tie: even code), 0."""
    y = np.zeros((1, 16))
    y[0, :5] = 448.0 * np.array([6, 3, -1.5, 0.75, 0.2])
    r = oracle.nvfp4_quantize(y)
    assert r["scale32"][0] == 1.0
    assert r["block"][0, 0] == 0x7E
    np.testing.assert_array_equal(r["codes"][0, :6], [7, 5, 8 | 3, 2, 0, 0])
    assert r["packed"][0, 0] == (7 | 5 << 4) and r["packed"][0, 1] == ((8 | 3) | 2 << 4) and r["packed"][0, 2] == 0
    np.testing.assert_array_equal(r["value"][0, :5], 448.0 * np.array([6, 3, -1.5, 1.0, 0]))


def test_quantiser_invariants():
    rng = np.random.default_rng(11)
    y = rng.standard_normal((64, 128)) * np.exp(rng.uniform(-3, 3, (64, 1)))
    y[:, rng.choice(128, 3, replace=False)] *= 20.0
    y[7] = 0.0
    r = oracle.nvfp4_quantize(y)
    s = r["scale32"].astype(np.float64)
    assert s[7] == 0 and (r["codes"][7] == 0).all() and (r["block"][7] == 0).all()
    bdec = oracle.e4m3_decode(r["block"])
    den = np.repeat(bdec * s[:, None], 16, axis=1)
    q = np.abs(y) / np.where(den > 0, den, 1)
    # error bound: at most half the local E2M1 step (no element goes past 6 by more
    # than the block scale's own rounding allows)
    mag = np.abs(oracle.e2m1_decode(r["codes"]))
    table = oracle.e2m1_values()
    hi = np.clip(np.searchsorted(table, np.minimum(q, 6.0)), 1, 7)
    half = 0.5 * (table[hi] - table[hi - 1])
    ok = (np.abs(q - mag) <= half + 1e-12) | (q > 6.0)
    assert ok[den > 0].all()
    # the row's largest block scale is 448 exactly; a block with a normal scale
    # sends its largest element to code magnitude 7 (6)
    nz = s > 0
    assert (r["block"][nz].max(axis=1) == 0x7E).all()
    braw = np.abs(y).reshape(64, 8, 16).max(axis=2) / (6 * np.where(s > 0, s, 1))[:, None]
    normal = (braw >= 2.0 ** -6) & nz[:, None]
    top = (r["codes"].reshape(64, 8, 16) & 7).max(axis=2)
    assert (top[normal] == 7).all()
    # decoded values are the codes times the two scales
    np.testing.assert_array_equal(r["value"], oracle.e2m1_decode(r["codes"]) * den)


def test_headwise_nvfp4_is_rows_times_factor():
    rng = np.random.default_rng(3)
    T, heads, D = 5, 3, 64
    x = rng.standard_normal((T, heads * D)).astype(np.float32)
    P = rng.standard_normal((D, D)).astype(np.float32) / 8
    bits = lambda a: (a.view(np.uint32) >> 16).astype(np.uint16)
    xb, Pb = bits(x), bits(P)
    r = oracle.headwise_transform_nvfp4(xb, Pb, heads, D)
    rows = (xb.astype(np.uint32) << 16).view(np.float32).astype(np.float64).reshape(T * heads, D)
    Pf = (Pb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    ref = oracle.nvfp4_quantize(rows @ Pf)
    for k in ("packed", "block", "scale32"):
        np.testing.assert_array_equal(r[k], ref[k])


def test_e2m1_boundary_distances():
    """Distance to the nearest rounding boundary, in units of the local step
    between the two neighbouring E2M1 magnitudes (the window the NVFP4 parity
    test allows a one-step difference in).  Hand values: 2.5 is the midpoint of
    2 and 3 (0); 2.75 is a quarter step above it (0.25); 5.5 lies between 4 and 6
    (step 2, midpoint 5: 0.25); 0.3 between 0 and 0.5 (step 0.5, midpoint 0.25:
    0.1); 1.0 sits on an entry, half a step from both boundaries (0.5); 3.375
    between 3 and 4 (midpoint 3.5, step 1: 0.125); the sign does not matter;
    6 and beyond saturate (inf: no boundary to be near)."""
    a = np.array([2.5, 2.75, 5.5, 0.3, 1.0, 3.375, -2.75, 6.0, 9.0])
    want = [0.0, 0.25, 0.25, 0.1, 0.5, 0.125, 0.25, np.inf, np.inf]
    _, d = oracle.e2m1_round(a)
    np.testing.assert_allclose(d, want, rtol=0, atol=1e-15)


def test_e4m3_boundary_distances():
    """The same for the E4M3 block scales: 1 + 1/16 is the midpoint of 1 and
    1.125 (0); 1 + 3/32 a quarter step above it (0.25); in the binade [2, 4)
    the step is 0.25, and 2.3125 lies between 2.25 and 2.5, a quarter step below
    their midpoint 2.375 (0.25); 1.25 * 2^-9 between the subnormals 2^-9 and 2^-8 (step 2^-9, midpoint
    1.5 * 2^-9: 0.25); 448 and beyond saturate (inf)."""
    a = np.array([1 + 1 / 16, 1 + 3 / 32, 2.3125, 1.25 * 2.0 ** -9, 448.0, 500.0])
    want = [0.0, 0.25, 0.25, 0.25, np.inf, np.inf]
    _, d = oracle.e4m3_round(a)
    np.testing.assert_allclose(d, want, rtol=0, atol=1e-15)


def test_nvfp4_distances_follow_the_scaled_values():
    """In nvfp4_quantize the element distance is taken on y / (block scale *
    row scale) and the block distance on max|y| / (6 * row scale): one row,
    built so that the row scale is 1 (max|y| = 6 * 448) and the second block's
    raw scale 1 + 3/32 (block distance 0.25, as in the E4M3 table above), and an
    element of the first block at 2.75 * 448 (element distance 0.25)."""
    y = np.zeros((1, 32))
    y[0, 0] = 6.0 * 448.0
    y[0, 1] = 2.75 * 448.0
    y[0, 16] = 6.0 * (1 + 3 / 32)
    r = oracle.nvfp4_quantize(y)
    assert r["scale32"][0] == 1.0
    assert r["block"][0, 0] == 0x7E and r["bdist"][0, 0] == np.inf   # 448 saturates
    assert r["bdist"][0, 1] == 0.25
    assert r["dist"][0, 1] == 0.25
