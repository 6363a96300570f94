"""fp64 CPU oracle for the fused Kronecker transform + INT4 path.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may import this package; the product path never
does.  The arithmetic lives in ``kq_oracle.c`` (plain C, fp64); this module
builds it with gcc when needed and marshals numpy arrays through ctypes.

Parity status of each function (pins live in ``tests/test_oracle_pins.py``):
  transform         pinned: explicit Kronecker matrix (brute force), exact
                    orthogonal factors (norm), hand-derived golden values,
                    permutation / diagonal / Hadamard special cases.
  quantize          pinned: hand-derived codes incl. ties and clipping,
                    quantiser invariants, high-rate error statistics.
  transform_quant   pinned: equals quantize(transform(.)) exactly.
  dequant_inverse   pinned: round trip against numpy fp64 inverse of the
                    explicit Kronecker matrix.
  w4a4_gemm         pinned: brute-force integer loops on small inputs,
                    hand-derived extreme-code products, scale placement.
  headwise_transform_quant
                    pinned: equals the Kronecker path with P1 = I (one row
                    per head), brute-force per-row quantisation, GQA head
                    counts.
  e2m1_round, e4m3_round, nvfp4_quantize, headwise_transform_nvfp4
                    pinned: the E2M1 and E4M3 value tables (count, extremes,
                    subnormals), ties to even and saturation cases worked by
                    hand, the quantiser's error bound and block-maximum
                    invariants, a hand-computed row.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kq_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libkq_oracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle in place (gcc, -O2, no FP contraction)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + ".tmp.%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fPIC", "-shared", "-o", tmp,
                               _SRC, "-lpthread", "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P = ctypes.c_void_p
            I64, I32, F32 = ctypes.c_int64, ctypes.c_int, ctypes.c_float
            lib.kqo_transform.argtypes = [P, P, P, P, I64, I32, I32, P, I32]
            lib.kqo_quantize.argtypes = [P, I64, I32, F32, P, P, P, P, P, I32]
            lib.kqo_transform_quant.argtypes = [P, P, P, P, F32, I64, I32, I32, P, P, P, P, P, I32]
            lib.kqo_dequant_inverse.argtypes = [P, P, P, P, P, I64, I32, I32, P, I32]
            for f in (lib.kqo_transform, lib.kqo_quantize, lib.kqo_transform_quant,
                      lib.kqo_dequant_inverse):
                f.restype = ctypes.c_int
            _lib = lib
    return _lib


def default_threads() -> int:
    return max(1, len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count() or 1)


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


def _check(st: int, what: str):
    if st != 0:
        raise RuntimeError("oracle %s failed with status %d" % (what, st))


def transform(x_bits, P1_bits, P2_bits, cinv, n1: int, n2: int, nthreads: Optional[int] = None) -> np.ndarray:
    """fp64 y[T, n] = (x * cinv) (P1 (x) P2), row-major vec, via P1^T X~ P2."""
    x = _c(x_bits, np.uint16).reshape(-1, n1 * n2)
    y = np.empty(x.shape, dtype=np.float64)
    st = _load().kqo_transform(_ptr(x), _ptr(_c(P1_bits, np.uint16)), _ptr(_c(P2_bits, np.uint16)),
                               _ptr(_c(cinv, np.float32)), x.shape[0], n1, n2, _ptr(y),
                               nthreads or default_threads())
    _check(st, "transform")
    return y


def quantize(y, alpha: float, nthreads: Optional[int] = None):
    """Per-token INT4 of fp64 rows.  Returns dict(codes, packed, scale64, scale32, dist)."""
    y = _c(y, np.float64)
    T, n = y.shape
    codes = np.empty((T, n), dtype=np.int8)
    packed = np.empty((T, n // 2), dtype=np.uint8)
    s64 = np.empty(T, dtype=np.float64)
    s32 = np.empty(T, dtype=np.float32)
    dist = np.empty((T, n), dtype=np.float64)
    st = _load().kqo_quantize(_ptr(y), T, n, float(alpha), _ptr(codes), _ptr(packed), _ptr(s64),
                              _ptr(s32), _ptr(dist), nthreads or default_threads())
    _check(st, "quantize")
    return dict(codes=codes, packed=packed, scale64=s64, scale32=s32, dist=dist)


def transform_quant(x_bits, P1_bits, P2_bits, cinv, alpha: float, n1: int, n2: int,
                    nthreads: Optional[int] = None, want_codes: bool = True):
    """Fused oracle: packed codes [T, n/2], fp32 scales [T] (+ codes, fp64 scales, dist)."""
    x = _c(x_bits, np.uint16).reshape(-1, n1 * n2)
    T, n = x.shape
    packed = np.empty((T, n // 2), dtype=np.uint8)
    s32 = np.empty(T, dtype=np.float32)
    codes = np.empty((T, n), dtype=np.int8) if want_codes else None
    s64 = np.empty(T, dtype=np.float64)
    dist = np.empty((T, n), dtype=np.float64) if want_codes else None
    st = _load().kqo_transform_quant(_ptr(x), _ptr(_c(P1_bits, np.uint16)), _ptr(_c(P2_bits, np.uint16)),
                                     _ptr(_c(cinv, np.float32)), float(alpha), T, n1, n2,
                                     _ptr(packed), _ptr(s32), _ptr(codes), _ptr(s64), _ptr(dist),
                                     nthreads or default_threads())
    _check(st, "transform_quant")
    return dict(packed=packed, scale32=s32, codes=codes, scale64=s64, dist=dist)


def dequant_inverse(packed, scale, P1inv, P2inv, c, n1: int, n2: int, nthreads: Optional[int] = None) -> np.ndarray:
    """fp64 x^[T, n] = ((q * s) (P1^-1 (x) P2^-1)) * c."""
    q = _c(packed, np.uint8).reshape(-1, n1 * n2 // 2)
    T = q.shape[0]
    xhat = np.empty((T, n1 * n2), dtype=np.float64)
    st = _load().kqo_dequant_inverse(_ptr(q), _ptr(_c(scale, np.float32)), _ptr(_c(P1inv, np.float64)),
                                     _ptr(_c(P2inv, np.float64)), _ptr(_c(c, np.float64)), T, n1, n2,
                                     _ptr(xhat), nthreads or default_threads())
    _check(st, "dequant_inverse")
    return xhat


def unpack_codes(packed) -> np.ndarray:
    """Packed nibbles [T, n/2] -> int8 codes [T, n] (two's complement, low nibble first)."""
    p = np.asarray(packed, dtype=np.uint8)
    lo = (p & 0xF).astype(np.int8)
    hi = (p >> 4).astype(np.int8)
    lo = np.where(lo >= 8, lo - 16, lo).astype(np.int8)
    hi = np.where(hi >= 8, hi - 16, hi).astype(np.int8)
    out = np.empty(p.shape[:-1] + (p.shape[-1] * 2,), dtype=np.int8)
    out[..., 0::2] = lo
    out[..., 1::2] = hi
    return out


def w4a4_gemm(qx_packed, sx, qw_packed, sw) -> np.ndarray:
    """The W4A4 product that consumes the codes (FlatQuant, "Kronecker
    factorization": Q(X P) Q(P^-1 W^T)), in fp64:

        y[m][o] = sx[m] * sw[o] * sum_k qx[m][k] * qw[o][k]

    qx [M, K/2] and qw [N, K/2] packed INT4 (as unpack_codes), sx [M], sw [N]
    fp32.  The integer sum is formed exactly (a float64 matrix product of small
    integers: every partial sum is an integer far below 2^53)."""
    qx = unpack_codes(qx_packed).astype(np.float64)
    qw = unpack_codes(qw_packed).astype(np.float64)
    acc = qx @ qw.T
    return acc * np.asarray(sx, dtype=np.float64)[:, None] * np.asarray(sw, dtype=np.float64)[None, :]


def headwise_transform_quant(x_bits, Ph_bits, alpha: float, heads: int, head_dim: int,
                             nthreads: Optional[int] = None):
    """Per-head transform of the key / value cache (FlatQuant page: P_h and P_v
    keep their full per-head shape; keys and values are transformed per head
    and quantised before storage): every row x[t, h, :] of head_dim values is
    multiplied by the same full factor Ph in fp64, then the INT4 rule of
    ``quantize`` is applied to each (token, head) row on its own.

    Returns dict(packed [T, heads*head_dim/2], scale32 [T, heads], scale64,
    codes [T, heads*head_dim], dist) with rows (t, h) laid out as in x."""
    x = np.asarray(x_bits, dtype=np.uint16).reshape(-1, heads * head_dim)
    T = x.shape[0]
    rows = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64).reshape(T * heads, head_dim)
    P = (np.asarray(Ph_bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    y = rows @ P.reshape(head_dim, head_dim)
    r = quantize(y, alpha, nthreads)
    return dict(packed=r["packed"].reshape(T, heads * head_dim // 2), scale32=r["scale32"].reshape(T, heads),
                scale64=r["scale64"].reshape(T, heads), codes=r["codes"].reshape(T, heads * head_dim),
                dist=r["dist"].reshape(T, heads * head_dim))


# ---------------------------------------------------------------------------
# NVFP4 (the 4-bit floating-point format with two levels of scale that the
# FlatQuant page names as the direction it leaves open; the High-Rate
# Quantized Matrix Multiplication page calls it a multi-scaled format with
# group scaling).  Reading of the format: blocks of 16 consecutive values of a
# row share one E4M3 scale; the elements are E2M1; each row has one fp32 scale.
#
# E2M1: sign, two exponent bits (bias 1), one mantissa bit; the magnitude code
# m = 0 .. 7 encodes 0, 0.5, 1, 1.5, 2, 3, 4, 6.  E4M3: sign, four exponent
# bits (bias 7), three mantissa bits, no infinities, magnitude code 0x7F is NaN:
# the largest finite value is 1.75 * 2^8 = 448, subnormals are m / 8 * 2^-6.

def e2m1_values() -> np.ndarray:
    """Magnitudes of the E2M1 codes 0 .. 7, increasing."""
    out = []
    for m in range(8):
        e, f = m >> 1, m & 1
        out.append(0.5 * f if e == 0 else (1.0 + 0.5 * f) * 2.0 ** (e - 1))
    return np.array(out)


def e4m3_values() -> np.ndarray:
    """Magnitudes of the finite E4M3 codes 0x00 .. 0x7E, increasing."""
    out = []
    for m in range(0x7F):
        e, f = m >> 3, m & 7
        out.append(f / 8.0 * 2.0 ** -6 if e == 0 else (1.0 + f / 8.0) * 2.0 ** (e - 7))
    return np.array(out)


def _round_to_table(a, table):
    """Round non-negative a to the nearest entry of the increasing table (the
    entry's index is the magnitude code); a tie goes to the even code; values
    beyond the last entry saturate to it.  Returns (code, distance of a to the
    nearest rounding boundary in units of the local step; inf when saturated
    beyond the last entry)."""
    a = np.asarray(a, dtype=np.float64)
    top = table[-1]
    sat = a >= top
    ac = np.minimum(a, top)
    hi = np.clip(np.searchsorted(table, ac, side="left"), 0, len(table) - 1)
    lo = np.maximum(hi - 1, 0)
    vh, vl = table[hi], table[lo]
    dh, dl = vh - ac, ac - vl
    pick_hi = (dh < dl) | ((dh == dl) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo)
    step = np.where(hi > lo, vh - vl, 1.0)
    mid = 0.5 * (vh + vl)
    dist = np.where(hi > lo, np.abs(ac - mid) / step, np.inf)
    dist = np.where(sat, np.inf, dist)
    return code.astype(np.int64), dist


def e2m1_round(a):
    """Signed values -> 4-bit E2M1 codes (bit 3 the sign), round to nearest even,
    saturating at +-6; also the distance to the nearest rounding boundary."""
    a = np.asarray(a, dtype=np.float64)
    m, dist = _round_to_table(np.abs(a), e2m1_values())
    sign = (a < 0) & (m > 0)
    return (m | (sign.astype(np.int64) << 3)).astype(np.uint8), dist


def e4m3_round(a):
    """Non-negative values -> E4M3 codes, round to nearest even, saturating at
    448; also the distance to the nearest rounding boundary."""
    m, dist = _round_to_table(np.asarray(a, dtype=np.float64), e4m3_values())
    return m.astype(np.uint8), dist


def e2m1_decode(codes) -> np.ndarray:
    c = np.asarray(codes, dtype=np.int64)
    v = e2m1_values()[c & 7]
    return np.where(c & 8, -v, v)


def e4m3_decode(codes) -> np.ndarray:
    return e4m3_values()[np.asarray(codes, dtype=np.int64) & 0x7F]


def nvfp4_quantize(y):
    """NVFP4 of fp64 rows y [R, D] (D a multiple of 16), step by step:
      1. row scale  s = max|y| / (6 * 448), rounded to fp32;
      2. block scale  b = E4M3(max over the block of |y| / (6 s)), per 16 values;
      3. element  q = E2M1(y / (decode(b) * s));
      4. two codes per byte, element 2k in the low nibble.
    A row (block) whose scale is zero gets zero block codes (element codes).
    Returns dict(packed [R, D/2] uint8, codes [R, D] uint8, block [R, D/16] uint8,
    scale32 [R] fp32, dist [R, D] (element rounding), bdist [R, D/16]
    (block-scale rounding), value [R, D] (the decoded values))."""
    y = np.asarray(y, dtype=np.float64)
    R, D = y.shape
    assert D % 16 == 0
    s32 = (np.abs(y).max(axis=1) / (6.0 * 448.0)).astype(np.float32) if D else np.zeros(R, np.float32)
    s = s32.astype(np.float64)
    yb = y.reshape(R, D // 16, 16)
    amax_b = np.abs(yb).max(axis=2)
    with np.errstate(divide="ignore", invalid="ignore"):
        braw = np.where(s[:, None] > 0, amax_b / (6.0 * s[:, None]), 0.0)
    bcode, bdist = e4m3_round(braw)
    bdec = e4m3_decode(bcode)
    den = bdec * s[:, None]
    with np.errstate(divide="ignore", invalid="ignore"):
        r = np.where(den[:, :, None] > 0, yb / den[:, :, None], 0.0)
    codes, dist = e2m1_round(r)
    codes = codes.reshape(R, D)
    dist = dist.reshape(R, D)
    packed = (codes[:, 0::2] & 0xF) | ((codes[:, 1::2] & 0xF) << 4)
    value = (e2m1_decode(codes).reshape(R, D // 16, 16) * den[:, :, None]).reshape(R, D)
    return dict(packed=packed.astype(np.uint8), codes=codes, block=bcode, scale32=s32, dist=dist, bdist=bdist,
                value=value)


def headwise_transform_nvfp4(x_bits, Ph_bits, heads: int, head_dim: int):
    """The per-head transform of ``headwise_transform_quant`` (rows x[t, h, :] times
    the full factor Ph, fp64) followed by ``nvfp4_quantize`` of every (token,
    head) row.  Returns the dict of ``nvfp4_quantize`` with rows (t, h) in order."""
    x = np.asarray(x_bits, dtype=np.uint16).reshape(-1, heads * head_dim)
    T = x.shape[0]
    rows = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64).reshape(T * heads, head_dim)
    P = (np.asarray(Ph_bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return nvfp4_quantize(rows @ P.reshape(head_dim, head_dim))
