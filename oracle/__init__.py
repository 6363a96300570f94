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
