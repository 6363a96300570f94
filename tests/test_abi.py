"""The C-ABI library: it loads, exports what include/kq.h declares, and rejects
bad arguments on the host before anything is launched (no GPU needed: every
call below fails validation, so no CUDA call is made)."""
import math
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kq.h")


@pytest.fixture(scope="module")
def kq():
    from kronecker_factored_transforms_b200 import build
    build.build()
    from kronecker_factored_transforms_b200 import _lib
    return _lib


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(kq_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for must in ("kq_transform_quant", "kq_transform", "kq_dequant_inverse", "kq_status_string",
                 "kq_kernel_name", "kq_kernel_for", "kq_device_error", "kq_version", "kq_w4a4_gemm", "kq_w4a4_gemm_bf16",
                 "kq_headwise_transform_quant", "kq_transform_quant_two_stage", "kq_two_stage_workspace_bytes",
                 "kq_headwise_transform_quant_nvfp4"):
        assert must in names


def test_library_exports_every_declared_symbol(kq):
    out = subprocess.run(["nm", "-D", "--defined-only", kq.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\bT\s+(kq_[a-z_0-9]+)$", out, flags=re.M))
    for name in declared_functions():
        assert name in exported, name
        getattr(kq.lib, name)


def test_version_and_strings(kq):
    assert kq.kq_version() >= 10000
    for st in range(-7, 1):
        assert kq.kq_status_string(st) not in ("", "unknown status")
    assert kq.kq_status_string(42) == "unknown status"


def test_kernel_name_for_shapes(kq):
    assert kq.kq_kernel_name(16, 16, False) != "unsupported"
    assert kq.kq_kernel_name(64, 128, True) != "unsupported"
    assert kq.kq_kernel_name(112, 128, False) != "unsupported"
    assert kq.kq_kernel_name(24, 16, False) == "unsupported"
    assert kq.kq_kernel_name(16, 144, False) == "unsupported"


def test_kernel_selection_rules(kq):
    """The dispatch rule, host side only (no GPU: kq_kernel_for assumes 148 SMs)."""
    tc, pair, warp = "kq_tc05_fused_kernel", "kq_fused_kernel", "kq_warp_mma_kernel"
    for n2 in (16, 32, 48, 64, 80, 96, 112, 128):  # n2 padded to 64 or 128 columns where needed
        assert kq.kq_kernel_name(112, n2, True) == tc
        assert kq.kq_kernel_name(16, n2, False) == tc
    assert kq.kq_kernel_for(2048, 64, 64, False, 0.88) == pair      # short launch at n1 = 64
    assert kq.kq_kernel_for(148 * 4, 64, 128, True, 0.85) == pair   # with cinv: 4 groups per SM
    assert kq.kq_kernel_for(148 * 4 + 1, 64, 128, True, 0.85) == tc
    assert kq.kq_kernel_for(148 * 56, 64, 128, False, 0.9) == pair  # without: 56 groups per SM
    assert kq.kq_kernel_for(148 * 56 + 1, 64, 128, False, 0.9) == tc
    assert kq.kq_kernel_for(148 * 112, 64, 64, False, 0.9) == pair  # two tokens per group at n2 = 64
    assert kq.kq_kernel_for(148 * 112 + 2, 64, 64, False, 0.9) == tc
    assert kq.kq_kernel_for(16, 64, 80, True, 0.85) == tc           # the pair kernel has n2 in {64, 128} only
    assert kq.kq_kernel_for(16, 112, 128, False, 0.9) == tc
    assert kq.kq_kernel_for(16, 64, 64, False, 2.0 ** -20) == warp  # alpha below 2^-19
    assert kq.kq_kernel_for(16, 24, 64, False, 0.9) == "unsupported"
    # 2^31 rows of x or more: past the 32-bit TMA row coordinates, the warp-MMA kernel
    assert kq.kq_kernel_for(2 ** 31 // 64 - 1, 64, 128, True, 0.85) == tc
    assert kq.kq_kernel_for(2 ** 31 // 64, 64, 128, True, 0.85) == warp


# Fake, never-dereferenced device addresses (validation rejects every call below).
X, P1, P2, CI, Q, S, Y = 0x10000000, 0x20000000, 0x20010000, 0x20020000, 0x30000000, 0x40000000, 0x50000000


def tq(kq, **kw):
    a = dict(x=X, P1=P1, P2=P2, cinv=CI, alpha=0.9, q=Q, s=S, T=8, n1=64, n2=128)
    a.update(kw)
    return kq.lib.kq_transform_quant(a["x"], a["P1"], a["P2"], a["cinv"], a["alpha"], a["q"], a["s"],
                                     a["T"], a["n1"], a["n2"], None)


def test_transform_quant_validation(kq):
    assert tq(kq, T=-1) == kq.KQ_ERR_SHAPE
    assert tq(kq, n1=0) == kq.KQ_ERR_SHAPE
    assert tq(kq, n2=-16) == kq.KQ_ERR_SHAPE
    for bad in (8, 24, 144, 256):
        assert tq(kq, n1=bad) == kq.KQ_ERR_UNSUPPORTED
        assert tq(kq, n2=bad) == kq.KQ_ERR_UNSUPPORTED
    for bad in (0.0, -0.5, 1.0000001, 2.0, math.nan, math.inf):
        assert tq(kq, alpha=bad) == kq.KQ_ERR_ARG
    assert tq(kq, T=2 ** 62) == kq.KQ_ERR_SHAPE
    # T == 0 is a no-op even with NULL pointers.
    assert tq(kq, T=0, x=None, P1=None, P2=None, cinv=None, q=None, s=None) == kq.KQ_OK
    for name in ("x", "P1", "P2", "q", "s"):
        assert tq(kq, **{name: None}) == kq.KQ_ERR_NULL
    for name in ("x", "P1", "P2", "q", "cinv"):
        assert tq(kq, **{name: {"x": X, "P1": P1, "P2": P2, "q": Q, "cinv": CI}[name] + 8}) == kq.KQ_ERR_ALIGN
    assert tq(kq, s=S + 2) == kq.KQ_ERR_ALIGN
    # Outputs overlapping inputs (or each other).
    assert tq(kq, q=X + 64) == kq.KQ_ERR_ARG
    assert tq(kq, s=P1 + 16) == kq.KQ_ERR_ARG
    assert tq(kq, s=Q + 16) == kq.KQ_ERR_ARG
    assert tq(kq, q=CI) == kq.KQ_ERR_ARG


def test_transform_validation(kq):
    f = kq.lib.kq_transform
    assert f(X, P1, P2, None, Y, -3, 64, 64, None) == kq.KQ_ERR_SHAPE
    assert f(X, P1, P2, None, Y, 3, 40, 64, None) == kq.KQ_ERR_UNSUPPORTED
    assert f(X, P1, P2, None, None, 3, 64, 64, None) == kq.KQ_ERR_NULL
    assert f(X, P1, P2, None, Y + 4, 3, 64, 64, None) == kq.KQ_ERR_ALIGN
    assert f(X, P1, P2, None, X + 16, 3, 64, 64, None) == kq.KQ_ERR_ARG
    assert f(None, None, None, None, None, 0, 64, 64, None) == kq.KQ_OK


def test_dequant_inverse_validation(kq):
    f = kq.lib.kq_dequant_inverse
    assert f(Q, S, P1, P2, None, Y, -1, 16, 16, None) == kq.KQ_ERR_SHAPE
    assert f(Q, S, P1, P2, None, Y, 4, 16, 20, None) == kq.KQ_ERR_UNSUPPORTED
    assert f(Q, None, P1, P2, None, Y, 4, 16, 16, None) == kq.KQ_ERR_NULL
    assert f(Q + 1, S, P1, P2, None, Y, 4, 16, 16, None) == kq.KQ_ERR_ALIGN
    assert f(Q, S, P1, P2, None, Q + 32, 4, 16, 16, None) == kq.KQ_ERR_ARG
    assert f(None, None, None, None, None, None, 0, 16, 16, None) == kq.KQ_OK


def test_w4a4_gemm_validation(kq):
    f = kq.lib.kq_w4a4_gemm
    # qx [4, 64], sx [4], qw [8, 64], sw [8], y [4, 8]: fake, well separated, aligned addresses
    qx, sx, qw, sw, y = 0x100000, 0x200000, 0x300000, 0x400000, 0x500000
    assert f(qx, sx, qw, sw, y, -1, 8, 128, None) == kq.KQ_ERR_SHAPE
    assert f(qx, sx, qw, sw, y, 4, -1, 128, None) == kq.KQ_ERR_SHAPE
    for bad_k in (0, 64, 100, 192, 262144 + 128):
        assert f(qx, sx, qw, sw, y, 4, 8, bad_k, None) == kq.KQ_ERR_SHAPE, bad_k
    assert f(qx, None, qw, sw, y, 4, 8, 128, None) == kq.KQ_ERR_NULL
    assert f(qx + 8, sx, qw, sw, y, 4, 8, 128, None) == kq.KQ_ERR_ALIGN
    assert f(qx, sx, qw + 4, sw, y, 4, 8, 128, None) == kq.KQ_ERR_ALIGN
    assert f(qx, sx + 2, qw, sw, y, 4, 8, 128, None) == kq.KQ_ERR_ALIGN
    assert f(qx, sx, qw, sw, qx + 64, 4, 8, 128, None) == kq.KQ_ERR_ARG   # y overlaps qx
    assert f(qx, sx, qw, sw, sw, 4, 8, 128, None) == kq.KQ_ERR_ARG        # y overlaps sw
    assert f(None, None, None, None, None, 0, 8, 128, None) == kq.KQ_OK   # empty: no-op
    assert f(None, None, None, None, None, 4, 0, 128, None) == kq.KQ_OK


def test_headwise_validation(kq):
    f = kq.lib.kq_headwise_transform_quant
    x, P, q, s_ = 0x100000, 0x200000, 0x300000, 0x400000
    assert f(x, P, 0.9, q, s_, -1, 8, 128, None) == kq.KQ_ERR_SHAPE
    assert f(x, P, 0.9, q, s_, 4, 0, 128, None) == kq.KQ_ERR_SHAPE
    assert f(x, P, 0.9, q, s_, 4, 8, 96, None) == kq.KQ_ERR_UNSUPPORTED
    assert f(x, P, 0.9, q, s_, 4, 8, 256, None) == kq.KQ_ERR_UNSUPPORTED
    assert f(x, P, 1.5, q, s_, 4, 8, 128, None) == kq.KQ_ERR_ARG
    assert f(x, P, 0.0, q, s_, 4, 8, 128, None) == kq.KQ_ERR_ARG
    assert f(x, P, 1e-7, q, s_, 4, 8, 128, None) == kq.KQ_ERR_UNSUPPORTED
    assert f(x, None, 0.9, q, s_, 4, 8, 128, None) == kq.KQ_ERR_NULL
    assert f(x + 2, P, 0.9, q, s_, 4, 8, 128, None) == kq.KQ_ERR_ALIGN
    assert f(x, P, 0.9, q + 8, s_, 4, 8, 128, None) == kq.KQ_ERR_ALIGN
    assert f(x, P, 0.9, x + 64, s_, 4, 8, 128, None) == kq.KQ_ERR_ARG   # codes over x
    assert f(x, P, 0.9, q, q + 16, 4, 8, 128, None) == kq.KQ_ERR_ARG    # scales over codes
    assert f(None, None, 0.9, None, None, 0, 8, 128, None) == kq.KQ_OK  # empty: no-op
    assert f(x, P, 0.9, q, s_, 1 << 30, 8, 128, None) == kq.KQ_ERR_SHAPE


def test_headwise_nvfp4_validation(kq):
    f = kq.lib.kq_headwise_transform_quant_nvfp4
    x, P, q, b, s_ = 0x100000, 0x200000, 0x300000, 0x380000, 0x400000
    assert f(x, P, q, b, s_, -1, 8, 128, None) == kq.KQ_ERR_SHAPE
    assert f(x, P, q, b, s_, 4, 8, 96, None) == kq.KQ_ERR_UNSUPPORTED
    assert f(x, None, q, b, s_, 4, 8, 128, None) == kq.KQ_ERR_NULL
    assert f(x, P, q, None, s_, 4, 8, 128, None) == kq.KQ_ERR_NULL
    assert f(x, P, q, b + 4, s_, 4, 8, 128, None) == kq.KQ_ERR_ALIGN
    assert f(x, P, q + 8, b, s_, 4, 8, 128, None) == kq.KQ_ERR_ALIGN
    assert f(x, P, q, q + 64, s_, 4, 8, 128, None) == kq.KQ_ERR_ARG   # block scales over codes
    assert f(x, P, x + 64, b, s_, 4, 8, 128, None) == kq.KQ_ERR_ARG   # codes over x
    assert f(None, None, None, None, None, 0, 8, 128, None) == kq.KQ_OK
    assert f(x, P, q, b, s_, 1 << 30, 8, 128, None) == kq.KQ_ERR_SHAPE


def test_two_stage_validation(kq):
    f = kq.lib.kq_transform_quant_two_stage
    x, P1, P2, c, q, s_, w = 0x1000000, 0x2000000, 0x3000000, 0x4000000, 0x5000000, 0x6000000, 0x10000000
    T, n1, n2 = 4, 256, 256
    need = kq.kq_two_stage_workspace_bytes(T, n1, n2)
    assert need == 4 * T * n1 * n2
    assert kq.kq_two_stage_workspace_bytes(3, 64, 144) == 4 * 3 * 64 * 256   # Z^T rows padded to 128-row slices
    assert kq.kq_two_stage_workspace_bytes(0, 256, 256) == 0 and kq.kq_two_stage_workspace_bytes(-3, 16, 16) == 0
    ok = (x, P1, P2, c, 0.9, q, s_, w, need)
    assert f(*ok[:8], need, -1, n1, n2, None) == kq.KQ_ERR_SHAPE
    assert f(*ok[:8], need, T, 0, n2, None) == kq.KQ_ERR_SHAPE
    for bad in ((272, 256), (256, 24), (8, 64), (64, 512)):
        assert f(*ok[:8], need, T, bad[0], bad[1], None) == kq.KQ_ERR_UNSUPPORTED
    assert f(*ok[:8], need, 1 << 15, 256, 256, None) == kq.KQ_ERR_SHAPE      # T n = 2^31
    assert f(x, P1, P2, c, 1.5, q, s_, w, need, T, n1, n2, None) == kq.KQ_ERR_ARG
    assert f(x, P1, P2, c, 1e-7, q, s_, w, need, T, n1, n2, None) == kq.KQ_ERR_UNSUPPORTED
    assert f(*ok[:8], need - 1, T, n1, n2, None) == kq.KQ_ERR_ARG            # workspace too small
    assert f(x, P1, P2, c, 0.9, q, s_, None, need, T, n1, n2, None) == kq.KQ_ERR_NULL
    assert f(x, P1, P2, c, 0.9, q, s_, w + 8, need, T, n1, n2, None) == kq.KQ_ERR_ALIGN
    assert f(x, P1, P2, c + 4, 0.9, q, s_, w, need, T, n1, n2, None) == kq.KQ_ERR_ALIGN
    assert f(x, P1, P2, c, 0.9, q, s_, x + 1024, need, T, n1, n2, None) == kq.KQ_ERR_ARG   # workspace over x
    assert f(x, P1, P2, c, 0.9, q, s_, q + 16, need, T, n1, n2, None) == kq.KQ_ERR_ARG     # workspace over codes
    assert f(x, P1, P2, c, 0.9, q, q + 64, w, need, T, n1, n2, None) == kq.KQ_ERR_ARG      # scales over codes
    assert f(None, None, None, None, 0.9, None, None, None, 0, 0, n1, n2, None) == kq.KQ_OK  # empty: no-op


def test_device_error_rejects_null(kq):
    assert kq.lib.kq_device_error(None, None) == kq.KQ_ERR_NULL


def test_binding_raises_on_bad_status(kq):
    with pytest.raises(kq.KQError) as e:
        kq.kq_transform_quant(X, P1, P2, None, 0.9, Q, S, 4, 24, 16, stream=0)
    assert e.value.status == kq.KQ_ERR_UNSUPPORTED


def test_build_covers_every_source_and_header():
    """Every .cu file of csrc is compiled into libkq.so and every header counts
    for the rebuild check, so no edit can leave a stale library behind."""
    import os
    from kronecker_factored_transforms_b200 import build as kb
    files = set(os.listdir(kb.CSRC))
    assert {f for f in files if f.endswith(".cu")} == set(kb.SOURCES)
    assert {f for f in files if f.endswith((".cuh", ".h"))} == set(kb.HEADERS)
