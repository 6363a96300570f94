"""ctypes binding to libkq.so -- argument marshalling only.

Every function here has the name of the C entry point it calls (include/kq.h)
and does nothing but turn tensors into pointers, pick the current stream and
raise on a nonzero status.  All arithmetic runs in the CUDA kernels.  If the
library is missing the import fails: there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libkq.so")

KQ_OK = 0
KQ_ERR_NULL = -1
KQ_ERR_SHAPE = -2
KQ_ERR_UNSUPPORTED = -3
KQ_ERR_ALIGN = -4
KQ_ERR_ARG = -5
KQ_ERR_CUDA = -6
KQ_ERR_TIMEOUT = -7


class KQError(RuntimeError):
    def __init__(self, fn: str, status: int, text: str):
        super().__init__("%s failed: %d (%s)" % (fn, status, text))
        self.status = status


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError("libkq.so not built at %s; run __graft_entry__.build() "
                          "(kronecker_factored_transforms_b200/build.py)" % LIB_PATH)
    lib = ctypes.CDLL(LIB_PATH)
    P, I64, I32, F32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float
    lib.kq_transform_quant.argtypes = [P, P, P, P, F32, P, P, I64, I32, I32, P]
    lib.kq_transform.argtypes = [P, P, P, P, P, I64, I32, I32, P]
    lib.kq_dequant_inverse.argtypes = [P, P, P, P, P, P, I64, I32, I32, P]
    lib.kq_device_error.argtypes = [P, ctypes.POINTER(ctypes.c_int)]
    lib.kq_selftest_bounded_wait.argtypes = [I64, P]
    lib.kq_w4a4_gemm.argtypes = [P, P, P, P, P, I64, I64, I64, P]
    lib.kq_w4a4_gemm_bf16.argtypes = [P, P, P, P, P, I64, I64, I64, P]
    lib.kq_headwise_transform_quant.argtypes = [P, P, F32, P, P, I64, I32, I32, P]
    lib.kq_transform_quant_two_stage.argtypes = [P, P, P, P, F32, P, P, P, ctypes.c_uint64, I64, I32, I32, P]
    lib.kq_transform_quant_two_stage_static.argtypes = [P, P, P, P, F32, P, P, I64, I32, I32, P]
    lib.kq_headwise_transform_quant_nvfp4.argtypes = [P, P, P, P, P, I64, I32, I32, P]
    for f in (lib.kq_transform_quant, lib.kq_transform, lib.kq_dequant_inverse, lib.kq_device_error,
              lib.kq_selftest_bounded_wait, lib.kq_w4a4_gemm, lib.kq_w4a4_gemm_bf16, lib.kq_headwise_transform_quant,
              lib.kq_transform_quant_two_stage, lib.kq_transform_quant_two_stage_static,
              lib.kq_headwise_transform_quant_nvfp4):
        f.restype = ctypes.c_int
    lib.kq_two_stage_workspace_bytes.argtypes = [I64, I32, I32]
    lib.kq_two_stage_workspace_bytes.restype = ctypes.c_uint64
    lib.kq_status_string.argtypes = [I32]
    lib.kq_status_string.restype = ctypes.c_char_p
    lib.kq_kernel_name.argtypes = [I32, I32, I32]
    lib.kq_kernel_name.restype = ctypes.c_char_p
    lib.kq_kernel_for.argtypes = [I64, I32, I32, I32, ctypes.c_float]
    lib.kq_kernel_for.restype = ctypes.c_char_p
    lib.kq_version.argtypes = []
    lib.kq_version.restype = ctypes.c_int
    return lib


lib = _load()

EXPORTED = ("kq_transform_quant", "kq_transform", "kq_dequant_inverse", "kq_device_error",
            "kq_selftest_bounded_wait", "kq_status_string", "kq_kernel_name", "kq_kernel_for", "kq_version", "kq_w4a4_gemm",
            "kq_w4a4_gemm_bf16",
            "kq_headwise_transform_quant", "kq_transform_quant_two_stage", "kq_two_stage_workspace_bytes",
            "kq_transform_quant_two_stage_static", "kq_headwise_transform_quant_nvfp4")

STATIC_WORKSPACE_BYTES = 64 * 1024 * 1024


def _ptr(t) -> Optional[int]:
    """Device pointer of a tensor (or an int address, or None)."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream or None
    if isinstance(stream, int):
        return stream or None
    return stream.cuda_stream or None


def _check(fn: str, st: int) -> None:
    if st != KQ_OK:
        raise KQError(fn, st, lib.kq_status_string(st).decode())


def kq_transform_quant(x, P1, P2, cinv, alpha: float, q_out, scale_out, T: int, n1: int, n2: int,
                       stream=None) -> None:
    _check("kq_transform_quant",
           lib.kq_transform_quant(_ptr(x), _ptr(P1), _ptr(P2), _ptr(cinv), float(alpha), _ptr(q_out),
                                  _ptr(scale_out), int(T), int(n1), int(n2), _stream(stream)))


def kq_headwise_transform_quant(x, Ph, alpha: float, q_out, scale_out, T: int, heads: int, head_dim: int,
                                stream=None) -> None:
    _check("kq_headwise_transform_quant",
           lib.kq_headwise_transform_quant(_ptr(x), _ptr(Ph), float(alpha), _ptr(q_out), _ptr(scale_out), int(T),
                                           int(heads), int(head_dim), _stream(stream)))


def kq_two_stage_workspace_bytes(T: int, n1: int, n2: int) -> int:
    return int(lib.kq_two_stage_workspace_bytes(int(T), int(n1), int(n2)))


def kq_transform_quant_two_stage(x, P1, P2, cinv, alpha: float, q_out, scale_out, workspace, workspace_bytes: int,
                                 T: int, n1: int, n2: int, stream=None) -> None:
    _check("kq_transform_quant_two_stage",
           lib.kq_transform_quant_two_stage(_ptr(x), _ptr(P1), _ptr(P2), _ptr(cinv), float(alpha), _ptr(q_out),
                                            _ptr(scale_out), _ptr(workspace), int(workspace_bytes), int(T), int(n1),
                                            int(n2), _stream(stream)))


def kq_transform_quant_two_stage_static(x, P1, P2, cinv, alpha: float, q_out, scale_out, T: int, n1: int, n2: int,
                                        stream=None) -> None:
    _check("kq_transform_quant_two_stage_static",
           lib.kq_transform_quant_two_stage_static(_ptr(x), _ptr(P1), _ptr(P2), _ptr(cinv), float(alpha), _ptr(q_out),
                                                   _ptr(scale_out), int(T), int(n1), int(n2), _stream(stream)))


def kq_headwise_transform_quant_nvfp4(x, Ph, q_out, block_scale_out, scale_out, T: int, heads: int, head_dim: int,
                                      stream=None) -> None:
    _check("kq_headwise_transform_quant_nvfp4",
           lib.kq_headwise_transform_quant_nvfp4(_ptr(x), _ptr(Ph), _ptr(q_out), _ptr(block_scale_out), _ptr(scale_out),
                                                 int(T), int(heads), int(head_dim), _stream(stream)))


def kq_w4a4_gemm(qx, sx, qw, sw, y, M: int, N: int, K: int, stream=None) -> None:
    _check("kq_w4a4_gemm",
           lib.kq_w4a4_gemm(_ptr(qx), _ptr(sx), _ptr(qw), _ptr(sw), _ptr(y), int(M), int(N), int(K),
                            _stream(stream)))


def kq_w4a4_gemm_bf16(qx, sx, qw, sw, y, M: int, N: int, K: int, stream=None) -> None:
    _check("kq_w4a4_gemm_bf16",
           lib.kq_w4a4_gemm_bf16(_ptr(qx), _ptr(sx), _ptr(qw), _ptr(sw), _ptr(y), int(M), int(N), int(K),
                                 _stream(stream)))


def kq_transform(x, P1, P2, cinv, y_out, T: int, n1: int, n2: int, stream=None) -> None:
    _check("kq_transform",
           lib.kq_transform(_ptr(x), _ptr(P1), _ptr(P2), _ptr(cinv), _ptr(y_out), int(T), int(n1),
                            int(n2), _stream(stream)))


def kq_dequant_inverse(q, scale, P1inv, P2inv, c, x_hat, T: int, n1: int, n2: int, stream=None) -> None:
    _check("kq_dequant_inverse",
           lib.kq_dequant_inverse(_ptr(q), _ptr(scale), _ptr(P1inv), _ptr(P2inv), _ptr(c), _ptr(x_hat),
                                  int(T), int(n1), int(n2), _stream(stream)))


def kq_device_error(stream=None) -> int:
    code = ctypes.c_int(0)
    _check("kq_device_error", lib.kq_device_error(_stream(stream), ctypes.byref(code)))
    return code.value


def kq_selftest_bounded_wait(limit_us: int, stream=None) -> None:
    _check("kq_selftest_bounded_wait", lib.kq_selftest_bounded_wait(int(limit_us), _stream(stream)))


def kq_status_string(status: int) -> str:
    return lib.kq_status_string(int(status)).decode()


def kq_kernel_name(n1: int, n2: int, has_cinv: bool) -> str:
    return lib.kq_kernel_name(int(n1), int(n2), int(bool(has_cinv))).decode()


def kq_kernel_for(T: int, n1: int, n2: int, has_cinv: bool, alpha: float = 0.9) -> str:
    return lib.kq_kernel_for(int(T), int(n1), int(n2), int(bool(has_cinv)), float(alpha)).decode()


def kq_version() -> int:
    return int(lib.kq_version())
