"""Fused Kronecker-factored transform + per-token INT4 quantisation for B200.

The product is the C-ABI library ``libkq.so`` (include/kq.h); this package
holds its CUDA sources (``csrc/``), the build step (``build.py``), a thin
ctypes binding (``_lib``) and the seeded synthetic input generator
(``workloads``).  Importing the binding requires the built library.
"""
__all__ = ["kq_transform_quant", "kq_transform", "kq_dequant_inverse", "kq_device_error",
           "kq_selftest_bounded_wait", "kq_status_string", "kq_kernel_name", "kq_version", "KQError"]


def __getattr__(name):
    # Load libkq lazily so that ``workloads`` and ``build`` import without it.
    if name in __all__:
        from . import _lib
        return getattr(_lib, name)
    raise AttributeError(name)
