"""libkq — B200-native fused dequant-GEMV over GGUF K-quant weights.

The kernels and the C ABI live in ``csrc/`` and ``include/kq.h``; ``kq`` is
the thin ctypes binding.  Build with ``python -m dequant_quant_gemv_b200.build``.
"""
from . import kq  # noqa: F401

__all__ = ["kq"]
