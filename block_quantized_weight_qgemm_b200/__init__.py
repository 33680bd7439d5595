"""Block-quantized-weight x bf16-activation GEMM for NVIDIA B200 (sm_100a).

The compute lives in ``libqgemm.so`` (hand-written CUDA behind a C ABI declared in
``include/qgemm.h``).  ``qgemm`` is its thin Python binding; importing this package
does not load the library -- the first call does, and raises if it is missing.
"""
from . import inputs  # noqa: F401

__all__ = ["inputs"]
