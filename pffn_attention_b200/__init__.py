"""B200-native Generalized Dot-Product Attention (GDPA).

The compute path is the CUDA library ``libgdpa.so`` (sm_100a kernels behind
the C ABI of ``include/gdpa.h``); ``pffn_attention_b200.gdpa`` is its ctypes
binding.  Build with ``python -m pffn_attention_b200.build``.
"""
from . import gdpa  # noqa: F401

__all__ = ["gdpa"]
