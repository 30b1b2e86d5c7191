"""B200-native W4A16 group-128 linear layer.

The compute lives in the CUDA library ``libw4a16.so`` (sources in ``csrc/``,
C-ABI in ``include/w4a16.h``).  ``gemm_w4a16_b200.w4a16`` is the thin ctypes
binding with the same entry-point names; importing this package loads nothing
until an entry point is called.
"""

__all__ = ["w4a16", "synth"]
