"""B200-native two-level sparse decode attention (AsyncTLS hot path).

The compute path is libtls.so (CUDA for sm_100a, C ABI in include/tls.h);
``tls`` is its ctypes binding and ``runtime.DecodeState`` keeps one layer's
buffers resident on the device.
"""

from . import tls  # noqa: F401

__all__ = ["tls"]
